"""Throughput of the H3-Omni block step on B200: packed tokens/s per block.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

The default workload is the longest single-GPU one, 768x1792_15s (124,016
packed tokens: 21:9 768x1792, 15 s at 24 fps, stereo audio, 512 text tokens);
768sq_2s and 768x1344_5s are the same line with --workload.
One step = the whole hot path once over one packed sequence: patchify + pack +
per-modality input projections, one full-width block (LN+modulate, QKV with
Q/K RMSNorm + 3-D RoPE, attention, gated out-projection, LN+modulate, gated
SwiGLU FFN), and the output head with the two Euler updates (video, audio)
in its GEMM epilogues (h3_head_euler).
Every rank processes its own sequence (independent requests, no collective):
weak scaling, value = tokens of all ranks / max-over-ranks time.

--impl reference times the float64 CPU oracle on a bounded sample of the same
workload (the reference arm of this comparison; it is not tuned).

--sp times sequence parallelism instead: one sequence split over the job's
ranks (strong scaling; its own line).
Separate lines (one GPU each, not the headline): --e4m3 (the block's four
GEMMs on e4m3 operands; with --qk-e4m3 also attention's Q K^T on e4m3
codes), --sampler (the 50-block, 8-step layered sampler on 768x1344_5s;
combinable with --e4m3 [--qk-e4m3]), --only CALL (one C-ABI call alone, for
ncu captures; prints a timing line, not the JSON contract line; --heads H
runs it with H heads instead of the workload's, for captures that must stay
small).

Roofline peaks: a timed region of a second or more runs under the 1 kW power
cap, so its fractions are against the measured sustained bf16 matmul figure;
a shorter one against the measured burst figure.  Every kernel also carries
its fraction of the burst figure and of the 2.25 PFLOP/s dense bf16 spec.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed tokens/s per Omni block (bf16, 1×B200) & % of dense bf16 tensor peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "768x1792_15s"
BF16_SPEC_TFLOPS = 2250.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def flops_per_call(w, L):
    """Algorithmic FLOPs of each C-ABI call at L valid tokens (no padding)."""
    D, I, F = w.D, w.I, w.F
    return {
        "h3_qkv_qknorm_mrope": 2.0 * L * D * 3 * I,
        "h3_attention": 4.0 * L * L * I,
        "h3_gated_residual": 2.0 * L * I * D,
        "h3_ffn_swiglu": 2.0 * L * D * 2 * F + 2.0 * L * F * D,
    }


def bytes_per_call(w, L, Lp):
    """Algorithmic HBM bytes of the memory-bound calls."""
    D = w.D
    n_lat = w.T_lat * w.H_lat * w.W_lat * w.C_lat + w.audio_channels * w.n_audio * w.C_audio
    n_gen = w.audio_channels * w.n_audio + w.T_lat * (w.H_lat // 2) * (w.W_lat // 2)   # audio + video rows
    return {
        "h3_adaln_norm_modulate": L * (4 * D + 2 * D) + (Lp - L) * 2 * D,
        # head + Euler: LN of the generated rows (read x fp32, write hn bf16),
        # the head GEMMs read hn and their weights, each latent element is read
        # and written once (fp32); the velocity never goes to memory
        "h3_head_euler": n_gen * (4 * D + 2 * D) + n_gen * 2 * D + (4 * w.C_lat + w.C_audio) * D * 2 + 8 * n_lat,
    }


# DRAM bytes (read + write) per launch from one ncu capture of the kernel on
# this workload (dram__bytes_read.sum + dram__bytes_write.sum), valid for the
# kernel as it was when captured.
TRAFFIC = {
    # mean over the block's QKV, out-projection, FFN gate/up and FFN down
    # launches (6.156 GB / 4)
    ("768sq_2s", "gemm_tc_kernel"): 1.539e9,
    # the same four launches with e4m3 operands (2.679 GB / 4)
    ("768sq_2s", "gemm_tc_kernel<e4m3>"): 0.670e9,
    # one attention launch at 124,016 tokens: DRAM read + write of a 2-head
    # launch (493.0 MB + 60.3 MB) times 28 for the 56 heads (heads are
    # independent CTAs, scheduled head after head, so the traffic grows with
    # them); q, k, v, o alone are 7.11 GB, the rest is K and V re-read by
    # CTAs that started at different times
    ("768x1792_15s", "attention_split_kernel"): 15.49e9,
    # the same with e4m3 q, k codes (2 of 16 exponentials on the FMA pipe):
    # 178.3 MB + 48.0 MB for 2 heads, times 28
    ("768x1792_15s", "attention_split_kernel<e4m3 QK>"): 6.34e9,
    # mean over the block's four pair-GEMM launches at 32,160 tokens
    # (39.65 GB / 4: A panels re-read per pass of the concurrent tiles, B once
    # per band, the outputs); every term grows with the rows, so 124,016
    # tokens take that times 124,016 / 32,160
    ("768x1344_5s", "gemm_tc_kernel"): 9.91e9,
    ("768x1792_15s", "gemm_tc_kernel"): 38.2e9,
}


def peak_for_region(peaks, region_s):
    """(peak TFLOP/s, its name) for a timed region of region_s seconds: the
    sustained figure once the region runs long enough to settle under the
    power cap (>= 1 s), else the burst figure."""
    if region_s >= 1.0:
        return peaks["bf16_tflops_sustained"], f"bf16 sustained, of {peaks['source']} (timed region {region_s:.1f} s)"
    return peaks["bf16_tflops"], f"bf16 burst, of {peaks['source']} (timed region {region_s:.2f} s)"


def kernel_entry(ms, launches, tflops, peak_tf, peaks, traffic):
    return {"ms_per_step": round(ms, 4), "launches_per_step": launches, "tflops": round(tflops, 1),
            "frac": round(tflops / peak_tf, 4), "frac_of_burst": round(tflops / peaks["bf16_tflops"], 4),
            "frac_of_spec_2250": round(tflops / BF16_SPEC_TFLOPS, 4), "traffic_per_launch": traffic}


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) == 7:
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[3:]))
                except ValueError:
                    pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def max_over_ranks(values, device=None):
    """Element-wise maximum of per-rank timings over the process group (the
    slowest rank sets a multi-GPU time).  Works for any backend; identity
    without an initialised group."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Units of all ranks per second when every rank processes its own
    units_per_rank in ms_per_step (the max over ranks)."""
    return world * units_per_rank / (ms_per_step / 1e3)


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    from omni_modal_diffusion_b200 import h3
    from omni_modal_diffusion_b200.pipeline import H3BlockStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + w.index + 7919 * rank)

    def randn(*shape, std=1.0, dtype=torch.bfloat16):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(dtype)

    # random-init weights of the block's architecture, N(0, 0.02), bf16
    W = {"W_text": randn(w.D, w.D_text, std=0.02), "W_vid": randn(w.D, 4 * w.C_lat, std=0.02),
         "W_aud": randn(w.D, w.C_audio, std=0.02), "Wqkv": randn(3 * w.I, w.D, std=0.02),
         "qn_w": (1 + 0.1 * torch.randn(128, generator=g, device=dev)).to(torch.bfloat16),
         "kn_w": (1 + 0.1 * torch.randn(128, generator=g, device=dev)).to(torch.bfloat16),
         "Wo": randn(w.D, w.I, std=0.02), "Wgu": randn(2 * w.F, w.D, std=0.02), "Wd": randn(w.D, w.F, std=0.02),
         "W_vhead": randn(4 * w.C_lat, w.D, std=0.02), "W_ahead": randn(w.C_audio, w.D, std=0.02)}
    st = H3BlockStep(w, device=dev, weights=W)
    if getattr(args, "qk_prologue", False):
        st.qk_flags = 0  # raw q, k; norm + RoPE in attention's prologue
    L, Lp = st.ranges.L, st.ranges.L_pad
    text = randn(w.n_text, w.D_text)
    video = randn(w.T_lat, w.H_lat, w.W_lat, w.C_lat)
    audio = randn(w.audio_channels, w.n_audio, w.C_audio)
    mod = randn(3, 6, w.D, std=0.1, dtype=torch.float32)
    lat_v = randn(w.T_lat, w.H_lat, w.W_lat, w.C_lat, dtype=torch.float32)
    lat_a = randn(w.audio_channels, w.n_audio, w.C_audio, dtype=torch.float32)
    sv = h3.h3_sigma_schedule(8, 12.0)
    sa = h3.h3_sigma_schedule(8, 3.0)
    stream = torch.cuda.current_stream(dev)

    calls = ["h3_embed_pack", "h3_adaln_norm_modulate", "h3_qkv_qknorm_mrope", "h3_attention",
             "h3_gated_residual", "h3_adaln_norm_modulate#2", "h3_ffn_swiglu", "h3_head_euler"]

    def step(i, ev=None):
        s = i % 8
        mark = (lambda k, j: ev[k][j].record(stream)) if ev is not None else (lambda k, j: None)
        d, r = st.dims, st.ranges
        mark(0, 0); st.embed(text, video, audio); mark(0, 1)
        mark(1, 0); h3.h3_adaln_norm_modulate(d, r, st.x, mod, h3.H3_MSA, st.xm); mark(1, 1)
        mark(2, 0)
        h3.h3_qkv_qknorm_mrope(d, r, st.xm, st.W["Wqkv"], st.W["qn_w"], st.W["kn_w"], st.pos, st.q, st.k, st.v,
                               flags=st.qk_flags)
        mark(2, 1)
        mark(3, 0)
        h3.h3_attention(d, r, st.q, st.k, st.v, st.o, qn_w=st.W["qn_w"], kn_w=st.W["kn_w"], pos=st.pos,
                        flags=st.qk_flags)
        mark(3, 1)
        mark(4, 0); h3.h3_gated_residual(d, r, st.x, st.o, st.W["Wo"], mod, h3.H3_MSA); mark(4, 1)
        mark(5, 0); h3.h3_adaln_norm_modulate(d, r, st.x, mod, h3.H3_MLP, st.xm); mark(5, 1)
        mark(6, 0); h3.h3_ffn_swiglu(d, r, st.x, st.xm, st.W["Wgu"], st.W["Wd"], mod, st.ws); mark(6, 1)
        mark(7, 0); st.head_euler(lat_v, lat_a, (sv[s], sv[s + 1]), (sa[s], sa[s + 1])); mark(7, 1)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for i in range(args.warmup):
        step(i)
    barrier()
    sampler = ClockSampler(local) if rank == 0 or world == 1 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in calls] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    t0.record(stream)
    for i in range(args.steps):
        step(i, ev[i])
    t1.record(stream)
    barrier()
    clocks = sampler.stop() if sampler else None
    ms_total = t0.elapsed_time(t1)
    per_call = {c: statistics.mean(ev[i][k][0].elapsed_time(ev[i][k][1]) for i in range(args.steps))
                for k, c in enumerate(calls)}
    status = h3.h3_device_status()
    if status != 0:
        raise RuntimeError(f"device-side wait gave up (code {status})")

    # ---- end to end: host buffers in pinned memory, every step's H2D of its
    # inputs and D2H of its updated latents inside the timed region.  The
    # copies run on two side streams into double-buffered device inputs, so
    # step i+1's inputs and step i's results move while step i computes.
    host_in = {k: t.cpu().pin_memory() for k, t in (("text", text), ("video", video), ("audio", audio), ("mod", mod),
                                                      ("lat_v", lat_v), ("lat_a", lat_a))}
    dev_in = [{k: torch.empty_like(t, device=dev) for k, t in host_in.items()} for _ in range(2)]
    host_out = {k: torch.empty_like(host_in[k]).pin_memory() for k in ("lat_v", "lat_a")}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n, start):
        """n end-to-end steps, enqueued after `start` (an event on stream);
        returns once the last D2H is ordered before stream's next work."""
        def h2d_copy(i):
            b = i & 1
            copy_in.wait_event(start)
            if i >= 2:  # buffer b was last read by step i-2's compute and D2H
                copy_in.wait_event(done[b])
                copy_in.wait_event(out_done[b])
            with torch.cuda.stream(copy_in):
                for k in host_in:
                    dev_in[b][k].copy_(host_in[k], non_blocking=True)
            in_ready[b].record(copy_in)

        h2d_copy(0)
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                h2d_copy(i + 1)
            stream.wait_event(in_ready[b])
            s = i % 8
            d = dev_in[b]
            st.step(d["text"], d["video"], d["audio"], d["mod"], d["lat_v"], d["lat_a"], (sv[s], sv[s + 1]),
                    (sa[s], sa[s + 1]))
            done[b].record(stream)
            copy_out.wait_event(done[b])
            with torch.cuda.stream(copy_out):
                host_out["lat_v"].copy_(d["lat_v"], non_blocking=True)
                host_out["lat_a"].copy_(d["lat_a"], non_blocking=True)
            out_done[b].record(copy_out)
        stream.wait_event(out_done[(n - 1) & 1])

    w0 = torch.cuda.Event()
    w0.record(stream)
    e2e_run(2, w0)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps, e0)
    e1.record(stream)
    barrier()
    ms_e2e = e0.elapsed_time(e1)
    # the last step's result as it arrived on the host equals the device copy
    if not (torch.equal(host_out["lat_v"], dev_in[(args.steps - 1) & 1]["lat_v"].cpu())
            and torch.equal(host_out["lat_a"], dev_in[(args.steps - 1) & 1]["lat_a"].cpu())):
        raise RuntimeError("end-to-end result copy mismatch")

    # max over ranks
    ms_total, ms_e2e = max_over_ranks([ms_total, ms_e2e], device=dev)
    per_call = dict(zip(calls, max_over_ranks([per_call[c] for c in calls], device=dev)))
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None

    ms_step = ms_total / args.steps
    value = job_throughput(world, L, ms_step)
    e2e_value = job_throughput(world, L, ms_e2e / args.steps)
    peaks = _peaks()
    fl = flops_per_call(w, L)
    by = bytes_per_call(w, L, Lp)
    tensor_calls = {c: fl[c] / (per_call[c] / 1e3) / 1e12 for c in fl}
    peak_tf, peak_kind = peak_for_region(peaks, ms_total / 1e3)
    # Kernels: the tcgen05 GEMM (gemm_tc2_kernel, CTA pairs, for QKV and the
    # out-projection; gemm_tc_kernel for the FFN's gate/up and down) runs the
    # block's four GEMM launches (the embed/head launches add < 0.4% of its
    # FLOPs and are not timed separately).  h3_attention with the norm
    # weights is attention_split_kernel plus the general kernel's fixup launch
    # (whose CTAs return at once unless the split kernel left them work).
    gemm_calls = ("h3_qkv_qknorm_mrope", "h3_gated_residual", "h3_ffn_swiglu")
    gemm_ms = sum(per_call[c] for c in gemm_calls)
    gemm_tf = sum(fl[c] for c in gemm_calls) / (gemm_ms / 1e3) / 1e12
    attn_tf = tensor_calls["h3_attention"]
    kernels = {"gemm_tc_kernel": kernel_entry(gemm_ms, 4, gemm_tf, peak_tf, peaks,
                                              TRAFFIC.get((w.name, "gemm_tc_kernel"))),
               "attention_split_kernel": kernel_entry(per_call["h3_attention"], 1, attn_tf, peak_tf, peaks,
                                                      TRAFFIC.get((w.name, "attention_split_kernel")))}
    dominant = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    block_flops = sum(fl.values())
    block_ms = sum(per_call[c] for c in ("h3_adaln_norm_modulate", "h3_qkv_qknorm_mrope", "h3_attention",
                                         "h3_gated_residual", "h3_adaln_norm_modulate#2", "h3_ffn_swiglu"))
    # the two LN + modulate launches of the block (attention and FFN branch)
    ln_each = [by["h3_adaln_norm_modulate"] / (per_call[c] / 1e3) / 1e9
               for c in ("h3_adaln_norm_modulate", "h3_adaln_norm_modulate#2")]
    ln_gbs = 2 * by["h3_adaln_norm_modulate"] / ((per_call["h3_adaln_norm_modulate"]
                                                  + per_call["h3_adaln_norm_modulate#2"]) / 1e3) / 1e9
    head_gbs = by["h3_head_euler"] / (per_call["h3_head_euler"] / 1e3) / 1e9
    launches = st.launches_per_step()
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) latents/text, N(0,0.02) random-init weights)",
        "config": {"workload": w.name, "packed_tokens": L, "L_pad": Lp, "hidden": w.D, "heads": w.H, "head_dim": 128,
                   "ffn": w.F, "text_tokens": w.n_text, "audio_tokens": w.audio_channels * w.n_audio,
                   "video_tokens": st.n_video, "video_latent": [w.T_lat, w.H_lat, w.W_lat, w.C_lat],
                   "parallelism": f"replicas x{world} (independent sequences)",
                   "qk_norm_rope": "attention prologue" if st.qk_flags == 0 else "QKV epilogue",
                   "l2": "inputs larger than L2: %.0f MB of weights + %.0f MB residual stream read per step" % (
                       sum(t.numel() * 2 for t in W.values()) / 1e6, Lp * w.D * 4 / 1e6)},
        "roofline": {"bound": "tensor", "kernel": dominant,
                     "achieved": kernels[dominant]["tflops"],
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": kernels[dominant]["frac"],
                     "peak_kind": peak_kind, "frac_of_burst": kernels[dominant]["frac_of_burst"],
                     "frac_of_spec_2250": kernels[dominant]["frac_of_spec_2250"],
                     "traffic": TRAFFIC.get((w.name, dominant))},
        "kernels": kernels,
        "block": {"tflops": round(block_flops / (block_ms / 1e3) / 1e12, 1),
                  "frac": round(block_flops / (block_ms / 1e3) / 1e12 / peak_tf, 4),
                  "frac_of_burst": round(block_flops / (block_ms / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
                  "frac_of_spec_2250": round(block_flops / (block_ms / 1e3) / 1e12 / BF16_SPEC_TFLOPS, 4),
                  "ms": round(block_ms, 4)},
        "per_call_ms": {c: round(v, 4) for c, v in per_call.items()},
        "per_call_tflops": {c: round(v, 1) for c, v in tensor_calls.items()},
        "ln_modulate_gbs": round(ln_gbs, 1), "ln_modulate_frac_hbm": round(ln_gbs / peaks["hbm_gbs"], 4),
        "ln_modulate_per_launch_gbs": [round(v, 1) for v in ln_each],
        "head_euler_gbs": round(head_gbs, 1), "head_euler_frac_hbm": round(head_gbs / peaks["hbm_gbs"], 4),
        "gpu_launches": launches * args.steps,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    return out


def run_e4m3(args, w):
    """The block step with its four GEMMs on e4m3 operands (per-token and
    per-output-channel scales, fp32 accumulate) and attention in bf16.  A
    separate line: the headline metric is the bf16 step.  One GPU."""
    import torch
    from omni_modal_diffusion_b200 import h3
    from omni_modal_diffusion_b200.pipeline import H3BlockStep

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + w.index)

    def randn(*shape, std=1.0, dtype=torch.bfloat16):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(dtype)

    W = {"W_text": randn(w.D, w.D_text, std=0.02), "W_vid": randn(w.D, 4 * w.C_lat, std=0.02),
         "W_aud": randn(w.D, w.C_audio, std=0.02), "Wqkv": randn(3 * w.I, w.D, std=0.02),
         "qn_w": (1 + 0.1 * torch.randn(128, generator=g, device=dev)).to(torch.bfloat16),
         "kn_w": (1 + 0.1 * torch.randn(128, generator=g, device=dev)).to(torch.bfloat16),
         "Wo": randn(w.D, w.I, std=0.02), "Wgu": randn(2 * w.F, w.D, std=0.02), "Wd": randn(w.D, w.F, std=0.02),
         "W_vhead": randn(4 * w.C_lat, w.D, std=0.02), "W_ahead": randn(w.C_audio, w.D, std=0.02)}
    st = H3BlockStep(w, device=dev, weights=W)
    W8 = st.quantize_block_weights_e4m3()
    st.alloc_e4m3()
    L, Lp = st.ranges.L, st.ranges.L_pad
    text = randn(w.n_text, w.D_text)
    video = randn(w.T_lat, w.H_lat, w.W_lat, w.C_lat)
    audio = randn(w.audio_channels, w.n_audio, w.C_audio)
    mod = randn(3, 6, w.D, std=0.1, dtype=torch.float32)
    lat_v = randn(w.T_lat, w.H_lat, w.W_lat, w.C_lat, dtype=torch.float32)
    lat_a = randn(w.audio_channels, w.n_audio, w.C_audio, dtype=torch.float32)
    sv = h3.h3_sigma_schedule(8, 12.0)
    sa = h3.h3_sigma_schedule(8, 3.0)
    stream = torch.cuda.current_stream(dev)
    calls = ["h3_embed_pack", "h3_adaln_norm_modulate_e4m3", "h3_qkv_qknorm_mrope_e4m3", "h3_attention",
             "h3_quantize_rows_e4m3", "h3_gated_residual_e4m3", "h3_adaln_norm_modulate_e4m3#2",
             "h3_ffn_swiglu_e4m3", "h3_head_euler"]

    # --qk-e4m3: q, k cross to attention as e4m3 codes (H3_QK_E4M3)
    qk_flags = h3.H3_QK_NORM_ROPE_IN_QKV | (h3.H3_QK_E4M3 if args.qk_e4m3 else 0)
    qb, kb = (st.q8, st.k8) if args.qk_e4m3 else (st.q, st.k)

    def step(i, ev=None):
        s = i % 8
        mark = (lambda k, j: ev[k][j].record(stream)) if ev is not None else (lambda k, j: None)
        d, r = st.dims, st.ranges
        mark(0, 0); st.embed(text, video, audio); mark(0, 1)
        mark(1, 0); h3.h3_adaln_norm_modulate_e4m3(d, r, st.x, mod, h3.H3_MSA, st.xq, st.xs); mark(1, 1)
        mark(2, 0)
        h3.h3_qkv_qknorm_mrope_e4m3(d, r, st.xq, st.xs, W8["Wqkv"], W8["Wqkv_s"], W8["qn_w"], W8["kn_w"], st.pos,
                                    qb, kb, st.v, flags=qk_flags)
        mark(2, 1)
        mark(3, 0)
        h3.h3_attention(d, r, qb, kb, st.v, st.o, qn_w=W8["qn_w"], kn_w=W8["kn_w"], flags=qk_flags)
        mark(3, 1)
        mark(4, 0); h3.h3_quantize_rows_e4m3(st.o, st.oq, st.os); mark(4, 1)
        mark(5, 0); h3.h3_gated_residual_e4m3(d, r, st.x, st.oq, st.os, W8["Wo"], W8["Wo_s"], mod); mark(5, 1)
        mark(6, 0); h3.h3_adaln_norm_modulate_e4m3(d, r, st.x, mod, h3.H3_MLP, st.xq, st.xs); mark(6, 1)
        mark(7, 0)
        h3.h3_ffn_swiglu_e4m3(d, r, st.x, st.xq, st.xs, W8["Wgu"], W8["Wgu_s"], W8["Wd"], W8["Wd_s"], mod, st.ws8)
        mark(7, 1)
        mark(8, 0); st.head_euler(lat_v, lat_a, (sv[s], sv[s + 1]), (sa[s], sa[s + 1])); mark(8, 1)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in calls] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for i in range(args.steps):
        step(i, ev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    status = h3.h3_device_status()
    if status != 0:
        raise RuntimeError(f"device-side wait gave up (code {status})")
    ms_step = t0.elapsed_time(t1) / args.steps
    per_call = {c: statistics.mean(ev[i][k][0].elapsed_time(ev[i][k][1]) for i in range(args.steps))
                for k, c in enumerate(calls)}
    peaks = _peaks()
    # e4m3 peak: the measured bf16 figure for this region's length times the
    # nominal 2x of the dense e4m3 / bf16 tensor rates
    peak16 = peak_for_region(peaks, ms_step * args.steps / 1e3)[0]
    peak_f8 = 2.0 * peak16
    fl = flops_per_call(w, L)
    gemm = {"h3_qkv_qknorm_mrope_e4m3": fl["h3_qkv_qknorm_mrope"], "h3_gated_residual_e4m3": fl["h3_gated_residual"],
            "h3_ffn_swiglu_e4m3": fl["h3_ffn_swiglu"]}
    gemm_ms = sum(per_call[c] for c in gemm)
    gemm_tf = sum(gemm.values()) / (gemm_ms / 1e3) / 1e12
    block_ms = sum(per_call[c] for c in calls[1:8])
    attn_tf = fl["h3_attention"] / (per_call["h3_attention"] / 1e3) / 1e12
    # e4m3 Q K^T at twice the bf16 rate and bf16 P V: half the FLOPs each,
    # so the attention's own peak is 2 / (1/2 + 1) = 4/3 of bf16
    attn_peak = peak16 * (4.0 / 3.0 if args.qk_e4m3 else 1.0)
    attn_name = "attention_split_kernel<e4m3 QK>" if args.qk_e4m3 else "attention_split_kernel"
    kernels = {"gemm_tc_kernel<e4m3>": {"ms_per_step": round(gemm_ms, 4), "tflops": round(gemm_tf, 1),
                                        "frac": round(gemm_tf / peak_f8, 4), "peak": round(peak_f8, 1),
                                        "launches_per_step": 4,
                                        "traffic_per_launch": TRAFFIC.get((w.name, "gemm_tc_kernel<e4m3>"))},
               attn_name: {"ms_per_step": round(per_call["h3_attention"], 4), "tflops": round(attn_tf, 1),
                           "frac": round(attn_tf / attn_peak, 4), "peak": round(attn_peak, 1),
                           "launches_per_step": 2, "traffic_per_launch": TRAFFIC.get((w.name, attn_name))}}
    dominant = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    return {
        "metric": ("packed tokens/s per Omni block (e4m3 GEMMs, e4m3 Q K^T, bf16 P V, 1×B200)" if args.qk_e4m3
                   else "packed tokens/s per Omni block (e4m3 GEMMs, bf16 attention, 1×B200)"),
        "value": round(L / (ms_step / 1e3), 1), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 GEMMs (fp32 accumulate), bf16 attention",
        "data": "synthetic (seeded N(0,1) latents/text, N(0,0.02) random-init weights quantised per output channel)",
        "config": {"workload": w.name, "packed_tokens": L, "L_pad": Lp, "hidden": w.D, "heads": w.H, "ffn": w.F,
                   "quantisation": "OFP8 e4m3, per-token activation and per-output-channel weight scales"},
        "roofline": {"bound": "tensor", "kernel": dominant, "achieved": kernels[dominant]["tflops"],
                     "peak": kernels[dominant]["peak"], "unit": "TFLOP/s", "frac": kernels[dominant]["frac"],
                     "peak_kind": ("e4m3 GEMM: 2 x the bf16 figure (sustained for a region >= 1 s, else burst) of measured, the nominal e4m3 / bf16 ratio"
                                   if dominant.startswith("gemm") else
                                   "attention: the bf16 figure (sustained for a region >= 1 s, else burst) of measured" + (
                                       ", x 4/3 for the e4m3 Q K^T half of its FLOPs" if args.qk_e4m3 else "")),
                     "traffic": kernels[dominant]["traffic_per_launch"]},
        "kernels": kernels,
        "block": {"ms": round(block_ms, 4),
                  "tflops": round(sum(fl.values()) / (block_ms / 1e3) / 1e12, 1)},
        "per_call_ms": {c: round(v, 4) for c, v in per_call.items()},
        "gpu_launches": st.launches_per_step(e4m3=True, qk_e4m3=args.qk_e4m3) * args.steps,
        "clocks": clocks,
    }


def run_sampler(args, w):
    """The layered flow sampler: args.layers blocks per denoise step, timed
    over args.steps denoise steps (after args.warmup untimed ones)."""
    import torch
    from omni_modal_diffusion_b200 import h3
    from omni_modal_diffusion_b200.pipeline import H3Sampler
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(99 + w.index)
    rnd = lambda *s, std=1.0, dt=torch.bfloat16: (torch.randn(*s, generator=g, device=dev) * std).to(dt)
    io = {"W_text": rnd(w.D, w.D_text, std=0.02), "W_vid": rnd(w.D, 4 * w.C_lat, std=0.02),
          "W_aud": rnd(w.D, w.C_audio, std=0.02), "W_vhead": rnd(4 * w.C_lat, w.D, std=0.02),
          "W_ahead": rnd(w.C_audio, w.D, std=0.02)}
    blocks = [{"Wqkv": rnd(3 * w.I, w.D, std=0.02), "qn_w": rnd(128, std=0.1) + 1, "kn_w": rnd(128, std=0.1) + 1,
               "Wo": rnd(w.D, w.I, std=0.02), "Wgu": rnd(2 * w.F, w.D, std=0.02), "Wd": rnd(w.D, w.F, std=0.02)}
              for _ in range(args.layers)]
    weights_gb = sum(t.numel() * 2 for b_ in blocks for t in b_.values()) / 1e9
    smp = H3Sampler(w, io, blocks, device=dev, e4m3=args.e4m3, qk_e4m3=args.qk_e4m3)
    if args.e4m3:
        del blocks  # the sampler keeps the e4m3 copies only
    L = smp.st.ranges.L
    n_total = args.warmup + args.steps
    text = rnd(w.n_text, w.D_text)
    lv = rnd(w.T_lat, w.H_lat, w.W_lat, w.C_lat, dt=torch.float32)
    la = rnd(w.audio_channels, w.n_audio, w.C_audio, dt=torch.float32)
    lv_bf, la_bf = lv.to(torch.bfloat16), la.to(torch.bfloat16)
    mod_all = rnd(n_total, args.layers, 3, 6, w.D, std=0.1, dt=torch.float32)
    sv = h3.h3_sigma_schedule(n_total, 12.0)
    sa = h3.h3_sigma_schedule(n_total, 3.0)
    stream = torch.cuda.current_stream(dev)
    for s in range(args.warmup):
        smp.step(s, text, lv, la, lv_bf, la_bf, mod_all, sv, sa)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for s in range(args.warmup, n_total):
        smp.step(s, text, lv, la, lv_bf, la_bf, mod_all, sv, sa)
    b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    assert h3.h3_device_status() == 0
    ms = a.elapsed_time(b) / args.steps
    fl = block_flops(w, L) * args.layers
    kind = ("e4m3 GEMMs, e4m3 Q K^T, bf16 P V" if args.qk_e4m3 else "e4m3 GEMMs, bf16 attention") if args.e4m3 \
        else "bf16"
    return {"metric": f"end-to-end denoise steps/s (layered flow sampler, {kind}, 1xB200)",
            "value": round(1e3 / ms, 4), "unit": "denoise steps/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": kind, "data": "synthetic (random-init bf16 weights, N(0,1) latents)",
            "config": {"workload": w.name, "packed_tokens": L, "layers": args.layers,
                       "weights_gb_bf16": round(weights_gb, 1)},
            "tokens_per_s_per_block": round(L * args.layers / (ms / 1e3), 1),
            "tflops": round(fl / (ms / 1e3) / 1e12, 1), "frac_of_bf16_sustained": round(
                fl / (ms / 1e3) / 1e12 / _peaks()["bf16_tflops_sustained"], 4),
            "gpu_launches": smp.launches_per_step() * args.steps, "clocks": clocks}


def run_sp(args, w):
    """Sequence parallelism (Ulysses, "MiniMax-H3 paper reading" §7.2): one
    packed sequence split over the N ranks of the job, one process per GPU,
    the exchange buffers opened through CUDA IPC and the two re-shardings
    fused into the QKV and attention epilogues (peer stores).  One timed unit
    is one block over the whole sequence (the ranks' shards together); the
    total work is fixed as N grows: strong scaling.  Embed, head and Euler are
    token-local and not part of this line."""
    import datetime
    import torch
    import torch.distributed as dist
    from omni_modal_diffusion_b200 import h3
    from omni_modal_diffusion_b200.pipeline import H3BlockStep
    from omni_modal_diffusion_b200.sp_runner import SPProcessRank

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if not (dist.is_available() and dist.is_initialized()):
        if "MASTER_ADDR" not in os.environ:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29533")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + w.index)            # the same weights and inputs on every rank

    def randn(*shape, std=1.0, dtype=torch.bfloat16):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(dtype)

    W = {"W_text": randn(w.D, w.D_text, std=0.02), "W_vid": randn(w.D, 4 * w.C_lat, std=0.02),
         "W_aud": randn(w.D, w.C_audio, std=0.02), "Wqkv": randn(3 * w.I, w.D, std=0.02),
         "qn_w": (1 + 0.1 * torch.randn(128, generator=g, device=dev)).to(torch.bfloat16),
         "kn_w": (1 + 0.1 * torch.randn(128, generator=g, device=dev)).to(torch.bfloat16),
         "Wo": randn(w.D, w.I, std=0.02), "Wgu": randn(2 * w.F, w.D, std=0.02), "Wd": randn(w.D, w.F, std=0.02),
         "W_vhead": randn(4 * w.C_lat, w.D, std=0.02), "W_ahead": randn(w.C_audio, w.D, std=0.02)}
    st = H3BlockStep(w, device=dev, weights=W)
    st.embed(randn(w.n_text, w.D_text), randn(w.T_lat, w.H_lat, w.W_lat, w.C_lat),
             randn(w.audio_channels, w.n_audio, w.C_audio))
    mod = randn(3, 6, w.D, std=0.1, dtype=torch.float32)
    L = st.ranges.L
    e4m3 = bool(getattr(args, "e4m3", False))
    qk8 = e4m3 and bool(getattr(args, "qk_e4m3", False))
    W8 = st.quantize_block_weights_e4m3() if e4m3 else None
    me = SPProcessRank(w, st.dims, st.ranges, dev, e4m3=e4m3, qk_e4m3=qk8)
    fwd = (lambda: me.block_forward_e4m3(mod, W8)) if e4m3 else (lambda: me.block_forward(mod, W))
    r = me.rank
    r.x.zero_()
    r.pos.zero_()
    lo, hi = r.rows.start, min(r.rows.stop, st.ranges.L_pad)
    x0 = torch.zeros_like(r.x)
    x0[: hi - lo].copy_(st.x[lo:hi])
    r.pos[: hi - lo].copy_(st.pos[lo:hi])
    del st                                    # only the shard stays resident
    stream = torch.cuda.current_stream(dev)
    me.barrier()
    for _ in range(args.warmup):
        r.x.copy_(x0)
        fwd()
    me.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        fwd()
    t1.record(stream)
    me.barrier()
    ms = t0.elapsed_time(t1) / args.steps
    status = h3.h3_device_status()
    (ms,) = max_over_ranks([ms], device=dev)
    me.close()
    dist.destroy_process_group()
    if status != 0:
        raise RuntimeError(f"device-side wait gave up (code {status})")
    if rank != 0:
        return None
    fl = block_flops(w, L)
    return {"metric": "packed tokens/s per Omni block, sequence-parallel (Ulysses) over the job's GPUs",
            "value": round(L / (ms / 1e3), 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None,
            "dtype": ("e4m3 GEMMs" + (", e4m3 Q K^T" if qk8 else "") + ", bf16 P V") if e4m3 else "bf16",
            "data": "synthetic (seeded N(0,1) latents/text, N(0,0.02) weights)",
            "config": {"workload": w.name, "packed_tokens": L, "parallelism": f"ulysses sp{world}",
                       "L_shard": me.layout.L_shard, "heads_per_rank": me.layout.heads,
                       "q_k_exchange": "e4m3 codes" if qk8 else "bf16"},
            "tflops": round(fl / (ms / 1e3) / 1e12, 1),
            # LN, QKV, attention (split + fixup), out-projection, LN, FFN x2 (e4m3: + 2 row quantisers)
            "gpu_launches": (10 if e4m3 else 8) * args.steps,
            "barriers_per_block": 2}


def run_only(args, w):
    """One C-ABI call on the workload's shapes, nothing else resident but its
    operands (for ncu captures of a single kernel)."""
    import dataclasses
    import torch
    from omni_modal_diffusion_b200 import h3
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(4321)
    rnd = lambda *s, std=1.0, dt=torch.bfloat16: (torch.randn(*s, generator=g, device=dev) * std).to(dt)
    if args.heads:
        w = dataclasses.replace(w, H=args.heads)
    d = h3.make_dims(w.D, w.H, w.F, rope=w.rope_split)
    r = h3.h3_make_ranges(w.n_text, w.audio_channels * w.n_audio, w.T_lat * (w.H_lat // 2) * (w.W_lat // 2))
    Lp = r.L_pad
    mod = rnd(3, 6, w.D, std=0.1, dt=torch.float32)
    if args.only == "attention_prologue":
        # raw N(0, 1) q, k (as the QKV call writes them without its norm and
        # RoPE) with norm weights and seeded positions: the prologue kernel
        q, k, v = (rnd(w.H, Lp, 128) for _ in range(3))
        qn, kn = rnd(128, std=0.1) + 1, rnd(128, std=0.1) + 1
        pos = torch.randint(0, 64, (Lp, 3), generator=g, device=dev).float()
        o = torch.empty(Lp, w.I, dtype=torch.bfloat16, device=dev)
        fn = lambda: h3.h3_attention(d, r, q, k, v, o, qn_w=qn, kn_w=kn, pos=pos, flags=0)
    elif args.only == "attention_qk8":
        # q, k as the e4m3 QKV epilogue leaves them: codes of the normalised
        # rows times 448 / (sqrt(128) max|w|) (input generation: torch's
        # float8 conversion), v bf16
        qn, kn = rnd(128, std=0.1) + 1, rnd(128, std=0.1) + 1
        def codes(wt):
            xf = rnd(w.H, Lp, 128).float()
            xf = xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + 1e-6) * wt.float()
            inv = 448.0 / (128 ** 0.5 * float(wt.float().abs().max()))
            return (xf * inv).to(torch.float8_e4m3fn).view(torch.uint8)
        q8, k8 = codes(qn), codes(kn)
        v = rnd(w.H, Lp, 128)
        o = torch.empty(Lp, w.I, dtype=torch.bfloat16, device=dev)
        fl = h3.H3_QK_NORM_ROPE_IN_QKV | h3.H3_QK_E4M3
        fn = lambda: h3.h3_attention(d, r, q8, k8, v, o, qn_w=qn, kn_w=kn, flags=fl)
    elif args.only in ("attention", "attention_raw"):
        # q, k rows as the QKV call leaves them: RMS-normalised and scaled by
        # the norm weights (attention then runs its split-softmax kernel);
        # attention_raw: unnormalised N(0, 1) rows, no norm weights (the
        # general kernel alone)
        q, k, v = (rnd(w.H, Lp, 128) for _ in range(3))
        qn, kn = rnd(128, std=0.1) + 1, rnd(128, std=0.1) + 1
        if args.only == "attention":
            def rms(x, wt):
                xf = x.float()
                return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + 1e-6) * wt.float()).to(torch.bfloat16)
            q, k = rms(q, qn), rms(k, kn)
        o = torch.empty(Lp, w.I, dtype=torch.bfloat16, device=dev)
        if args.only == "attention":
            fn = lambda: h3.h3_attention(d, r, q, k, v, o, qn_w=qn, kn_w=kn)
        else:
            fn = lambda: h3.h3_attention(d, r, q, k, v, o)
    elif args.only == "qkv":
        xm = rnd(Lp, w.D)
        Wqkv = rnd(3 * w.I, w.D, std=0.02)
        qn, kn = rnd(128, std=0.1) + 1, rnd(128, std=0.1) + 1
        pos = torch.zeros(Lp, 3, device=dev)
        q, k, v = (torch.empty(w.H, Lp, 128, dtype=torch.bfloat16, device=dev) for _ in range(3))
        fn = lambda: h3.h3_qkv_qknorm_mrope(d, r, xm, Wqkv, qn, kn, pos, q, k, v)
    elif args.only == "out":
        x = rnd(Lp, w.D, dt=torch.float32)
        o = rnd(Lp, w.I)
        Wo = rnd(w.D, w.I, std=0.02)
        fn = lambda: h3.h3_gated_residual(d, r, x, o, Wo, mod, h3.H3_MSA)
    elif args.only == "ffn":
        x = rnd(Lp, w.D, dt=torch.float32)
        xm = rnd(Lp, w.D)
        Wgu, Wd = rnd(2 * w.F, w.D, std=0.02), rnd(w.D, w.F, std=0.02)
        ws = torch.empty(Lp, w.F, dtype=torch.bfloat16, device=dev)
        fn = lambda: h3.h3_ffn_swiglu(d, r, x, xm, Wgu, Wd, mod, ws)
    elif args.only == "euler":
        # the video and audio latents of the workload, updated in place
        n_lat = w.T_lat * w.H_lat * w.W_lat * w.C_lat + w.audio_channels * w.n_audio * w.C_audio
        lat, vel = rnd(n_lat, dt=torch.float32), rnd(n_lat, dt=torch.float32)
        fn = lambda: h3.h3_euler_step(lat, vel, 0.5, 0.4)
    else:
        x = rnd(Lp, w.D, dt=torch.float32)
        xm = torch.empty(Lp, w.D, dtype=torch.bfloat16, device=dev)
        fn = lambda: h3.h3_adaln_norm_modulate(d, r, x, mod, h3.H3_MSA, xm)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    ms = a.elapsed_time(b) / args.steps
    extra = ""
    if args.only.startswith("attention"):
        L = r.L
        extra = f", {4.0 * L * L * w.I / (ms / 1e3) / 1e12:.1f} TFLOP/s"
    print(f"{args.only} on {w.name} (H={w.H}): {ms:.4f} ms per call{extra}", flush=True)


def block_flops(w, L):
    """Algorithmic FLOPs of one block over L valid tokens."""
    return 2.0 * L * (w.D * 3 * w.I + w.I * w.D + 2 * w.D * w.F + w.F * w.D) + 4.0 * L * L * w.I


_SAMPLE_CACHE = {}


def _oracle_sample_inputs(w, frames):
    """Seeded inputs of the cut workload and its packing, drawn once per
    process (drawing the full-width weights takes longer than the sample)."""
    key = (w.name, frames)
    if key not in _SAMPLE_CACHE:
        import dataclasses
        from oracle import h3_oracle as O
        from omni_modal_diffusion_b200 import synthetic as S
        ws = dataclasses.replace(w, T_lat=min(frames, w.T_lat))
        inp = S.make_inputs(ws)
        t_g, i_g, j_g = O.token_grid(ws.T_lat, ws.H_lat, ws.W_lat)
        r = O.pack_ranges(ws.n_text, ws.audio_channels * ws.n_audio, t_g * i_g * j_g)
        pos = O.positions(r, t_g, i_g, j_g, ws.audio_channels, ws.n_audio)
        _SAMPLE_CACHE[key] = (ws, inp, r, pos)
    return _SAMPLE_CACHE[key]


def cpu_baseline(w, frames=None):
    """The float64 oracle on the host cores, on a bounded sample of the same
    workload: the whole block (packing, projections, LN+modulate, QKV,
    RMSNorm, RoPE, attention, gated out-projection, SwiGLU FFN) on the same
    text and audio with the video cut to `frames` latent frames (2, or 1 for
    the 15 s workload, whose 1,200 audio and 1,344 video tokens per frame
    already make a ~6 s sample), timed in full, then scaled to the workload's
    length by the block's algorithmic FLOPs (the oracle is matmul-bound)."""
    if frames is None:
        frames = 1 if w.T_lat > 60 else 2
    from oracle import h3_oracle as O
    try:
        import threadpoolctl
        threads = max(info.get("num_threads", 0) for info in threadpoolctl.threadpool_info()) or os.cpu_count()
    except Exception:  # pragma: no cover
        threads = os.cpu_count()
    ws, inp, r, pos = _oracle_sample_inputs(w, frames)
    t0 = time.perf_counter()
    x = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    O.block_forward(x, inp["mod"], r, pos, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"], inp["Wgu"],
                    inp["Wd"], ws.H)
    t_s = time.perf_counter() - t0
    Ls = r["L"]
    L = w.n_text + w.audio_channels * w.n_audio + w.T_lat * (w.H_lat // 2) * (w.W_lat // 2)
    t_full = t_s * block_flops(w, L) / block_flops(w, Ls)
    return {"value": round(L / t_full, 2), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"float64 oracle block on {w.name} cut to {ws.T_lat} latent frames ({Ls} packed tokens, "
                      f"{t_s:.1f} s measured), scaled to {L} tokens by algorithmic FLOPs "
                      f"({block_flops(w, L) / block_flops(w, Ls):.2f}x)",
            "seconds_per_block_extrapolated": round(t_full, 2), "sample_seconds": round(t_s, 3)}


def run_reference(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    vals, secs = [], []
    base = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(w)   # times the oracle block alone (inputs drawn once, untimed)
        if i >= args.warmup:
            vals.append(cb["value"])
            secs.append(cb["sample_seconds"])
            base = cb
    value = statistics.mean(vals)
    return {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(secs), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": {"workload": w.name},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"]},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 100; sampler: 8)")
    ap.add_argument("--warmup", type=int, default=None, help="untimed steps (default 10; sampler: 3)")
    ap.add_argument("--sampler", action="store_true",
                    help="time the layered flow sampler (denoise steps/s) instead of the single-block step")
    ap.add_argument("--layers", type=int, default=50)
    ap.add_argument("--sp", action="store_true",
                    help="sequence parallelism: one sequence split over the job's ranks (a separate line)")
    ap.add_argument("--qk-prologue", action="store_true",
                    help="the per-head Q/K RMSNorm + RoPE in attention's prologue (raw q, k from the QKV call) "
                         "instead of the QKV epilogue")
    ap.add_argument("--e4m3", action="store_true",
                    help="the block step with its four GEMMs in e4m3 (a separate line; one GPU)")
    ap.add_argument("--qk-e4m3", action="store_true",
                    help="with --e4m3: q and k cross to attention as e4m3 codes (Q K^T on e4m3 MMAs)")
    ap.add_argument("--only", default=None, choices=["attention", "attention_raw", "attention_prologue",
                                                     "attention_qk8", "qkv", "out", "ffn", "ln", "euler"],
                    help="launch only this call (small ncu captures); prints timing, no JSON contract line")
    ap.add_argument("--heads", type=int, default=None, help="with --only: this many heads instead of the workload's")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None, help=f"default {DEFAULT_WORKLOAD}; sampler: 768x1344_5s")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    from omni_modal_diffusion_b200 import synthetic as S
    w = S.WORKLOADS[args.workload or ("768x1344_5s" if args.sampler else DEFAULT_WORKLOAD)]
    long_seq = w.T_lat * (w.H_lat // 2) * (w.W_lat // 2) > 60000  # ~0.5 s per block step
    if args.steps is None:
        args.steps = 8 if args.sampler else (20 if long_seq else 100)
    if args.warmup is None:
        args.warmup = 3 if args.sampler else (5 if long_seq else 10)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference" and args.warmup > 1:
        args.warmup = 1            # each oracle step is a ~10-30 s CPU sample
    if args.only:
        run_only(args, w)
        return
    if args.sampler:
        print(json.dumps(run_sampler(args, w)), flush=True)
        return
    if args.sp:
        out = run_sp(args, w)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if args.e4m3:
        print(json.dumps(run_e4m3(args, w)), flush=True)
        return
    out = run_reference(args, w) if args.impl == "reference" else run_ours(args, w)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()

// C ABI of the H3-Omni block step (declarations and contracts: include/h3.h).
// Argument validation happens here, before any launch; the kernels live in
// the files included below (one translation unit, so the device error word
// and wait limit are shared by every kernel without relocatable device code).
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/h3.h"
#include "elementwise.cu"
#include "gemm_tc.cu"
#include "attention_tc.cu"
#include "attention_split.cu"

using namespace h3;

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = 0;
  return H3_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(H3_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// NVTX range over one C-ABI call, named after it, for a profiler that
// attaches (NVTX3 is header-only: with no tool attached push and pop return
// at once).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
#define H3_TRACE() NvtxRange h3_trace_range_(__func__)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define H3_REQUIRE_PTR(p)                                                   \
  do {                                                                      \
    if (!(p)) return fail(H3_ERR_NULL, "%s: argument '%s' is NULL", __func__, #p); \
    if (!aligned16(p)) return fail(H3_ERR_ALIGN, "%s: argument '%s' is not 16-byte aligned", __func__, #p); \
  } while (0)

int check_dims(const h3_dims* d, const char* fn) {
  if (!d) return fail(H3_ERR_NULL, "%s: dims is NULL", fn);
  if (d->head_dim != 128) return fail(H3_ERR_UNSUPPORTED, "%s: head_dim must be 128 (got %d)", fn, d->head_dim);
  if (d->H <= 0 || d->I != d->H * d->head_dim)
    return fail(H3_ERR_SHAPE, "%s: I (%d) must equal H (%d) * head_dim", fn, d->I, d->H);
  if (d->D <= 0 || d->D % 64 != 0 || d->D > 8192)
    return fail(H3_ERR_UNSUPPORTED, "%s: D must be a positive multiple of 64, at most 8192 (got %d)", fn, d->D);
  if (d->F <= 0 || d->F % 128 != 0)
    return fail(H3_ERR_UNSUPPORTED, "%s: F must be a positive multiple of 128 (got %d)", fn, d->F);
  if (d->rope_t < 0 || d->rope_h < 0 || d->rope_w < 0 || (d->rope_t | d->rope_h | d->rope_w) & 1 ||
      d->rope_t + d->rope_h + d->rope_w != d->head_dim)
    return fail(H3_ERR_SHAPE, "%s: rope_t + rope_h + rope_w must equal head_dim, each even", fn);
  if (!(d->theta > 0.f) || !(d->eps_ln > 0.f) || !(d->eps_qk > 0.f))
    return fail(H3_ERR_SHAPE, "%s: theta, eps_ln, eps_qk must be positive", fn);
  return H3_OK;
}

int check_ranges(const h3_ranges* r, const char* fn) {
  if (!r) return fail(H3_ERR_NULL, "%s: ranges is NULL", fn);
  if (r->L <= 0) return fail(H3_ERR_SHAPE, "%s: L must be positive (got %d)", fn, r->L);
  if (r->L_pad % 128 != 0 || r->L_pad < r->L)
    return fail(H3_ERR_SHAPE, "%s: L_pad (%d) must be a multiple of 128 and at least L (%d)", fn, r->L_pad, r->L);
  long total = 0;
  for (int m = 0; m < 3; ++m) {
    if (r->start[m] < 0 || r->count[m] < 0 || (long)r->start[m] + r->count[m] > r->L)
      return fail(H3_ERR_SHAPE, "%s: range %d [%d, +%d) outside [0, L)", fn, m, r->start[m], r->count[m]);
    total += r->count[m];
    for (int n = 0; n < m; ++n) {
      const long a0 = r->start[m], a1 = a0 + r->count[m], b0 = r->start[n], b1 = b0 + r->count[n];
      if (r->count[m] > 0 && r->count[n] > 0 && a0 < b1 && b0 < a1)
        return fail(H3_ERR_SHAPE, "%s: ranges %d and %d overlap", fn, n, m);
    }
  }
  if (total != r->L) return fail(H3_ERR_SHAPE, "%s: ranges cover %ld rows, L is %d", fn, total, r->L);
  return H3_OK;
}

#define H3_CHECK(expr)          \
  do {                          \
    int _rc = (expr);           \
    if (_rc != H3_OK) return _rc; \
  } while (0)

GemmProblem gemm_base(const void* A, long lda, int M, int K, const void* B, long ldb, int N_b_rows, int n_tiles) {
  GemmProblem p;
  memset(&p, 0, sizeof(p));
  p.A = A;
  p.lda = lda;
  p.B = B;
  p.ldb = ldb;
  p.N_b_rows = N_b_rows;
  p.M = M;
  p.K = K;
  p.n_tiles = n_tiles;
  p.b_second_half_off = 128;
  return p;
}

void set_ranges(GemmEpilogue& e, const h3_ranges* r) {
  for (int m = 0; m < 3; ++m) {
    e.rstart[m] = r->start[m];
    e.rcount[m] = r->count[m];
  }
}

// The block's GEMM problems, shared by the bf16 and e4m3 entry points (the
// e4m3 ones then set f8 and the scales).
GemmProblem qkv_problem(const h3_dims* dims, const h3_ranges* ranges, const void* xm, const void* Wqkv,
                        const h3_bf16* qn_w, const h3_bf16* kn_w, const float* pos, h3_bf16* q, h3_bf16* k,
                        h3_bf16* v) {
  const int D = dims->D, I = dims->I, Lp = ranges->L_pad;
  GemmProblem p = gemm_base(xm, D, Lp, D, Wqkv, D, 3 * I, (3 * I + 255) / 256);
  p.pair = 1;
  GemmEpilogue& ep = p.epi;
  ep.mode = EPI_QKV;
  ep.M = Lp;
  ep.N = 3 * I;
  set_ranges(ep, ranges);
  ep.q = reinterpret_cast<bf16*>(q);
  ep.k = reinterpret_cast<bf16*>(k);
  ep.v = reinterpret_cast<bf16*>(v);
  ep.qn_w = reinterpret_cast<const bf16*>(qn_w);
  ep.kn_w = reinterpret_cast<const bf16*>(kn_w);
  ep.pos = pos;
  ep.L_pad = Lp;
  ep.I = I;
  ep.rope_t = dims->rope_t;
  ep.rope_h = dims->rope_h;
  ep.rope_w = dims->rope_w;
  ep.theta = dims->theta;
  ep.eps_qk = dims->eps_qk;
  return p;
}

// x += gate[slot] * (A W^T), A [L_pad][K], W [D][K]
GemmProblem gated_problem(const h3_dims* dims, const h3_ranges* ranges, float* x, const void* A, int K,
                          const void* W, const float* mod, int gate_slot) {
  const int D = dims->D, Lp = ranges->L_pad;
  GemmProblem p = gemm_base(A, K, Lp, K, W, K, D, (D + 255) / 256);
  p.pair = 1;
  p.epi.mode = EPI_GATED_RESID;
  p.epi.M = Lp;
  p.epi.N = D;
  p.epi.ldo = D;
  p.epi.out = x;
  set_ranges(p.epi, ranges);
  p.epi.mod = mod;
  p.epi.gate_slot = gate_slot;
  p.epi.D = D;
  return p;
}

// ws = bf16(SiLU(xm Wg^T) * (xm Wu^T)), Wgu = [gate rows; up rows]
GemmProblem swiglu_problem(const h3_dims* dims, int Lp, const void* xm, const void* Wgu, void* ws) {
  const int D = dims->D, F = dims->F;
  GemmProblem p = gemm_base(xm, D, Lp, D, Wgu, D, 2 * F, F / 128);
  p.pair = 1;
  p.b_second_half_off = F;
  p.epi.mode = EPI_SWIGLU;
  p.epi.M = Lp;
  p.epi.N = F;
  p.epi.ldo = F;
  p.epi.out = ws;
  return p;
}

}  // namespace

extern "C" {

const char* h3_last_error(void) { return g_err; }

int h3_version(void) { return 100; }

int h3_make_ranges(int n_text, int n_audio_tokens, int n_video_tokens, h3_ranges* out) {
  if (!out) return fail(H3_ERR_NULL, "h3_make_ranges: out is NULL");
  if (n_text < 0 || n_audio_tokens < 0 || n_video_tokens < 0)
    return fail(H3_ERR_SHAPE, "h3_make_ranges: negative token count");
  const long L = (long)n_text + n_audio_tokens + n_video_tokens;
  if (L <= 0 || L > (1L << 30)) return fail(H3_ERR_SHAPE, "h3_make_ranges: L = %ld out of range", L);
  out->start[H3_TEXT] = 0;
  out->count[H3_TEXT] = n_text;
  out->start[H3_AUDIO] = n_text;
  out->count[H3_AUDIO] = n_audio_tokens;
  out->start[H3_VIDEO] = n_text + n_audio_tokens;
  out->count[H3_VIDEO] = n_video_tokens;
  out->L = (int)L;
  out->L_pad = (int)((L + 127) / 128 * 128);
  return ok();
}

int h3_sigma_schedule(int n_steps, float shift, float* out) {
  if (!out) return fail(H3_ERR_NULL, "h3_sigma_schedule: out is NULL");
  if (n_steps <= 0 || !(shift > 0.f)) return fail(H3_ERR_SHAPE, "h3_sigma_schedule: n_steps > 0 and shift > 0 required");
  for (int i = 0; i <= n_steps; ++i) {
    const double s = 1.0 - (double)i / n_steps;
    out[i] = (float)(shift * s / (1.0 + (shift - 1.0) * s));
  }
  return ok();
}

int h3_embed_pack(const h3_dims* dims, const h3_ranges* ranges, const h3_bf16* text, int D_text,
                  const h3_bf16* video, int T, int Hl, int Wl, int C_lat, const h3_bf16* audio,
                  int audio_channels, int n_audio, int C_audio, const h3_bf16* W_text, const h3_bf16* W_vid,
                  const h3_bf16* W_aud, h3_bf16* patches, float* x_out, float* pos_out, uint8_t* mod_out,
                  void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  const int nt = ranges->count[H3_TEXT], na = ranges->count[H3_AUDIO], nv = ranges->count[H3_VIDEO];
  if (T < 0 || Hl < 0 || Wl < 0 || (Hl & 1) || (Wl & 1))
    return fail(H3_ERR_SHAPE, "%s: video latent T, Hl, Wl must be >= 0 with Hl, Wl even", __func__);
  if ((long)T * (Hl / 2) * (Wl / 2) != nv)
    return fail(H3_ERR_SHAPE, "%s: count[VIDEO] (%d) != T*(Hl/2)*(Wl/2) (%ld)", __func__, nv, (long)T * (Hl / 2) * (Wl / 2));
  if (audio_channels < 0 || n_audio < 0 || (long)audio_channels * n_audio != na)
    return fail(H3_ERR_SHAPE, "%s: count[AUDIO] (%d) != audio_channels*n_audio", __func__, na);
  if (nt > 0 && (D_text <= 0 || D_text % 8))
    return fail(H3_ERR_UNSUPPORTED, "%s: D_text must be a positive multiple of 8", __func__);
  if (nv > 0 && (C_lat <= 0 || C_lat % 4))
    return fail(H3_ERR_UNSUPPORTED, "%s: C_lat must be a positive multiple of 4", __func__);
  if (na > 0 && (C_audio <= 0 || C_audio % 8))
    return fail(H3_ERR_UNSUPPORTED, "%s: C_audio must be a positive multiple of 8", __func__);
  H3_REQUIRE_PTR(x_out);
  H3_REQUIRE_PTR(pos_out);
  H3_REQUIRE_PTR(mod_out);
  if (nt > 0) { H3_REQUIRE_PTR(text); H3_REQUIRE_PTR(W_text); }
  if (na > 0) { H3_REQUIRE_PTR(audio); H3_REQUIRE_PTR(W_aud); }
  if (nv > 0) { H3_REQUIRE_PTR(video); H3_REQUIRE_PTR(W_vid); H3_REQUIRE_PTR(patches); }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = dims->D;
  cudaError_t e = launch_pack(reinterpret_cast<const bf16*>(video), T, Hl, Wl, C_lat, n_audio, audio_channels,
                              ranges->start, ranges->count, ranges->L, ranges->L_pad, reinterpret_cast<bf16*>(patches),
                              pos_out, mod_out, x_out, D, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_embed_pack: pack");
  struct Src { const void* A; int K; const void* W; int mod; } srcs[3] = {
      {text, D_text, W_text, H3_TEXT}, {audio, C_audio, W_aud, H3_AUDIO}, {patches, 4 * C_lat, W_vid, H3_VIDEO}};
  for (const Src& s : srcs) {
    const int M = ranges->count[s.mod];
    if (M == 0) continue;
    GemmProblem p = gemm_base(s.A, s.K, M, s.K, s.W, s.K, D, (D + 255) / 256);
    p.epi.mode = EPI_STORE_F32;
    p.epi.M = M;
    p.epi.N = D;
    p.epi.row_off = ranges->start[s.mod];
    p.epi.ldo = D;
    p.epi.out = x_out;
    e = launch_gemm(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "h3_embed_pack: input projection");
  }
  return ok();
}

int h3_adaln_norm_modulate(const h3_dims* dims, const h3_ranges* ranges, const float* x, const float* mod,
                           int branch, h3_bf16* xm, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (branch != H3_MSA && branch != H3_MLP) return fail(H3_ERR_SHAPE, "%s: branch must be H3_MSA or H3_MLP", __func__);
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(mod);
  H3_REQUIRE_PTR(xm);
  cudaError_t e = launch_ln_modulate(x, mod, branch, ranges->start, ranges->count, ranges->L, ranges->L_pad, dims->D,
                                     dims->eps_ln, reinterpret_cast<bf16*>(xm), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_adaln_norm_modulate");
  return ok();
}

int h3_qkv_qknorm_mrope(const h3_dims* dims, const h3_ranges* ranges, const h3_bf16* xm, const h3_bf16* Wqkv,
                        const h3_bf16* qn_w, const h3_bf16* kn_w, const float* pos, int flags, h3_bf16* q,
                        h3_bf16* k, h3_bf16* v, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (flags & ~H3_QK_NORM_ROPE_IN_QKV)
    return fail(H3_ERR_UNSUPPORTED, "%s: e4m3 q/k output needs h3_qkv_qknorm_mrope_e4m3", __func__);
  const bool in_qkv = (flags & H3_QK_NORM_ROPE_IN_QKV) != 0;
  H3_REQUIRE_PTR(xm);
  H3_REQUIRE_PTR(Wqkv);
  if (in_qkv) {  // without the flag q, k leave raw and qn_w, kn_w, pos go to h3_attention instead
    H3_REQUIRE_PTR(qn_w);
    H3_REQUIRE_PTR(kn_w);
    H3_REQUIRE_PTR(pos);
  }
  H3_REQUIRE_PTR(q);
  H3_REQUIRE_PTR(k);
  H3_REQUIRE_PTR(v);
  GemmProblem p = qkv_problem(dims, ranges, xm, Wqkv, qn_w, kn_w, pos, q, k, v);
  p.epi.qk_raw = in_qkv ? 0 : 1;
  cudaError_t e = launch_gemm(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_qkv_qknorm_mrope");
  return ok();
}

int h3_attention(const h3_dims* dims, const h3_ranges* ranges, const h3_bf16* q, const h3_bf16* k,
                 const h3_bf16* v, const h3_bf16* qn_w, const h3_bf16* kn_w, const float* pos, int flags,
                 h3_bf16* o, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (flags & ~(H3_QK_NORM_ROPE_IN_QKV | H3_QK_E4M3)) return fail(H3_ERR_UNSUPPORTED, "%s: unknown flags", __func__);
  if ((flags & H3_QK_E4M3) && !(flags & H3_QK_NORM_ROPE_IN_QKV))
    return fail(H3_ERR_UNSUPPORTED, "%s: e4m3 q, k are written by the QKV epilogue after its norm and RoPE", __func__);
  H3_REQUIRE_PTR(q);
  H3_REQUIRE_PTR(k);
  H3_REQUIRE_PTR(v);
  H3_REQUIRE_PTR(o);
  AttnProblem p;
  memset(&p, 0, sizeof(p));
  if (!(flags & H3_QK_NORM_ROPE_IN_QKV)) {  // raw q, k: RMSNorm and RoPE in attention's prologue
    H3_REQUIRE_PTR(qn_w);
    H3_REQUIRE_PTR(kn_w);
    H3_REQUIRE_PTR(pos);
    p.prologue = 1;
    p.pos = pos;
    p.rope_t = dims->rope_t;
    p.rope_h = dims->rope_h;
    p.rope_w = dims->rope_w;
    p.theta = dims->theta;
    p.eps_qk = dims->eps_qk;
  } else if (flags & H3_QK_E4M3) {  // q, k: e4m3 codes whose scales follow from qn_w, kn_w
    H3_REQUIRE_PTR(qn_w);
    H3_REQUIRE_PTR(kn_w);
    p.qk8 = 1;
  } else if (qn_w || kn_w) {  // bf16 q, k normalised with these weights: the split-softmax kernel
    H3_REQUIRE_PTR(qn_w);
    H3_REQUIRE_PTR(kn_w);
  }
  p.qn_w = reinterpret_cast<const bf16*>(qn_w);
  p.kn_w = reinterpret_cast<const bf16*>(kn_w);
  p.q = reinterpret_cast<const bf16*>(q);
  p.k = reinterpret_cast<const bf16*>(k);
  p.v = reinterpret_cast<const bf16*>(v);
  p.o = reinterpret_cast<bf16*>(o);
  p.H = dims->H;
  p.L = ranges->L;
  p.L_pad = ranges->L_pad;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->head_dim));
  cudaError_t e = launch_attention(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_attention");
  return ok();
}

int h3_gated_residual(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_bf16* o,
                      const h3_bf16* Wo, const float* mod, int branch, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (branch != H3_MSA && branch != H3_MLP) return fail(H3_ERR_SHAPE, "%s: branch must be H3_MSA or H3_MLP", __func__);
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(o);
  H3_REQUIRE_PTR(Wo);
  H3_REQUIRE_PTR(mod);
  GemmProblem p = gated_problem(dims, ranges, x, o, dims->I, Wo, mod, 3 * branch + 2);
  cudaError_t e = launch_gemm(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_gated_residual");
  return ok();
}

size_t h3_ffn_workspace_bytes(const h3_dims* dims, int L_pad) {
  if (!dims || L_pad <= 0 || dims->F <= 0) return 0;
  return (size_t)L_pad * (size_t)dims->F * 2;
}

int h3_ffn_swiglu(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_bf16* xm,
                  const h3_bf16* Wgu, const h3_bf16* Wd, const float* mod, h3_bf16* ws, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(xm);
  H3_REQUIRE_PTR(Wgu);
  H3_REQUIRE_PTR(Wd);
  H3_REQUIRE_PTR(mod);
  H3_REQUIRE_PTR(ws);
  const int Lp = ranges->L_pad;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GemmProblem p1 = swiglu_problem(dims, Lp, xm, Wgu, ws);
  cudaError_t e = launch_gemm(p1, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu: gate/up");
  GemmProblem p2 = gated_problem(dims, ranges, x, ws, dims->F, Wd, mod, 5);
  e = launch_gemm(p2, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu: down");
  return ok();
}

namespace {
// The head (A10) and, with euler set, the Euler step (A11) in the head
// GEMMs' epilogues.  Without euler: out_v / out_a receive the velocities.
// With euler: out_v / out_a hold the latents, updated in place by
// (sigma_next - sigma) * velocity, and out_v16 / out_a16 (nullable) receive
// their bf16 copies.
int head_impl(const char* fn, const h3_dims* dims, const h3_ranges* ranges, const float* x, const h3_bf16* W_vhead,
              const h3_bf16* W_ahead, int T, int Hl, int Wl, int C_lat, int audio_channels, int n_audio, int C_audio,
              h3_bf16* hn, float* out_v, float* out_a, bool euler, float ds_v, float ds_a, h3_bf16* out_v16,
              h3_bf16* out_a16, void* stream) {
  H3_CHECK(check_dims(dims, fn));
  H3_CHECK(check_ranges(ranges, fn));
  const int na = ranges->count[H3_AUDIO], nv = ranges->count[H3_VIDEO];
  if (T < 0 || (Hl & 1) || (Wl & 1) || (long)T * (Hl / 2) * (Wl / 2) != nv)
    return fail(H3_ERR_SHAPE, "%s: count[VIDEO] != T*(Hl/2)*(Wl/2)", fn);
  if ((long)audio_channels * n_audio != na) return fail(H3_ERR_SHAPE, "%s: count[AUDIO] != channels*n_audio", fn);
  if (nv > 0 && (C_lat <= 0 || C_lat % 4)) return fail(H3_ERR_UNSUPPORTED, "%s: C_lat must be a multiple of 4", fn);
  if (na > 0 && (C_audio <= 0 || C_audio % 4)) return fail(H3_ERR_UNSUPPORTED, "%s: C_audio must be a multiple of 4", fn);
  if (!x) return fail(H3_ERR_NULL, "%s: argument 'x' is NULL", fn);
  if (!aligned16(x)) return fail(H3_ERR_ALIGN, "%s: argument 'x' is not 16-byte aligned", fn);
  if (!hn) return fail(H3_ERR_NULL, "%s: argument 'hn' is NULL", fn);
  if (!aligned16(hn)) return fail(H3_ERR_ALIGN, "%s: argument 'hn' is not 16-byte aligned", fn);
  const char* vname = euler ? "lat_video" : "v_video";
  const char* aname = euler ? "lat_audio" : "v_audio";
  if (nv > 0) {
    if (!W_vhead || !out_v) return fail(H3_ERR_NULL, "%s: W_vhead or %s is NULL", fn, vname);
    if (!aligned16(W_vhead) || !aligned16(out_v)) return fail(H3_ERR_ALIGN, "%s: W_vhead or %s not 16-byte aligned", fn, vname);
    if (out_v16 && !aligned16(out_v16)) return fail(H3_ERR_ALIGN, "%s: lat_video_bf16 not 16-byte aligned", fn);
  }
  if (na > 0) {
    if (!W_ahead || !out_a) return fail(H3_ERR_NULL, "%s: W_ahead or %s is NULL", fn, aname);
    if (!aligned16(W_ahead) || !aligned16(out_a)) return fail(H3_ERR_ALIGN, "%s: W_ahead or %s not 16-byte aligned", fn, aname);
    if (out_a16 && !aligned16(out_a16)) return fail(H3_ERR_ALIGN, "%s: lat_audio_bf16 not 16-byte aligned", fn);
  }
  const int D = dims->D;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_ln_modulate(x, nullptr, 0, ranges->start, ranges->count, ranges->L, ranges->L_pad, D,
                                     dims->eps_ln, reinterpret_cast<bf16*>(hn), st);
  if (e != cudaSuccess) return cuda_fail(e, "head: norm");
  if (nv > 0) {
    const h3_bf16* A = hn + (size_t)ranges->start[H3_VIDEO] * D;
    GemmProblem p = gemm_base(A, D, nv, D, W_vhead, D, 4 * C_lat, (4 * C_lat + 255) / 256);
    p.epi.mode = EPI_UNPATCH;
    p.epi.M = nv;
    p.epi.N = 4 * C_lat;
    p.epi.out = out_v;
    p.epi.Ht = Hl / 2;
    p.epi.Wt = Wl / 2;
    p.epi.C_lat = C_lat;
    p.epi.euler = euler ? 1 : 0;
    p.epi.dsigma = ds_v;
    p.epi.out_bf16 = reinterpret_cast<bf16*>(out_v16);
    e = launch_gemm(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "head: video");
  }
  if (na > 0) {
    const h3_bf16* A = hn + (size_t)ranges->start[H3_AUDIO] * D;
    GemmProblem p = gemm_base(A, D, na, D, W_ahead, D, C_audio, (C_audio + 255) / 256);
    p.epi.mode = EPI_STORE_F32;
    p.epi.M = na;
    p.epi.N = C_audio;
    p.epi.ldo = C_audio;
    p.epi.out = out_a;
    p.epi.euler = euler ? 1 : 0;
    p.epi.dsigma = ds_a;
    p.epi.out_bf16 = reinterpret_cast<bf16*>(out_a16);
    e = launch_gemm(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "head: audio");
  }
  return ok();
}
}  // namespace

int h3_head_unpack(const h3_dims* dims, const h3_ranges* ranges, const float* x, const h3_bf16* W_vhead,
                   const h3_bf16* W_ahead, int T, int Hl, int Wl, int C_lat, int audio_channels, int n_audio,
                   int C_audio, h3_bf16* hn, float* v_video, float* v_audio, void* stream) {
  H3_TRACE();
  return head_impl(__func__, dims, ranges, x, W_vhead, W_ahead, T, Hl, Wl, C_lat, audio_channels, n_audio, C_audio,
                   hn, v_video, v_audio, false, 0.f, 0.f, nullptr, nullptr, stream);
}

int h3_head_euler(const h3_dims* dims, const h3_ranges* ranges, const float* x, const h3_bf16* W_vhead,
                  const h3_bf16* W_ahead, int T, int Hl, int Wl, int C_lat, int audio_channels, int n_audio,
                  int C_audio, h3_bf16* hn, float* lat_video, float* lat_audio, float sigma_video,
                  float sigma_video_next, float sigma_audio, float sigma_audio_next, h3_bf16* lat_video_bf16,
                  h3_bf16* lat_audio_bf16, void* stream) {
  H3_TRACE();
  return head_impl(__func__, dims, ranges, x, W_vhead, W_ahead, T, Hl, Wl, C_lat, audio_channels, n_audio, C_audio,
                   hn, lat_video, lat_audio, true, sigma_video_next - sigma_video, sigma_audio_next - sigma_audio,
                   lat_video_bf16, lat_audio_bf16, stream);
}

size_t h3_adaln_workspace_bytes(int n, int c_dim) {
  return (n > 0 && c_dim > 0) ? (size_t)n * (size_t)c_dim * 2 : 0;
}

int h3_adaln_modulation(const h3_dims* dims, const float* c, int n, int c_dim, const h3_bf16* W, h3_bf16* ws,
                        float* mod, int64_t ld_mod, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  if (n <= 0) return fail(H3_ERR_SHAPE, "%s: n must be positive (got %d)", __func__, n);
  if (c_dim <= 0 || c_dim % 8 != 0)
    return fail(H3_ERR_UNSUPPORTED, "%s: c_dim must be a positive multiple of 8 (got %d)", __func__, c_dim);
  H3_REQUIRE_PTR(c);
  H3_REQUIRE_PTR(W);
  H3_REQUIRE_PTR(ws);
  H3_REQUIRE_PTR(mod);
  const int N = 18 * dims->D;
  if (ld_mod == 0) ld_mod = N;
  if (ld_mod < N || ld_mod % 4 != 0)
    return fail(H3_ERR_SHAPE, "%s: ld_mod must be 0 or a multiple of 4 of at least 18 D (got %lld)", __func__,
                (long long)ld_mod);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_silu_bf16(c, (long long)n * c_dim, reinterpret_cast<bf16*>(ws), st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_adaln_modulation: silu");
  GemmProblem p = gemm_base(ws, c_dim, n, c_dim, W, c_dim, N, (N + 255) / 256);
  p.epi.mode = EPI_STORE_F32;
  p.epi.M = n;
  p.epi.N = N;
  p.epi.ldo = ld_mod;
  p.epi.out = mod;
  e = launch_gemm(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_adaln_modulation: linear");
  return ok();
}

int h3_euler_step(float* lat, const float* vel, int64_t n, float sigma, float sigma_next, void* stream) {
  H3_TRACE();
  if (n < 0) return fail(H3_ERR_SHAPE, "h3_euler_step: n < 0");
  if (n == 0) return ok();
  H3_REQUIRE_PTR(lat);
  H3_REQUIRE_PTR(vel);
  cudaError_t e = launch_euler(lat, vel, (long long)n, sigma_next - sigma, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_euler_step");
  return ok();
}

int h3_text_refine(const h3_dims* dims, const h3_ranges* ranges, float* x, int n_blocks, const float* const* mods,
                   const float* pos, const h3_block_weights* w, const h3_block_buffers* buf, int flags, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (n_blocks < 0) return fail(H3_ERR_SHAPE, "%s: n_blocks must be >= 0", __func__);
  const int n_text = ranges->count[H3_TEXT];
  if (n_blocks == 0 || n_text == 0) return ok();
  if (ranges->start[H3_TEXT] != 0)
    return fail(H3_ERR_SHAPE, "%s: the text range must start at row 0 of the packing", __func__);
  if (!mods || !w) return fail(H3_ERR_NULL, "%s: mods and w are required", __func__);
  for (int b = 0; b < n_blocks; ++b)
    if (!mods[b]) return fail(H3_ERR_NULL, "%s: mods[%d] is NULL", __func__, b);
  h3_ranges t;
  memset(&t, 0, sizeof(t));
  t.start[H3_TEXT] = 0;
  t.count[H3_TEXT] = n_text;
  t.start[H3_AUDIO] = n_text;
  t.start[H3_VIDEO] = n_text;
  t.L = n_text;
  t.L_pad = (n_text + 127) / 128 * 128;
  for (int b = 0; b < n_blocks; ++b)
    H3_CHECK(h3_block_forward(dims, &t, x, mods[b], pos, &w[b], buf, flags, stream));
  return ok();
}

int h3_euler_step_bf16(float* lat, const float* vel, int64_t n, float sigma, float sigma_next, h3_bf16* lat_bf16,
                       void* stream) {
  H3_TRACE();
  if (n < 0) return fail(H3_ERR_SHAPE, "h3_euler_step_bf16: n < 0");
  if (n == 0) return ok();
  H3_REQUIRE_PTR(lat);
  H3_REQUIRE_PTR(vel);
  H3_REQUIRE_PTR(lat_bf16);
  cudaError_t e = launch_euler_bf16(lat, vel, (long long)n, sigma_next - sigma, reinterpret_cast<bf16*>(lat_bf16),
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_euler_step_bf16");
  return ok();
}

int h3_block_forward(const h3_dims* dims, const h3_ranges* ranges, float* x, const float* mod, const float* pos,
                     const h3_block_weights* w, const h3_block_buffers* buf, int flags, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (!w) return fail(H3_ERR_NULL, "%s: weights is NULL", __func__);
  if (!buf) return fail(H3_ERR_NULL, "%s: buffers is NULL", __func__);
  if (flags & ~H3_QK_NORM_ROPE_IN_QKV) return fail(H3_ERR_UNSUPPORTED, "%s: unknown flags", __func__);
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(mod);
  H3_REQUIRE_PTR(pos);
  H3_REQUIRE_PTR(w->Wqkv);
  H3_REQUIRE_PTR(w->qn_w);
  H3_REQUIRE_PTR(w->kn_w);
  H3_REQUIRE_PTR(w->Wo);
  H3_REQUIRE_PTR(w->Wgu);
  H3_REQUIRE_PTR(w->Wd);
  H3_REQUIRE_PTR(buf->xm);
  H3_REQUIRE_PTR(buf->q);
  H3_REQUIRE_PTR(buf->k);
  H3_REQUIRE_PTR(buf->v);
  H3_REQUIRE_PTR(buf->o);
  H3_REQUIRE_PTR(buf->ws);
  H3_CHECK(h3_adaln_norm_modulate(dims, ranges, x, mod, H3_MSA, buf->xm, stream));
  H3_CHECK(h3_qkv_qknorm_mrope(dims, ranges, buf->xm, w->Wqkv, w->qn_w, w->kn_w, pos, flags, buf->q, buf->k, buf->v,
                               stream));
  H3_CHECK(h3_attention(dims, ranges, buf->q, buf->k, buf->v, w->qn_w, w->kn_w, pos, flags, buf->o, stream));
  H3_CHECK(h3_gated_residual(dims, ranges, x, buf->o, w->Wo, mod, H3_MSA, stream));
  H3_CHECK(h3_adaln_norm_modulate(dims, ranges, x, mod, H3_MLP, buf->xm, stream));
  H3_CHECK(h3_ffn_swiglu(dims, ranges, x, buf->xm, w->Wgu, w->Wd, mod, buf->ws, stream));
  return ok();
}

int h3_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  H3_TRACE();
  if (limit_ns == 0 || limit_ns > 10000000000ull)
    return fail(H3_ERR_SHAPE, "h3_selftest_wait_timeout: limit must be in (0, 10 s]");
  cudaError_t e = launch_wait_timeout_selftest((unsigned long long)limit_ns, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_selftest_wait_timeout");
  return ok();
}

int h3_device_status(void* stream, int* code_out) {
  H3_TRACE();
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_device_status: synchronize");
  int code = 0;
  e = cudaMemcpyFromSymbol(&code, g_h3_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "h3_device_status: read");
  if (code != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_h3_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "h3_device_status: clear");
  }
  if (code_out) *code_out = code;
  if (code == 2)
    return fail(H3_ERR_BOUND, "h3_device_status: attention with its norm and RoPE in the prologue met scores "
                              "outside the bound its norm weights give (those rows hold NaN)");
  if (code != 0) return fail(H3_ERR_TIMEOUT, "h3_device_status: a device-side wait gave up (code %d)", code);
  return ok();
}

int h3_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return fail(H3_ERR_SHAPE, "h3_set_wait_limit_ns: limit must be > 0");
  unsigned long long v = ns;
  cudaError_t e = cudaMemcpyToSymbol(g_h3_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "h3_set_wait_limit_ns");
  return ok();
}

}  // extern "C"

// Workspace-free variant of h3_ffn_swiglu (uses this file's checks and launcher).
#include "h3_fp8.cu"
#include "h3_sp.cu"
#include "h3_noalloc.cu"

// The e4m3 (FP8) entry points: row quantisation, the modulated LayerNorm
// with e4m3 output, and the block's four GEMMs on e4m3 operands through the
// same tcgen05 kernels and fused epilogues as the bf16 path (kind::f8f6f4;
// the epilogue scales the fp32 accumulator by the row scale of A and the
// output-channel scale of B first).  The pages report community FP8
// quantisations of the trunk ("H3's omni-modal ambition" (0539edu.com),
// ecosystem paragraph) but fix no format; the format is OCP OFP8 E4M3 with
// one scale per token and one per output channel.
//
// Included into h3_api.cu (one translation unit): it uses that file's
// argument checks and GEMM problem builders.

namespace {

// Offsets inside the h3_ffn_swiglu_e4m3 workspace: bf16 h, then its codes,
// then its row scales (each offset a multiple of 256 bytes since L_pad is a
// multiple of 128 and F of 128).
struct FfnE4m3Ws {
  size_t h_bf16, h_codes, h_scale, total;
};
FfnE4m3Ws ffn_e4m3_layout(int L_pad, int F) {
  FfnE4m3Ws w;
  w.h_bf16 = 0;
  w.h_codes = (size_t)L_pad * F * 2;
  w.h_scale = w.h_codes + (size_t)L_pad * F;
  w.total = w.h_scale + (size_t)L_pad * 4;
  return w;
}

GemmProblem with_e4m3(GemmProblem p, const float* a_scale, const float* b_scale) {
  p.f8 = 1;
  p.a_scale = a_scale;
  p.b_scale = b_scale;
  return p;
}

}  // namespace

extern "C" {

int h3_quantize_rows_e4m3(const h3_bf16* in, int64_t ld_in, int rows, int cols, h3_e4m3* q, int64_t ld_q,
                          float* scale, void* stream) {
  H3_TRACE();
  if (rows < 0 || cols <= 0 || cols % 8 || ld_in < cols || ld_q < cols || ld_in % 8 || ld_q % 8)
    return fail(H3_ERR_SHAPE, "%s: need rows >= 0, cols > 0, cols, ld_in, ld_q multiples of 8, ld >= cols",
                __func__);
  if (rows == 0) return ok();
  H3_REQUIRE_PTR(in);
  H3_REQUIRE_PTR(q);
  H3_REQUIRE_PTR(scale);
  cudaError_t e = launch_quantize_rows_e4m3(reinterpret_cast<const bf16*>(in), (long)ld_in, rows, cols, q,
                                            (long)ld_q, scale, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_quantize_rows_e4m3");
  return ok();
}

int h3_adaln_norm_modulate_e4m3(const h3_dims* dims, const h3_ranges* ranges, const float* x, const float* mod,
                                int branch, h3_e4m3* xq, float* xs, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (branch != H3_MSA && branch != H3_MLP) return fail(H3_ERR_SHAPE, "%s: branch must be H3_MSA or H3_MLP", __func__);
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(mod);
  H3_REQUIRE_PTR(xq);
  H3_REQUIRE_PTR(xs);
  cudaError_t e = launch_ln_modulate_e4m3(x, mod, branch, ranges->start, ranges->count, ranges->L, ranges->L_pad,
                                          dims->D, dims->eps_ln, xq, xs, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_adaln_norm_modulate_e4m3");
  return ok();
}

int h3_qkv_qknorm_mrope_e4m3(const h3_dims* dims, const h3_ranges* ranges, const h3_e4m3* xq, const float* xs,
                             const h3_e4m3* Wq, const float* Ws, const h3_bf16* qn_w, const h3_bf16* kn_w,
                             const float* pos, int flags, h3_bf16* q, h3_bf16* k, h3_bf16* v, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (!(flags & H3_QK_NORM_ROPE_IN_QKV))
    return fail(H3_ERR_UNSUPPORTED, "%s: flags must include H3_QK_NORM_ROPE_IN_QKV in this version", __func__);
  H3_REQUIRE_PTR(xq);
  H3_REQUIRE_PTR(Wq);
  H3_REQUIRE_PTR(xs);
  H3_REQUIRE_PTR(Ws);
  H3_REQUIRE_PTR(qn_w);
  H3_REQUIRE_PTR(kn_w);
  H3_REQUIRE_PTR(pos);
  H3_REQUIRE_PTR(q);
  H3_REQUIRE_PTR(k);
  H3_REQUIRE_PTR(v);
  if (flags & ~(H3_QK_NORM_ROPE_IN_QKV | H3_QK_E4M3)) return fail(H3_ERR_UNSUPPORTED, "%s: unknown flags", __func__);
  GemmProblem p = with_e4m3(qkv_problem(dims, ranges, xq, Wq, qn_w, kn_w, pos, q, k, v), xs, Ws);
  p.epi.qk_e4m3 = (flags & H3_QK_E4M3) ? 1 : 0;
  cudaError_t e = launch_gemm(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_qkv_qknorm_mrope_e4m3");
  return ok();
}

int h3_gated_residual_e4m3(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_e4m3* oq,
                           const float* os, const h3_e4m3* Wq, const float* Ws, const float* mod, int branch,
                           void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (branch != H3_MSA && branch != H3_MLP) return fail(H3_ERR_SHAPE, "%s: branch must be H3_MSA or H3_MLP", __func__);
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(oq);
  H3_REQUIRE_PTR(Wq);
  H3_REQUIRE_PTR(os);
  H3_REQUIRE_PTR(Ws);
  H3_REQUIRE_PTR(mod);
  GemmProblem p = with_e4m3(gated_problem(dims, ranges, x, oq, dims->I, Wq, mod, 3 * branch + 2), os, Ws);
  cudaError_t e = launch_gemm(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "h3_gated_residual_e4m3");
  return ok();
}

size_t h3_ffn_e4m3_workspace_bytes(const h3_dims* dims, int L_pad) {
  if (!dims || L_pad <= 0 || dims->F <= 0) return 0;
  return ffn_e4m3_layout(L_pad, dims->F).total;
}

int h3_ffn_swiglu_e4m3(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_e4m3* xq,
                       const float* xs, const h3_e4m3* Wgu_q, const float* Wgu_s, const h3_e4m3* Wd_q,
                       const float* Wd_s, const float* mod, void* ws, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(xq);
  H3_REQUIRE_PTR(Wgu_q);
  H3_REQUIRE_PTR(Wd_q);
  H3_REQUIRE_PTR(xs);
  H3_REQUIRE_PTR(Wgu_s);
  H3_REQUIRE_PTR(Wd_s);
  H3_REQUIRE_PTR(mod);
  H3_REQUIRE_PTR(ws);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(H3_ERR_ALIGN, "%s: ws must be 256-byte aligned", __func__);
  const int F = dims->F, Lp = ranges->L_pad;
  const FfnE4m3Ws lay = ffn_e4m3_layout(Lp, F);
  uint8_t* base = static_cast<uint8_t*>(ws);
  bf16* h = reinterpret_cast<bf16*>(base + lay.h_bf16);
  uint8_t* hq = base + lay.h_codes;
  float* hs = reinterpret_cast<float*>(base + lay.h_scale);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GemmProblem p1 = with_e4m3(swiglu_problem(dims, Lp, xq, Wgu_q, h), xs, Wgu_s);
  cudaError_t e = launch_gemm(p1, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu_e4m3: gate/up");
  e = launch_quantize_rows_e4m3(h, F, Lp, F, hq, F, hs, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu_e4m3: quantise h");
  GemmProblem p2 = with_e4m3(gated_problem(dims, ranges, x, hq, F, Wd_q, mod, 5), hs, Wd_s);
  e = launch_gemm(p2, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu_e4m3: down");
  return ok();
}

int h3_block_forward_e4m3(const h3_dims* dims, const h3_ranges* ranges, float* x, const float* mod,
                          const float* pos, const h3_block_weights_e4m3* w, const h3_block_buffers_e4m3* buf,
                          int flags, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  if (!w) return fail(H3_ERR_NULL, "%s: weights is NULL", __func__);
  if (!buf) return fail(H3_ERR_NULL, "%s: buffers is NULL", __func__);
  if (!(flags & H3_QK_NORM_ROPE_IN_QKV))
    return fail(H3_ERR_UNSUPPORTED, "%s: flags must include H3_QK_NORM_ROPE_IN_QKV in this version", __func__);
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(mod);
  H3_REQUIRE_PTR(pos);
  H3_REQUIRE_PTR(w->Wqkv);
  H3_REQUIRE_PTR(w->Wo);
  H3_REQUIRE_PTR(w->Wgu);
  H3_REQUIRE_PTR(w->Wd);
  H3_REQUIRE_PTR(w->Wqkv_s);
  H3_REQUIRE_PTR(w->Wo_s);
  H3_REQUIRE_PTR(w->Wgu_s);
  H3_REQUIRE_PTR(w->Wd_s);
  H3_REQUIRE_PTR(w->qn_w);
  H3_REQUIRE_PTR(w->kn_w);
  H3_REQUIRE_PTR(buf->xq);
  H3_REQUIRE_PTR(buf->oq);
  H3_REQUIRE_PTR(buf->o);
  H3_REQUIRE_PTR(buf->xs);
  H3_REQUIRE_PTR(buf->os);
  H3_REQUIRE_PTR(buf->q);
  H3_REQUIRE_PTR(buf->k);
  H3_REQUIRE_PTR(buf->v);
  H3_REQUIRE_PTR(buf->ws);
  if (reinterpret_cast<uintptr_t>(buf->ws) & 255u)
    return fail(H3_ERR_ALIGN, "%s: ws must be 256-byte aligned", __func__);
  const int I = dims->I, Lp = ranges->L_pad;
  H3_CHECK(h3_adaln_norm_modulate_e4m3(dims, ranges, x, mod, H3_MSA, buf->xq, buf->xs, stream));
  H3_CHECK(h3_qkv_qknorm_mrope_e4m3(dims, ranges, buf->xq, buf->xs, w->Wqkv, w->Wqkv_s, w->qn_w, w->kn_w, pos,
                                    flags, buf->q, buf->k, buf->v, stream));
  H3_CHECK(h3_attention(dims, ranges, buf->q, buf->k, buf->v, w->qn_w, w->kn_w, pos, flags, buf->o, stream));
  H3_CHECK(h3_quantize_rows_e4m3(buf->o, I, Lp, I, buf->oq, I, buf->os, stream));
  H3_CHECK(h3_gated_residual_e4m3(dims, ranges, x, buf->oq, buf->os, w->Wo, w->Wo_s, mod, H3_MSA, stream));
  H3_CHECK(h3_adaln_norm_modulate_e4m3(dims, ranges, x, mod, H3_MLP, buf->xq, buf->xs, stream));
  H3_CHECK(h3_ffn_swiglu_e4m3(dims, ranges, x, buf->xq, buf->xs, w->Wgu, w->Wgu_s, w->Wd, w->Wd_s, mod, buf->ws,
                              stream));
  return ok();
}

}  // extern "C"

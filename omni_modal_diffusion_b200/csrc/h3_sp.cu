// Sequence parallelism (Ulysses) for the block: the layout of a rank's shard
// and the two exchange points, each fused into the kernel that produces the
// data (bf16 q, k, v, or with e4m3 operands e4m3 q, k codes and bf16 v).  "MiniMax-H3 paper reading" (gojay.top) §7.2 gives Ulysses degree 4
// as the trunk's deployment; the all-to-all structure (tokens -> heads before
// attention, heads -> tokens after it) is the method's, the fusion is ours:
//   - h3_qkv_qknorm_mrope_sp: the QKV epilogue stores head group g of the
//     shard into rank g's q/k/v buffers at the shard's global rows;
//   - h3_attention_sp: each output row is stored into its owner's o buffer at
//     this rank's head columns.
// The kernels write through plain device pointers (peer memory mapped by the
// caller, or local buffers when the ranks share a GPU); there is no TMA or
// bulk load from another GPU's memory.
//
// Included into h3_api.cu (one translation unit): it uses that file's
// argument checks and GEMM problem builders.

namespace {

int check_layout(const h3_dims* dims, const h3_sp_layout* l, const char* fn) {
  if (!l) return fail(H3_ERR_NULL, "%s: layout is NULL", fn);
  if (l->n_ranks < 1 || l->n_ranks > H3_SP_MAX_RANKS || l->rank < 0 || l->rank >= l->n_ranks)
    return fail(H3_ERR_SHAPE, "%s: rank %d of %d ranks (at most %d)", fn, l->rank, l->n_ranks, H3_SP_MAX_RANKS);
  if (dims->H % l->n_ranks || l->heads != dims->H / l->n_ranks)
    return fail(H3_ERR_SHAPE, "%s: H (%d) must split evenly into %d ranks of %d heads", fn, dims->H, l->n_ranks,
                l->heads);
  if (l->L_shard <= 0 || l->L_shard % 128 || l->L_total != l->n_ranks * l->L_shard ||
      l->row0 != l->rank * l->L_shard || l->L <= (l->n_ranks - 1) * l->L_shard || l->L > l->L_total)
    return fail(H3_ERR_SHAPE, "%s: inconsistent layout (use h3_sp_make_layout)", fn);
  return H3_OK;
}

int check_peers(const h3_sp_peers* p, int n, bool qkv, bool o, const char* fn) {
  if (!p) return fail(H3_ERR_NULL, "%s: peers is NULL", fn);
  for (int g = 0; g < n; ++g) {
    const void* ptrs[4] = {p->q[g], p->k[g], p->v[g], p->o[g]};
    for (int i = 0; i < 4; ++i) {
      if ((i < 3 && !qkv) || (i == 3 && !o)) continue;
      if (!ptrs[i]) return fail(H3_ERR_NULL, "%s: peer buffer %c[%d] is NULL", fn, "qkvo"[i], g);
      if (!aligned16(ptrs[i])) return fail(H3_ERR_ALIGN, "%s: peer buffer %c[%d] is not 16-byte aligned", fn, "qkvo"[i], g);
    }
  }
  return H3_OK;
}

}  // namespace

extern "C" {

int h3_sp_make_layout(const h3_dims* dims, const h3_ranges* global, int n_ranks, int rank, h3_sp_layout* out,
                      h3_ranges* shard) {
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(global, __func__));
  if (!out || !shard) return fail(H3_ERR_NULL, "%s: out and shard are required", __func__);
  if (n_ranks < 1 || n_ranks > H3_SP_MAX_RANKS || rank < 0 || rank >= n_ranks)
    return fail(H3_ERR_SHAPE, "%s: rank %d of %d ranks (at most %d)", __func__, rank, n_ranks, H3_SP_MAX_RANKS);
  if (dims->H % n_ranks) return fail(H3_ERR_SHAPE, "%s: H (%d) is not a multiple of %d ranks", __func__, dims->H, n_ranks);
  const long L = global->L;
  const long per = (L + n_ranks - 1) / n_ranks;
  const long L_shard = (per + 127) / 128 * 128;
  if (L <= (long)(n_ranks - 1) * L_shard)
    return fail(H3_ERR_SHAPE, "%s: %ld tokens leave the last of %d shards of %ld rows empty", __func__, L, n_ranks,
                L_shard);
  h3_sp_layout l;
  l.n_ranks = n_ranks;
  l.rank = rank;
  l.L = (int)L;
  l.L_shard = (int)L_shard;
  l.L_total = (int)(L_shard * n_ranks);
  l.row0 = (int)(L_shard * rank);
  l.heads = dims->H / n_ranks;
  h3_ranges s;
  const long a = l.row0, b = l.row0 + L_shard;
  for (int m = 0; m < 3; ++m) {
    const long s0 = global->start[m], s1 = s0 + global->count[m];
    const long lo = s0 > a ? s0 : a, hi = s1 < b ? s1 : b;
    s.start[m] = (int)((hi > lo ? lo : a) - a);
    s.count[m] = (int)(hi > lo ? hi - lo : 0);
  }
  s.L = (int)((L < b ? L : b) - a);
  s.L_pad = (int)L_shard;
  *out = l;
  *shard = s;
  return ok();
}

int h3_qkv_qknorm_mrope_sp(const h3_dims* dims, const h3_ranges* shard, const h3_sp_layout* layout,
                           const h3_bf16* xm, const h3_bf16* Wqkv, const h3_bf16* qn_w, const h3_bf16* kn_w,
                           const float* pos, int flags, const h3_sp_peers* peers, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(shard, __func__));
  H3_CHECK(check_layout(dims, layout, __func__));
  if (shard->L_pad != layout->L_shard)
    return fail(H3_ERR_SHAPE, "%s: shard L_pad (%d) != layout L_shard (%d)", __func__, shard->L_pad, layout->L_shard);
  if (!(flags & H3_QK_NORM_ROPE_IN_QKV))
    return fail(H3_ERR_UNSUPPORTED, "%s: flags must include H3_QK_NORM_ROPE_IN_QKV in this version", __func__);
  if (flags & ~H3_QK_NORM_ROPE_IN_QKV)
    return fail(H3_ERR_UNSUPPORTED, "%s: only H3_QK_NORM_ROPE_IN_QKV (e4m3 q/k are not sequence parallel)", __func__);
  H3_REQUIRE_PTR(xm);
  H3_REQUIRE_PTR(Wqkv);
  H3_REQUIRE_PTR(qn_w);
  H3_REQUIRE_PTR(kn_w);
  H3_REQUIRE_PTR(pos);
  H3_CHECK(check_peers(peers, layout->n_ranks, true, false, __func__));
  GemmProblem p = qkv_problem(dims, shard, xm, Wqkv, qn_w, kn_w, pos, nullptr, nullptr, nullptr);
  GemmEpilogue& e = p.epi;
  e.sp_n = layout->n_ranks;
  e.sp_heads = layout->heads;
  e.sp_L_total = layout->L_total;
  e.sp_row0 = layout->row0;
  for (int g = 0; g < layout->n_ranks; ++g) {
    e.sp_q[g] = reinterpret_cast<bf16*>(peers->q[g]);
    e.sp_k[g] = reinterpret_cast<bf16*>(peers->k[g]);
    e.sp_v[g] = reinterpret_cast<bf16*>(peers->v[g]);
  }
  cudaError_t err = launch_gemm(p, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "h3_qkv_qknorm_mrope_sp");
  return ok();
}

int h3_qkv_qknorm_mrope_sp_e4m3(const h3_dims* dims, const h3_ranges* shard, const h3_sp_layout* layout,
                                const h3_e4m3* xq, const float* xs, const h3_e4m3* Wq, const float* Ws,
                                const h3_bf16* qn_w, const h3_bf16* kn_w, const float* pos, int flags,
                                const h3_sp_peers* peers, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(shard, __func__));
  H3_CHECK(check_layout(dims, layout, __func__));
  if (shard->L_pad != layout->L_shard)
    return fail(H3_ERR_SHAPE, "%s: shard L_pad (%d) != layout L_shard (%d)", __func__, shard->L_pad, layout->L_shard);
  if (!(flags & H3_QK_NORM_ROPE_IN_QKV))
    return fail(H3_ERR_UNSUPPORTED, "%s: flags must include H3_QK_NORM_ROPE_IN_QKV in this version", __func__);
  if (flags & ~(H3_QK_NORM_ROPE_IN_QKV | H3_QK_E4M3)) return fail(H3_ERR_UNSUPPORTED, "%s: unknown flags", __func__);
  H3_REQUIRE_PTR(xq);
  H3_REQUIRE_PTR(xs);
  H3_REQUIRE_PTR(Wq);
  H3_REQUIRE_PTR(Ws);
  H3_REQUIRE_PTR(qn_w);
  H3_REQUIRE_PTR(kn_w);
  H3_REQUIRE_PTR(pos);
  H3_CHECK(check_peers(peers, layout->n_ranks, true, false, __func__));
  GemmProblem p = with_e4m3(qkv_problem(dims, shard, xq, Wq, qn_w, kn_w, pos, nullptr, nullptr, nullptr), xs, Ws);
  GemmEpilogue& e = p.epi;
  e.qk_e4m3 = (flags & H3_QK_E4M3) ? 1 : 0;
  e.sp_n = layout->n_ranks;
  e.sp_heads = layout->heads;
  e.sp_L_total = layout->L_total;
  e.sp_row0 = layout->row0;
  for (int g = 0; g < layout->n_ranks; ++g) {
    e.sp_q[g] = reinterpret_cast<bf16*>(peers->q[g]);
    e.sp_k[g] = reinterpret_cast<bf16*>(peers->k[g]);
    e.sp_v[g] = reinterpret_cast<bf16*>(peers->v[g]);
  }
  cudaError_t err = launch_gemm(p, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "h3_qkv_qknorm_mrope_sp_e4m3");
  return ok();
}

int h3_attention_sp(const h3_dims* dims, const h3_sp_layout* layout, const h3_sp_peers* peers,
                    const h3_bf16* qn_w, const h3_bf16* kn_w, int flags, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_layout(dims, layout, __func__));
  if (!(flags & H3_QK_NORM_ROPE_IN_QKV))
    return fail(H3_ERR_UNSUPPORTED, "%s: flags must include H3_QK_NORM_ROPE_IN_QKV in this version", __func__);
  if (flags & ~(H3_QK_NORM_ROPE_IN_QKV | H3_QK_E4M3)) return fail(H3_ERR_UNSUPPORTED, "%s: unknown flags", __func__);
  H3_CHECK(check_peers(peers, layout->n_ranks, false, true, __func__));
  const int r = layout->rank;
  if (!peers->q[r] || !peers->k[r] || !peers->v[r])
    return fail(H3_ERR_NULL, "%s: this rank's q, k, v buffers are required", __func__);
  if (!aligned16(peers->q[r]) || !aligned16(peers->k[r]) || !aligned16(peers->v[r]))
    return fail(H3_ERR_ALIGN, "%s: this rank's q, k, v buffers must be 16-byte aligned", __func__);
  if (qn_w || kn_w || (flags & H3_QK_E4M3)) {  // e4m3 codes: their scales follow from the norm weights
    H3_REQUIRE_PTR(qn_w);
    H3_REQUIRE_PTR(kn_w);
  }
  AttnProblem p;
  memset(&p, 0, sizeof(p));
  p.qk8 = (flags & H3_QK_E4M3) ? 1 : 0;
  p.qn_w = reinterpret_cast<const bf16*>(qn_w);
  p.kn_w = reinterpret_cast<const bf16*>(kn_w);
  p.q = reinterpret_cast<const bf16*>(peers->q[r]);
  p.k = reinterpret_cast<const bf16*>(peers->k[r]);
  p.v = reinterpret_cast<const bf16*>(peers->v[r]);
  p.H = layout->heads;
  p.L = layout->L;
  p.L_pad = layout->L_total;
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->head_dim));
  p.sp_n = layout->n_ranks;
  p.sp_L_shard = layout->L_shard;
  p.sp_head0 = r * layout->heads;
  p.sp_ld = (long)dims->H * 128;
  for (int g = 0; g < layout->n_ranks; ++g) p.sp_o[g] = reinterpret_cast<bf16*>(peers->o[g]);
  cudaError_t err = launch_attention(p, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "h3_attention_sp");
  return ok();
}

}  // extern "C"

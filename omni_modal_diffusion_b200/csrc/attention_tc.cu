// Non-causal flash attention on tcgen05 tensor cores, one CTA per
// (128-query tile, head).  softmax(q k^T / sqrt(128)) v over all valid
// tokens of the packed sequence; keys at or beyond L are masked ("MiniMax-H3:
// native joint audio-video generation" (note.shouss.top) §5: full non-causal
// attention, padding handled by the sequence boundary).
//
// Warp 0: TMA producer (Q once, K/V tiles through a 2-stage ring).
// Warp 1: TMEM owner and MMA issuer: S_j = Q K_j^T into one of two TMEM
//         S buffers, O += P_j V_j into the TMEM O accumulator.
// Warps 2-5: one query row per thread: read S_j from TMEM, online softmax in
//         the log2 domain with a lazily moved reference max (O is rescaled in
//         TMEM only when the row max grows by more than 2^8), write P_j as
//         bf16 into 128-byte-swizzled shared memory, and finally O / l.
#include "h3_internal.cuh"
#include "ptx.cuh"

namespace h3 {

namespace attn_detail {
constexpr int NUM_THREADS = 192;
constexpr int TILE = 128;
constexpr int HALF_BYTES = TILE * 64 * 2;  // 128 rows x 64 bf16 = 16 KB
constexpr int TILE_BYTES = 2 * HALF_BYTES; // 32 KB
constexpr int SMEM_Q = 0;
constexpr int SMEM_K = SMEM_Q + TILE_BYTES;       // 2 stages
constexpr int SMEM_V = SMEM_K + 2 * TILE_BYTES;   // 2 stages
constexpr int SMEM_P = SMEM_V + 2 * TILE_BYTES;
constexpr int SMEM_BAR = SMEM_P + TILE_BYTES;
constexpr int SMEM_BYTES = SMEM_BAR + 256 + 1024;
constexpr int TMEM_COLS = 512;                    // S0 | S1 | O | unused
constexpr float RESCALE_THRESHOLD = 8.0f;         // log2 units

__global__ void __launch_bounds__(NUM_THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ out, int H, int L, int L_pad,
                        float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem + SMEM_Q;
  uint8_t* sK = smem + SMEM_K;
  uint8_t* sV = smem + SMEM_V;
  uint8_t* sP = smem + SMEM_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* kv_empty = bars + 5;  // [2]
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* s_free = bars + 9;    // [2]
  uint64_t* p_full = bars + 11;
  uint64_t* pv_done = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = blockIdx.x, h = blockIdx.y;
  const int nkv = (L + TILE - 1) / TILE;
  const int row0 = h * L_pad;  // first row of this head in the [H*L_pad, 128] views

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      tma_load_2d(sQ, &tmQ, q_full, 0, row0 + qt * TILE);
      tma_load_2d(sQ + HALF_BYTES, &tmQ, q_full, 64, row0 + qt * TILE);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1)) break;
        uint8_t* dk = sK + st * TILE_BYTES;
        uint8_t* dv = sV + st * TILE_BYTES;
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        tma_load_2d(dk, &tmK, &k_full[st], 0, row0 + j * TILE);
        tma_load_2d(dk + HALF_BYTES, &tmK, &k_full[st], 64, row0 + j * TILE);
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        tma_load_2d(dv, &tmV, &v_full[st], 0, row0 + j * TILE);
        tma_load_2d(dv + HALF_BYTES, &tmV, &v_full[st], 64, row0 + j * TILE);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      const uint32_t idesc_o = idesc_bf16_f32(128, 128, true);  // V is MN-major (d contiguous)
      const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0);
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(p_full, i & 1)) return false;
        if (!mbar_wait(&v_full[i & 1], (i >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + (i & 1) * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = sdesc_sw128(p_addr + (kk >> 2) * HALF_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(v_addr + kk * 2048, HALF_BYTES, 1024);
          umma_bf16(tmem + 256, ad, bd, idesc_o, (i | kk) != 0 ? 1u : 0u);
        }
        umma_commit(pv_done);
        umma_commit(&kv_empty[i & 1]);
        return true;
      };
      for (int j = 0; j < nkv && ok; ++j) {
        const int b = j & 1;
        if (!mbar_wait(&k_full[b], (j >> 1) & 1)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&s_free[b], ((j - 2) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + b * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(q_addr + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_addr + off, 16, 1024);
          umma_bf16(tmem + b * 128, ad, bd, idesc_s, kk != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[b]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(nkv - 1);
    }
  } else {
    const int qw = warp & 3;
    const int r = qw * 32 + lane;  // query row inside the tile
    const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    uint8_t* prow = sP + r * 128;
    const int sw = r & 7;
    for (int j = 0; j < nkv; ++j) {
      const int b = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (j >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + b * 128 + c * 32, reinterpret_cast<uint32_t*>(s + c * 32));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);

      const int valid = L - j * TILE;  // keys [0, valid) of this tile are real
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        if (c >= valid) s[c] = -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      const float m_new = fmaxf(m_ref, mx * scale_log2);
      const bool move = (m_new - m_ref) > RESCALE_THRESHOLD;  // true at j == 0 (m_ref = -inf)
      const float m_use = move ? m_new : m_ref;
      const float alpha = move ? ex2_approx(m_ref - m_new) : 1.0f;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = ex2_approx(fmaf(s[c], scale_log2, -m_use));
        rs += s[c];
      }
      l_sum = fmaf(l_sum, alpha, rs);
      m_ref = m_use;

      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, move)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            const uint32_t ta = tmem + lane_off + 256 + c * 32;
            tmem_ld32(ta, reinterpret_cast<uint32_t*>(o));
            tmem_wait_ld();
#pragma unroll
            for (int d = 0; d < 32; ++d) o[d] *= alpha;
            tmem_st32(ta, reinterpret_cast<const uint32_t*>(o));
          }
          tmem_wait_st();
        }
      }
      // P row -> shared memory, 128-byte swizzle: 16-byte chunk q of the row
      // lands at chunk q ^ (row % 8)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float* src = s + hf * 64 + q * 8;
          uint4 w;
          w.x = pack_bf16x2(src[0], src[1]);
          w.y = pack_bf16x2(src[2], src[3]);
          w.z = pack_bf16x2(src[4], src[5]);
          w.w = pack_bf16x2(src[6], src[7]);
          *reinterpret_cast<uint4*>(prow + hf * HALF_BYTES + ((q ^ sw) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (nkv - 1) & 1));
    if (ok) {
      tc_fence_after();
      const int grow = qt * TILE + r;
      const float inv = (grow < L) ? 1.0f / l_sum : 0.0f;
      bf16* dst = out + (long)grow * (H * 128) + h * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_off + 256 + c * 32, reinterpret_cast<uint32_t*>(o));
        tmem_wait_ld();
#pragma unroll
        for (int d = 0; d < 32; d += 8) {
          uint4 w;
          w.x = pack_bf16x2(o[d] * inv, o[d + 1] * inv);
          w.y = pack_bf16x2(o[d + 2] * inv, o[d + 3] * inv);
          w.z = pack_bf16x2(o[d + 4] * inv, o[d + 5] * inv);
          w.w = pack_bf16x2(o[d + 6] * inv, o[d + 7] * inv);
          *reinterpret_cast<uint4*>(dst + c * 32 + d) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace attn_detail
using namespace attn_detail;

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                    uint32_t box_rows);

cudaError_t launch_attention(const AttnProblem& p, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t err =
        cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_detail::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    attr_set = true;
  }
  CUtensorMap tq, tk, tv;
  const uint64_t rows = (uint64_t)p.H * p.L_pad;
  if (!make_tmap_bf16(&tq, p.q, rows, 128, 128, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tk, p.k, rows, 128, 128, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tv, p.v, rows, 128, 128, 128)) return cudaErrorInvalidValue;
  dim3 grid(p.L_pad / attn_detail::TILE, p.H);
  attention_tc_kernel<<<grid, attn_detail::NUM_THREADS, attn_detail::SMEM_BYTES, stream>>>(tq, tk, tv, p.o, p.H, p.L, p.L_pad, p.scale_log2);
  return cudaGetLastError();
}

}  // namespace h3

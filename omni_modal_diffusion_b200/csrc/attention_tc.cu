// Non-causal flash attention on tcgen05 tensor cores.  softmax(q k^T /
// sqrt(128)) v over all valid tokens of the packed sequence; keys at or beyond
// L are masked ("MiniMax-H3: native joint audio-video generation"
// (note.shouss.top) §5: full non-causal attention, padding handled by the
// sequence boundary).
//
// One CTA per (pair of 128-query tiles, head); the two query tiles share the
// K/V stream and ping-pong on the tensor core:
//   Warp 0     TMA producer: both Q tiles once, K/V tiles through a 2-stage ring.
//   Warp 1     TMEM owner and MMA issuer (the whole warp, converged), in the order
//              S0_0 S1_0 | PV0_0 S0_1 | PV1_0 S1_1 | PV0_1 S0_2 | ...
//              so that while one softmax warpgroup works on its S tile the
//              tensor core runs the other tile's PV and next S.
//   Warps 2-5  softmax of query tile 0, warps 6-9 of tile 1, one query row
//              per thread: S from TMEM, online softmax in the log2 domain
//              against a lazily moved reference (the first key tile's row
//              max; it moves only when a 64-key half's exponentials sum past
//              2^16, with O rescaled in TMEM and that half redone), P written
//              back over S in TMEM as packed bf16 in two halves of 64 keys,
//              each released to the PV MMA as soon as it is stored, finally
//              O / l to global memory.
// Optionally (H3_ATTN_POLY_COLS of every 16 columns, default 0) part of each
// row's exponentials are taken on the FMA pipe (exp2_fma2) instead of the
// MUFU unit; measured slower on B200.  attention_split_kernel
// (attention_split.cu) replaces this kernel when q and k come with their norm
// weights; this one then recomputes only the CTAs that kernel leaves to it.
// With an odd number of query tiles the last CTA runs tile 0 alone.
// TMEM (512 columns): tile t owns columns [256t, 256t + 128) for S / P and
// [256t + 128, 256t + 256) for O.
// The QK8 instantiation (H3_QK_E4M3) reads Q and K as e4m3 codes with one
// static scale each and takes S with kind::f8f6f4 MMAs (half the tensor time
// of the bf16 S, which sits on each tile's critical chain); P V stays bf16.
#include "h3_internal.cuh"
#include "ptx.cuh"

namespace h3 {

namespace attn_detail {
// 8-column TMEM load / store (32 lanes x 8 columns), for the rare rescale of
// O where the softmax registers are all live
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
constexpr int NUM_THREADS = 320;
constexpr int TILE = 128;
constexpr int HALF_BYTES = TILE * 64 * 2;   // 128 rows x 64 bf16 = 16 KB
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // 32 KB
// Q and K tiles: bf16 (32 KB, two 64-column halves) or, with QK8, e4m3 codes
// (16 KB, one 128-byte row per token)
constexpr int VS = 2;  // V stages
template <bool QK8> struct Layout {
  static constexpr int QK_TILE = QK8 ? TILE * 128 : TILE_BYTES;
  static constexpr int Q = 0;                  // 2 query tiles
  static constexpr int K = Q + 2 * QK_TILE;    // 2 stages
  static constexpr int V = K + 2 * QK_TILE;    // VS stages
  static constexpr int BAR = V + VS * TILE_BYTES;
  static constexpr int BYTES = BAR + 256 + 1024;
  static_assert(BYTES <= 232448, "shared memory per CTA");
};
constexpr int TMEM_COLS = 512;
// Of every 16 key columns of a row, how many take their exponential on the
// FMA pipe (exp2_fma2) instead of the MUFU unit (0..16, even).
#ifndef H3_ATTN_POLY_COLS
#define H3_ATTN_POLY_COLS 0
#endif
static_assert(H3_ATTN_POLY_COLS >= 0 && H3_ATTN_POLY_COLS <= 16 && H3_ATTN_POLY_COLS % 2 == 0,
              "H3_ATTN_POLY_COLS: an even count of 0..16");
// S is read from TMEM in two 64-key halves (1: half 1 is loaded while P of
// half 0 is stored, and only 64 scores are live in registers at a time) or
// whole (0).
#ifndef H3_ATTN_S_HALVES
#define H3_ATTN_S_HALVES 1
#endif
// A 64-key half whose exponentials (against the current reference) sum past
// this moves the reference: every p of an accepted half is <= 2^16, so p, the
// row sum and O stay far from the fp32 range (and bf16 P keeps its relative
// precision at any scale).
constexpr float P_HALF_SUM_LIMIT = 65536.0f;
// How the MMA issuer waits: polling (1) or suspending try_wait (0).  The
// suspending wait leaves the issue slots of its sub-partition to the softmax
// warps that share it: 1.486 vs 1.499 ms at 7,904 tokens, equal at 32,160.
#ifndef H3_ATTN_MMA_SPIN
#define H3_ATTN_MMA_SPIN 0
#endif
#if H3_ATTN_MMA_SPIN
#define MMA_WAIT_WARP mbar_wait_spin_warp
#else
#define MMA_WAIT_WARP mbar_wait_warp
#endif

// Where output rows go: row R (of the L_pad rows this launch covers) to
// shard[R / L_shard], row R % L_shard, row stride ld, head column offset
// (head0 + h) * 128.  One shard for a plain launch; one per rank (the owners
// of the rows) for a sequence-parallel one.
struct AttnOut {
  long ld;
  int head0, L_shard;
  bf16* shard[8];
};

// RMSNorm + 3-D RoPE taken in the attention prologue (split kernel, PRO):
// positions [L_pad][3], the t | h | w section widths, the base, the norm eps
struct AttnRope {
  const float* pos;
  int rope_t, rope_h, rope_w;
  float theta, eps;
};

// QK8: Q and K are e4m3 codes of q * 448 / (sqrt(128) max|qn_w|) and of
// k * 448 / (sqrt(128) max|kn_w|); S = Q K^T is taken with kind::f8f6f4 MMAs
// and the two scales folded into the softmax scale.  P V stays bf16.
template <bool QK8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnOut out, int H, int L,
                        int L_pad, float scale_log2, const bf16* qn_w, const bf16* kn_w, int fixup) {
  // fixup: recompute only the CTAs that attention_split_kernel left to this
  // kernel (a NaN sentinel, bf16 0x7FC0, in their first output element)
  if (fixup) {
    const int g = blockIdx.x * 2 * TILE;
    const int owner = g / out.L_shard;
    const bf16* first = out.shard[owner] + (long)(g - owner * out.L_shard) * out.ld + (out.head0 + blockIdx.y) * 128;
    if (__bfloat16_as_ushort(*first) != (unsigned short)0x7FC0) return;
  }
  using LY = Layout<QK8>;
  constexpr int QK_TILE = LY::QK_TILE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem + LY::Q;
  uint8_t* sK = smem + LY::K;
  uint8_t* sV = smem + LY::V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2] per K stage
  uint64_t* k_empty = bars + 3;   // [2] per K stage: freed after the tile's last S MMA
  uint64_t* v_full = bars + 5;    // [VS] per V stage
  uint64_t* v_empty = bars + 8;   // [VS] per V stage: freed after the tile's last PV MMA
  uint64_t* s_full = bars + 11;   // [2] per query tile
  uint64_t* o_final = bars + 13;  // [2] per query tile
  uint64_t* p_full = bars + 15;   // [2 tiles][2 halves of the key tile]: P half in TMEM (4 warp arrivals)
  uint64_t* drain = bars + 19;    // the MMA issuer's last commit before teardown
  uint64_t* pv0_done = bars + 20; // [2] per query tile: PV on the first key half complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  float* qk_scale = reinterpret_cast<float*>(bars + 25);  // QK8: dequantisation of S

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = L_pad / TILE;
  const int qt0 = blockIdx.x * 2;
  const bool two = qt0 + 1 < n_qt;  // odd tile count: the last CTA has tile 0 only
  const int nt = two ? 2 : 1;
  const int qt1 = two ? qt0 + 1 : qt0;
  const int h = blockIdx.y;
  const int nkv = (L + TILE - 1) / TILE;
  const int row0 = h * L_pad;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[2 * s], 4);
      mbar_init(&p_full[2 * s + 1], 4);
      mbar_init(&pv0_done[s], 1);
      mbar_init(&o_final[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (QK8 && warp == 2) {
    // (sqrt(128) max|qn_w| / 448) (sqrt(128) max|kn_w| / 448)
    float mq = 0.f, mk = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mq = fmaxf(mq, fabsf(__bfloat162float(qn_w[lane * 4 + i])));
      mk = fmaxf(mk, fabsf(__bfloat162float(kn_w[lane * 4 + i])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
      mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
    }
    if (lane == 0) *qk_scale = ((11.3137085f * mq) / 448.0f) * ((11.3137085f * mk) / 448.0f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, nt * QK_TILE);
      for (int t = 0; t < nt; ++t) {
        const int qrow = row0 + (t == 0 ? qt0 : qt1) * TILE;
        tma_load_2d(sQ + t * QK_TILE, &tmQ, q_full, 0, qrow);
        if (!QK8) tma_load_2d(sQ + t * QK_TILE + HALF_BYTES, &tmQ, q_full, 64, qrow);
      }
      long long k_issued = 0, v_issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        uint8_t* dk = sK + st * QK_TILE;
        const int sv = j % VS;
        uint8_t* dv = sV + sv * TILE_BYTES;
        if (!mbar_wait(&k_empty[st], ((j >> 1) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(&k_full[st], QK_TILE);
        tma_load_2d(dk, &tmK, &k_full[st], 0, row0 + j * TILE);
        if (!QK8) tma_load_2d(dk + HALF_BYTES, &tmK, &k_full[st], 64, row0 + j * TILE);
        ++k_issued;
        if (!mbar_wait(&v_empty[sv], ((j / VS) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(&v_full[sv], TILE_BYTES);
        tma_load_2d(dv, &tmV, &v_full[sv], 0, row0 + j * TILE);
        tma_load_2d(dv + HALF_BYTES, &tmV, &v_full[sv], 64, row0 + j * TILE);
        ++v_issued;
      }
      // every load of this CTA has landed before it leaves
      mbar_wait(q_full, 0);
      drain_loads(k_full, 2, k_issued);
      drain_loads(v_full, VS, v_issued);
    }
  } else if (warp == 1) {
    // The whole warp runs the issue loop, converged; one elected lane issues.
    const uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
    const uint32_t idesc_s8 = idesc_e4m3_f32(128, 128);
    const uint32_t idesc_o = idesc_bf16_f32(128, 128, true);  // V is MN-major (d contiguous)
    // Shared-memory descriptors are computed once; an MMA then costs one
    // 64-bit add (the start-address field is bits [0,14) in 16-byte units,
    // and every offset below stays inside the 228 KB window).
    const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t k_desc = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t v_desc = sdesc_sw128(smem_u32(sV), HALF_BYTES, 1024);
    // S_t = Q_t K_j^T into TMEM columns [256t, 256t + 128)
    auto issue_s = [&](int t, int j) {
      const uint64_t qd = q_desc + (uint64_t)((t * QK_TILE) >> 4);
      const uint64_t kd = k_desc + (uint64_t)(((j & 1) * QK_TILE) >> 4);
      if constexpr (QK8) {
        // one 128-byte row per token: four MMAs of K = 32 codes (32 bytes)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_e4m3(tmem + t * 256, qd + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), idesc_s8, kk != 0 ? 1u : 0u);
      } else {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
          umma_bf16(tmem + t * 256, qd + off, kd + off, idesc_s, kk != 0 ? 1u : 0u);
        }
      }
      umma_commit(&s_full[t]);
    };
    // O_t += P_t V_j for keys [64 hf, 64 hf + 64): P_t (bf16, two per column)
    // read from TMEM columns [32 hf, 32 hf + 32) where S_t was
    auto issue_pv_half = [&](int t, int j, int hf) {
      const uint64_t vd = v_desc + (uint64_t)(((j % VS) * TILE_BYTES) >> 4);
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int kk = hf * 4 + k4;
        umma_bf16_tmem_a(tmem + t * 256 + 128, tmem + t * 256 + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_o,
                         (j | kk) != 0 ? 1u : 0u);
      }
    };
    bool ok = MMA_WAIT_WARP(q_full, 0) && MMA_WAIT_WARP(&k_full[0], 0);
    if (ok) {
      tc_fence_after();
      issue_s(0, 0);
      if (two) issue_s(1, 0);
      umma_commit(&k_empty[0]);
    }
    for (int j = 0; j < nkv && ok; ++j) {
      const bool more = j + 1 < nkv;
      // V(j) and K(j + 1) were requested a step or more ago: checked before
      // the wait for tile 0's P, off the P -> P V path (measured 1.6-2.6%
      // faster than waiting for each just before its MMAs)
      ok = MMA_WAIT_WARP(&v_full[j % VS], (j / VS) & 1) &&
           (!more || MMA_WAIT_WARP(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1));
      for (int t = 0; t < nt && ok; ++t) {
        // P is released in two halves: PV on keys [0, 64) runs while the
        // softmax warps still take the second half's exponentials
        for (int hf = 0; hf < 2; ++hf) {
          if (!MMA_WAIT_WARP(&p_full[2 * t + hf], j & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv_half(t, j, hf);
          if (hf == 0) umma_commit(&pv0_done[t]);
        }
        if (!ok) break;
        if (more) {
          issue_s(t, j + 1);
          if (t == nt - 1) umma_commit(&k_empty[(j + 1) & 1]);
        } else {
          umma_commit(&o_final[t]);
        }
      }
      umma_commit(&v_empty[j % VS]);
    }
    drain_mmas(drain);
  } else if ((warp - 2) >> 2 < nt) {
    const int t = (warp - 2) >> 2;  // query tile of this warpgroup
    // log2(e) / sqrt(128), times the dequantisation of e4m3 S.  A zero
    // dequantisation (an all-zero norm weight: every code of q or k is 0,
    // so S is 0) is raised to a tiny positive scale, so that masked keys
    // (-inf) still give -inf and not 0 * inf = NaN: the softmax is uniform.
    const float sl2 = QK8 ? fmaxf(scale_log2 * *qk_scale, 1e-30f) : scale_log2;
    const int qw = warp & 3;        // TMEM lane quarter this warp may access
    const int r = qw * 32 + lane;   // query row inside the tile
    const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 256;
    const uint32_t tO = tS + 128;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait_warp(&s_full[t], j & 1);
      if (!ok) break;
      tc_fence_after();
      float s[128];
      constexpr int kFirstLoad = H3_ATTN_S_HALVES ? 2 : 4;  // 32-column chunks loaded up front
#pragma unroll
      for (int c = 0; c < kFirstLoad; ++c) tmem_ld32(tS + c * 32, reinterpret_cast<uint32_t*>(s + c * 32));
      tmem_wait_ld();

      const int valid = L - j * TILE;  // keys [0, valid) of this tile are real
      if (valid < TILE) {
#pragma unroll
        for (int c = 0; c < 32 * kFirstLoad; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      // row max over keys [c0, c0 + n)
      auto row_max = [&](int c0, int n) {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = c0; c < c0 + n; c += 8) {
          m4[0] = max3f(m4[0], s[c], s[c + 1]);
          m4[1] = max3f(m4[1], s[c + 2], s[c + 3]);
          m4[2] = max3f(m4[2], s[c + 4], s[c + 5]);
          m4[3] = max3f(m4[3], s[c + 6], s[c + 7]);
        }
        return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      };
      // The reference m_ref is the row max of the first key tile, and moves
      // only when a later tile would overflow against it: the exponentials
      // of each 64-key half are taken against the current reference, and a
      // half whose row sum exceeds 2^16 (some p > 2^16) is redone against
      // that half's row max, with O and the sums rescaled first.  A half that
      // passed the check lies within 2^16 of the reference, so it stays in
      // range when the reference moves up.  No per-tile row max otherwise.
      // (with S in halves: the first half's max; the second half of the
      // first key tile then takes the overflow check like any later half)
      if (j == 0) m_ref = row_max(0, 32 * kFirstLoad) * sl2;
      const uint64_t sc2 = f2_pack(sl2, sl2);
      // p = 2^(s * sl2 - m_ref); returns this row's sum over the half.  The
      // last key tile (masked keys at -inf, which give exactly 0) takes every
      // exponential on the MUFU unit; the others take H3_ATTN_POLY_COLS of
      // every 16 on the FMA pipe.
      auto exp_half = [&](int hf, uint32_t* pk, auto poly_tag) {
        constexpr int kPolyCols = decltype(poly_tag)::value;  // of every 16 columns
        const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
        const float pa = sl2 * (1.0f / 252.0f), pb = (125.0f - m_ref) * (1.0f / 252.0f);
        uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const int cc = hf * 64 + c;
          uint64_t p2;
          if (kPolyCols > 0 && (c & 15) < kPolyCols) {
            p2 = exp2_fma2(s[cc], s[cc + 1], pa, pb);
          } else {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s[cc], s[cc + 1]), sc2, nm2), x0, x1);
            p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          float p0, p1;
          f2_unpack(p2, p0, p1);
          acc[(c >> 1) & 1] = f2_add(acc[(c >> 1) & 1], p2);
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        float a0, a1, a2, a3;
        f2_unpack(acc[0], a0, a1);
        f2_unpack(acc[1], a2, a3);
        return (a0 + a1) + (a2 + a3);
      };
      using NoPoly = std::integral_constant<int, 0>;
      auto exp_half_sel = [&](int hf, uint32_t* pk) {
        if (valid < TILE) return exp_half(hf, pk, NoPoly{});
        return exp_half(hf, pk, std::integral_constant<int, H3_ATTN_POLY_COLS>{});
      };
      float hsum[2];
      // P for keys [64 hf, 64 hf + 64) goes to TMEM columns [32 hf, 32 hf + 32)
      // (it only overwrites S columns already in registers)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[32];
        if (H3_ATTN_S_HALVES && hf == 1) {
          // the second half's scores, loaded while P of the first half was stored
          tmem_wait_ld();
          if (valid < TILE) {
#pragma unroll
            for (int c = 64; c < 128; ++c)
              if (c >= valid) s[c] = -INFINITY;
          }
        }
        float hs = exp_half_sel(hf, pk);
        if ((j > 0 || (H3_ATTN_S_HALVES && hf == 1)) && __any_sync(0xffffffffu, !(hs <= P_HALF_SUM_LIMIT))) {
          // this half's scores again, from TMEM: P has not overwritten them
          // (P of keys [0, 64) goes to columns [0, 32))
          tmem_ld32(tS + hf * 64, reinterpret_cast<uint32_t*>(s + hf * 64));
          tmem_ld32(tS + hf * 64 + 32, reinterpret_cast<uint32_t*>(s + hf * 64 + 32));
          tmem_wait_ld();
          if (valid < TILE) {
#pragma unroll
            for (int c = hf * 64; c < hf * 64 + 64; ++c)
              if (c >= valid) s[c] = -INFINITY;
          }
          const float m_new = fmaxf(m_ref, row_max(hf * 64, 64) * sl2);
          const float a = ex2_approx(m_ref - m_new);  // 1 where the reference holds
          m_ref = m_new;
          // O must hold every PV issued against the old reference before it
          // is rescaled: PV_t,j-1 completed before S_t,j was signalled; the
          // first half of PV_t,j has its own barrier
          if (hf == 1) {
            if (!__all_sync(0xffffffffu, mbar_wait(&pv0_done[t], j & 1))) { ok = false; break; }
            tc_fence_after();
            hsum[0] *= a;
          }
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            uint32_t o[8];
            tmem_ld8(tO + c * 8, o);
            tmem_wait_ld();
#pragma unroll
            for (int d = 0; d < 8; ++d) o[d] = __float_as_uint(__uint_as_float(o[d]) * a);
            tmem_st8(tO + c * 8, o);
          }
          tmem_wait_st();
          l_sum *= a;
          hs = exp_half_sel(hf, pk);
        }
        hsum[hf] = hs;
        if (H3_ATTN_S_HALVES && hf == 0) {
          // load the second half's scores (columns [64, 128), which no P
          // store touches) while this half's P is stored
          tmem_ld32(tS + 64, reinterpret_cast<uint32_t*>(s + 64));
          tmem_ld32(tS + 96, reinterpret_cast<uint32_t*>(s + 96));
        }
        tmem_st32(tS + hf * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[2 * t + hf]);
      }
      if (!ok) break;
      l_sum += hsum[0] + hsum[1];
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_final[t], 0));
    const int qt = t == 0 ? qt0 : qt1;
    if (ok) {
      tc_fence_after();
      const int grow = qt * TILE + r;
      const float inv = (grow < L) ? 1.0f / l_sum : 0.0f;
      const int owner = grow / out.L_shard;
      bf16* dst = out.shard[owner] + (long)(grow - owner * out.L_shard) * out.ld + (out.head0 + h) * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tO + c * 32, reinterpret_cast<uint32_t*>(o));
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
bool make_tmap_e4m3(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                    uint32_t box_rows);

// attention_split.cu: the split-softmax kernel on q, k normalised as the QKV
// call writes them
cudaError_t launch_attention_split(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                   const attn_detail::AttnOut& out, dim3 grid, int H, int L, int L_pad,
                                   float scale_log2, const bf16* qn_w, const bf16* kn_w, bool qk8,
                                   const attn_detail::AttnRope* rope, cudaStream_t stream);

cudaError_t launch_attention(const AttnProblem& p, cudaStream_t stream) {
  const bool qk8 = p.qk8 != 0;
  if (qk8 && (p.qn_w == nullptr || p.kn_w == nullptr)) return cudaErrorInvalidValue;
  static unsigned long long attr_done[2] = {0, 0};
  const void* kfn = qk8 ? reinterpret_cast<const void*>(attention_tc_kernel<true>)
                        : reinterpret_cast<const void*>(attention_tc_kernel<false>);
  cudaError_t aerr = ensure_smem_attr(kfn, qk8 ? Layout<true>::BYTES : Layout<false>::BYTES, &attr_done[qk8 ? 1 : 0]);
  if (aerr != cudaSuccess) return aerr;
  CUtensorMap tq, tk, tv;
  const uint64_t rows = (uint64_t)p.H * p.L_pad;
  if (qk8) {
    if (!make_tmap_e4m3(&tq, p.q, rows, 128, 128, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_e4m3(&tk, p.k, rows, 128, 128, 128)) return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_bf16(&tq, p.q, rows, 128, 128, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&tk, p.k, rows, 128, 128, 128)) return cudaErrorInvalidValue;
  }
  if (!make_tmap_bf16(&tv, p.v, rows, 128, 128, 128)) return cudaErrorInvalidValue;
  const int n_qt = p.L_pad / attn_detail::TILE;
  AttnOut out;
  memset(&out, 0, sizeof(out));
  if (p.sp_n > 0) {
    if (p.sp_n > 8 || p.sp_L_shard <= 0 || (long)p.sp_n * p.sp_L_shard < p.L_pad) return cudaErrorInvalidValue;
    out.ld = p.sp_ld;
    out.head0 = p.sp_head0;
    out.L_shard = p.sp_L_shard;
    for (int i = 0; i < p.sp_n; ++i) out.shard[i] = p.sp_o[i];
  } else {
    out.ld = (long)p.H * 128;
    out.head0 = 0;
    out.L_shard = p.L_pad;
    out.shard[0] = p.o;
  }
  dim3 grid((n_qt + 1) / 2, p.H);
#ifndef H3_ATTN_SPLIT
#define H3_ATTN_SPLIT 1
#endif
  if (p.prologue) {
    // raw q, k: the split kernel normalises and rotates them in its
    // prologue.  No recomputing launch follows (the general kernel takes q, k
    // as given): a CTA whose static bound fails leaves its sentinel and code
    // 2 in the device error word.
    if (qk8 || p.qn_w == nullptr || p.kn_w == nullptr || p.pos == nullptr) return cudaErrorInvalidValue;
    attn_detail::AttnRope rope{p.pos, p.rope_t, p.rope_h, p.rope_w, p.theta, p.eps_qk};
    return launch_attention_split(tq, tk, tv, out, grid, p.H, p.L, p.L_pad, p.scale_log2, p.qn_w, p.kn_w, false,
                                  &rope, stream);
  }
  if (H3_ATTN_SPLIT && p.qn_w != nullptr && p.kn_w != nullptr) {
    // the split-softmax kernel on normalised q, k (bf16 or e4m3 codes); then
    // this kernel on the CTAs it left (usually none: each such CTA returns
    // at once)
    aerr = launch_attention_split(tq, tk, tv, out, grid, p.H, p.L, p.L_pad, p.scale_log2, p.qn_w, p.kn_w, qk8,
                                  nullptr, stream);
    if (aerr != cudaSuccess) return aerr;
    if (qk8)
      attention_tc_kernel<true><<<grid, attn_detail::NUM_THREADS, Layout<true>::BYTES, stream>>>(
          tq, tk, tv, out, p.H, p.L, p.L_pad, p.scale_log2, p.qn_w, p.kn_w, 1);
    else
      attention_tc_kernel<false><<<grid, attn_detail::NUM_THREADS, Layout<false>::BYTES, stream>>>(
          tq, tk, tv, out, p.H, p.L, p.L_pad, p.scale_log2, nullptr, nullptr, 1);
    return cudaGetLastError();
  }
  if (qk8) {
    attention_tc_kernel<true><<<grid, attn_detail::NUM_THREADS, Layout<true>::BYTES, stream>>>(
        tq, tk, tv, out, p.H, p.L, p.L_pad, p.scale_log2, p.qn_w, p.kn_w, 0);
    return cudaGetLastError();
  }
  attention_tc_kernel<false><<<grid, attn_detail::NUM_THREADS, Layout<false>::BYTES, stream>>>(
      tq, tk, tv, out, p.H, p.L, p.L_pad, p.scale_log2, nullptr, nullptr, 0);
  return cudaGetLastError();
}

}  // namespace h3

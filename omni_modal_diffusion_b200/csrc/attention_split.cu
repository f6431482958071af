// Non-causal flash attention with each query row's exponentials split over
// two warps ("MiniMax-H3: native joint audio-video generation"
// (note.shouss.top) §5: full attention over the packed sequence).
//
// Same work split as attention_tc_kernel (one CTA per pair of 128-query
// tiles of one head, S and O in TMEM, P written back over S as bf16, the MMA
// warp issuing P V and the next S of one tile while the other tile's softmax
// runs), but each (query tile, TMEM lane quarter) has two softmax warps, one
// per 64-key half of the key tile.  The two warps of a quarter share one
// sub-partition and its MUFU unit: while one waits on its exponentials or on
// TMEM the other issues, so a tile's softmax phase approaches the MUFU time
// of its 16,384 exponentials instead of one warp's latency chain.
//
//   Warp 0       TMA producer (Q tiles once, K/V through 2-stage rings)
//   Warp 1       TMEM owner and MMA issuer
//   Warps 2-17   softmax: tile t = (w - 2) / 8, key half hf = ((w - 2) / 4) % 2,
//                lane quarter w % 4 (the quarter a warp may access in TMEM)
//   Warps 18-21  PRO only: RMSNorm + RoPE of the raw Q tiles and of each K
//                tile in shared memory, one row per thread
//
// The MMA warp holds one wait on each tile's path from P to P V: the tile's
// eight softmax warps arrive on one barrier, and the waits for V(j) and
// K(j + 1), loaded a step or more earlier, come before the wait for tile 0's
// P.  Every extra wait there showed in the time (a barrier per key half,
// the V and K waits between the P V and S MMAs: 3% slower; a barrier per
// 32-key chunk: 25% slower).
//
// The two halves of a row cannot move a softmax reference independently (O
// accumulates both halves' P V against one reference), and agreeing on it
// every key tile would put a handshake on each tile's critical path.  So
// this kernel takes no running maximum at all: q and k as the QKV call
// writes them are RMS-normalised rows scaled by the norm weights qn_w, kn_w,
// so ||q|| <= sqrt(128) max|qn_w|, ||k|| <= sqrt(128) max|kn_w| (bf16
// rounding adds at most 2^-8 to the product), and every score in log2 units
// is within B = 16.32 max|qn_w| max|kn_w| (1.01 margin) of 0.  Each p is taken
// as 2^(x - B) <= 1: no overflow, and with B <= 60 no p falls below 2^-120,
// so nothing flushes.  A CTA whose scores break the bound (a key-half sum
// above 2^32: q, k not normalised as stated) or whose norm weights give
// B > 60 leaves a NaN sentinel in its first output element instead of its
// rows, and a second launch of attention_tc_kernel recomputes exactly those
// CTAs with its moving reference.
//
// QK8: Q and K arrive as e4m3 codes of q * 448 / (sqrt(128) max|qn_w|) and
// k * 448 / (sqrt(128) max|kn_w|) (the QKV epilogue's H3_QK_E4M3 output); S
// is four kind::f8f6f4 MMAs per tile and its dequantisation folds into the
// exponent scale.  Rounding q and k to e4m3 (3 mantissa bits) moves each
// element by at most 2^-4 of itself, so the bound takes the factor
// (1 + 2^-4)^2 = 1.129: B = 16.32 * 1.14 max|qn_w| max|kn_w|.
//
// PRO: the alternative placement of the per-head Q/K RMSNorm + RoPE, in this
// kernel's prologue instead of the QKV epilogue (raw q, k in).  It redoes
// the normalisation and rotation of every key row for every CTA of its head
// and measures 2.4-2.7x slower per call; the library's default placement is
// the QKV epilogue.
#include "h3_internal.cuh"
#include "ptx.cuh"

namespace h3 {

namespace attn_split {
using attn_detail::AttnOut;
using attn_detail::HALF_BYTES;
using attn_detail::TILE;
using attn_detail::TILE_BYTES;
using attn_detail::TMEM_COLS;

constexpr int SVS = 2;  // V stages
// PRO: q and k arrive raw (as the QKV GEMM leaves them) and the kernel takes
// their per-head RMSNorm and 3-D RoPE in its prologue: four more warps
// normalise and rotate each Q tile once and each K tile as it lands in
// shared memory, before the MMA warp may read it.
// e4m3 Q K^T: 2 of every 16 exponentials on the FMA pipe.  Measured per call
// (TFLOP/s at 7,904 tokens / 124,016 tokens with 8 heads): 1,399 / 1,387 all
// on MUFU; 1,504 / 1,446 with 2; 1,503 / 1,427 with 4; 1,495 / 1,418 with 6.
// The bf16 kernel measured slower with any share (its tensor pipe, not
// MUFU, is the busier unit), so it takes none.
#ifndef H3_ATTN_SPLIT_QK8_POLY
#define H3_ATTN_SPLIT_QK8_POLY 2
#endif
static_assert(H3_ATTN_SPLIT_QK8_POLY >= 0 && H3_ATTN_SPLIT_QK8_POLY <= 16 && H3_ATTN_SPLIT_QK8_POLY % 2 == 0,
              "H3_ATTN_SPLIT_QK8_POLY: an even count of 0..16");
template <bool QK8, bool PRO = false>
struct SLayout {
  static_assert(!(QK8 && PRO), "the prologue takes bf16 q, k");
  static constexpr int WARPS = PRO ? 22 : 18;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int QK_TILE = QK8 ? TILE_BYTES / 2 : TILE_BYTES;  // a Q or K tile (e4m3: 128-byte rows)
  static constexpr int SQ = 0;                                        // 2 query tiles
  static constexpr int SK = SQ + 2 * QK_TILE;                         // 2 stages
  static constexpr int SV = SK + 2 * QK_TILE;                         // SVS stages
  static constexpr int SBAR = SV + SVS * TILE_BYTES;
  // PRO: rotation frequency and axis of each of the 64 pairs, the two norm
  // weights as fp32
  static constexpr int SMISC = SBAR + 256;
  static constexpr int BYTES = SMISC + (PRO ? 1536 : 0) + 1024;
  // [2 tiles][2 halves][128 rows] row sums (2 KB), written after a warp's key
  // loop: over the K stage that held K(nkv - 2), whose last S MMA completed
  // before any tile's last S (the other stage may still feed the other
  // tile's last S)
  static constexpr int SSUM = SK;
  static_assert(BYTES <= 232448, "shared memory per CTA");
  static_assert(QK_TILE >= 2 * 2 * 128 * 4, "row sums fit in a K stage");
};
constexpr float B_MAX = 60.0f;              // largest bound whose p stay >= 2^-120
constexpr float HALF_SUM_LIMIT = 4294967296.0f;  // 2^32: a key half above it breaks the bound

// 32 lanes x 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Where the first output element of the CTA's first query tile lives.
__device__ __forceinline__ bf16* sentinel_ptr(const AttnOut& out, int grow, int h) {
  const int owner = grow / out.L_shard;
  return out.shard[owner] + (long)(grow - owner * out.L_shard) * out.ld + (out.head0 + h) * 128;
}

template <bool QK8, bool PRO>
__global__ void __launch_bounds__(SLayout<QK8, PRO>::THREADS, 1)
    attention_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnOut out, int H,
                           int L, int L_pad, float scale_log2, const bf16* qn_w, const bf16* kn_w,
                           const __grid_constant__ attn_detail::AttnRope rope) {
  using Y = SLayout<QK8, PRO>;
  constexpr int SQ = Y::SQ, SK = Y::SK, SV = Y::SV, SBAR = Y::SBAR, SSUM = Y::SSUM, QK_TILE = Y::QK_TILE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem + SQ;
  uint8_t* sK = smem + SK;
  uint8_t* sV = smem + SV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SBAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;    // [SVS]
  uint64_t* v_empty = bars + 8;   // [SVS]
  uint64_t* s_full = bars + 11;   // [2] per query tile
  uint64_t* o_final = bars + 13;  // [2] per query tile
  uint64_t* p_full = bars + 15;   // [2] per query tile: its 8 softmax warps' arrivals
  uint64_t* drain = bars + 17;
  uint64_t* sums_done = bars + 18;  // [2] every softmax warp has written its row sums / its low-side verdict
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  float* bound = reinterpret_cast<float*>(bars + 21);
  int* cta_bad = reinterpret_cast<int*>(bars + 22);
  float* qk_scale = reinterpret_cast<float*>(bars + 23);  // QK8: dequantisation of S
  uint64_t* q_ready = bars + 24;  // PRO: both Q tiles normalised and rotated (4 prologue warps)
  uint64_t* k_ready = bars + 25;  // PRO: [2] the K stage normalised and rotated (4 prologue warps)
  float* pro_freq = reinterpret_cast<float*>(smem + Y::SMISC);  // PRO: [64]
  float* pro_qw = pro_freq + 64;                                 // PRO: [128] qn_w
  float* pro_kw = pro_qw + 128;                                  // PRO: [128] kn_w
  uint8_t* pro_axis = reinterpret_cast<uint8_t*>(pro_kw + 128);  // PRO: [64]
  float* lsum = reinterpret_cast<float*>(smem + SSUM + (((L + TILE - 1) / TILE) & 1) * QK_TILE);  // [t][hf][row]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = L_pad / TILE;
  const int qt0 = blockIdx.x * 2;
  const bool two = qt0 + 1 < n_qt;
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
      mbar_init(&o_final[s], 1);
      mbar_init(&p_full[s], 8);
    }
    for (int s = 0; s < SVS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(drain, 1);
    if (PRO) {
      mbar_init(q_ready, 4);
      mbar_init(&k_ready[0], 4);
      mbar_init(&k_ready[1], 4);
    }
    mbar_init(&sums_done[0], 8 * nt);
    mbar_init(&sums_done[1], 8 * nt);
    *cta_bad = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) {
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
    // 128 mq mk (1 + 2^-9)^2 log2(e) / sqrt(128), with a 1% margin (QK8:
    // times the e4m3 factor 1.129, with a 1% margin)
    if (lane == 0) {
      *bound = 16.3219f * (QK8 ? 1.14f : 1.01f) * mq * mk;
      if (QK8) *qk_scale = ((11.3137085f * mq) / 448.0f) * ((11.3137085f * mk) / 448.0f);
    }
  }
  if (PRO && warp >= 18) {
    // the norm weights as fp32, and each pair's rotation: pair i of the
    // section of width d it falls in (t | h | w) turns by theta^(-2i/d) per
    // unit of that axis' position (the QKV epilogue's table)
    const int i = threadIdx.x - 18 * 32;  // 0 .. 127
    pro_qw[i] = __bfloat162float(qn_w[i]);
    pro_kw[i] = __bfloat162float(kn_w[i]);
    if (i < 64) {
      const int pt = rope.rope_t / 2, ph = rope.rope_h / 2;
      int ax, i_sec, d_sec;
      if (i < pt) { ax = 0; i_sec = i; d_sec = rope.rope_t; }
      else if (i < pt + ph) { ax = 1; i_sec = i - pt; d_sec = rope.rope_h; }
      else { ax = 2; i_sec = i - pt - ph; d_sec = rope.rope_w; }
      pro_freq[i] = powf(rope.theta, -2.0f * (float)i_sec / (float)d_sec);
      pro_axis[i] = (uint8_t)ax;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float B = *bound;
  const bool fast = B <= B_MAX;  // uniform across the CTA

  if (!fast) {
    // the bound is too wide for p to stay normal: leave the CTA to the
    // recomputing launch
    if (threadIdx.x == 0) {
      *sentinel_ptr(out, qt0 * TILE, h) = __ushort_as_bfloat16((unsigned short)0x7FC0);
      if (PRO) atomicCAS(&g_h3_device_error, 0, 2);  // no launch recomputes it
    }
  } else if (warp == 0) {
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
        if (!mbar_wait(&k_empty[st], ((j >> 1) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(&k_full[st], QK_TILE);
        tma_load_2d(sK + st * QK_TILE, &tmK, &k_full[st], 0, row0 + j * TILE);
        if (!QK8) tma_load_2d(sK + st * QK_TILE + HALF_BYTES, &tmK, &k_full[st], 64, row0 + j * TILE);
        ++k_issued;
        const int sv = j % SVS;
        if (!mbar_wait(&v_empty[sv], ((j / SVS) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(&v_full[sv], TILE_BYTES);
        tma_load_2d(sV + sv * TILE_BYTES, &tmV, &v_full[sv], 0, row0 + j * TILE);
        tma_load_2d(sV + sv * TILE_BYTES + HALF_BYTES, &tmV, &v_full[sv], 64, row0 + j * TILE);
        ++v_issued;
      }
      mbar_wait(q_full, 0);
      drain_loads(k_full, 2, k_issued);
      drain_loads(v_full, SVS, v_issued);
    }
  } else if (warp == 1) {
    const uint32_t idesc_s = QK8 ? idesc_e4m3_f32(128, 128) : idesc_bf16_f32(128, 128, false);
    const uint32_t idesc_o = idesc_bf16_f32(128, 128, true);  // V is MN-major
    const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t k_desc = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t v_desc = sdesc_sw128(smem_u32(sV), HALF_BYTES, 1024);
    auto issue_s = [&](int t, int j) {
      const uint64_t qd = q_desc + (uint64_t)((t * QK_TILE) >> 4);
      const uint64_t kd = k_desc + (uint64_t)(((j & 1) * QK_TILE) >> 4);
      if constexpr (QK8) {
        // one 128-byte row per token: four MMAs of K = 32 codes (32 bytes)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_e4m3(tmem + t * 256, qd + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), idesc_s, kk != 0 ? 1u : 0u);
      } else {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
          umma_bf16(tmem + t * 256, qd + off, kd + off, idesc_s, kk != 0 ? 1u : 0u);
        }
      }
      umma_commit(&s_full[t]);
    };
    // O_t += P_t V_j: the P of keys [64 hf, 64 hf + 64) sits in TMEM columns
    // [64 hf, 64 hf + 32) of the tile's S region (written by that half's warps)
    auto issue_pv = [&](int t, int j) {
      const uint64_t vd = v_desc + (uint64_t)(((j % SVS) * TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_bf16_tmem_a(tmem + t * 256 + 128, tmem + t * 256 + (kk >> 2) * 64 + (kk & 3) * 8,
                         vd + (uint64_t)((kk * 2048) >> 4), idesc_o, (j | kk) != 0 ? 1u : 0u);
    };
    // PRO: Q and each K stage are read once the prologue warps have
    // normalised and rotated them
    uint64_t* q_in = PRO ? q_ready : q_full;
    uint64_t* k_in = PRO ? k_ready : k_full;
    bool ok = mbar_wait_warp(q_in, 0) && mbar_wait_warp(&k_in[0], 0);
    if (ok) {
      tc_fence_after();
      issue_s(0, 0);
      if (two) issue_s(1, 0);
      umma_commit(&k_empty[0]);
    }
    for (int j = 0; j < nkv && ok; ++j) {
      const bool more = j + 1 < nkv;
      // V(j) and K(j + 1) were requested a step or more ago: check them before
      // waiting for tile 0's P, so that each tile's P -> P V path holds one
      // wait (measured 3% faster than waiting for each just before its MMAs)
      ok = mbar_wait_warp(&v_full[j % SVS], (j / SVS) & 1) &&
           (!more || mbar_wait_warp(&k_in[(j + 1) & 1], ((j + 1) >> 1) & 1));
      for (int t = 0; t < nt && ok; ++t) {
        if (!mbar_wait_warp(&p_full[t], j & 1)) { ok = false; break; }
        tc_fence_after();
        issue_pv(t, j);
        if (more) {
          issue_s(t, j + 1);
          if (t == nt - 1) umma_commit(&k_empty[(j + 1) & 1]);
        } else {
          umma_commit(&o_final[t]);
        }
      }
      umma_commit(&v_empty[j % SVS]);
    }
    drain_mmas(drain);
  } else if (PRO && warp >= 18) {
    // One row per thread: RMSNorm (fp32, weights and eps of the QKV
    // epilogue) then RoPE of row r of both Q tiles once, and of row r of
    // every K tile as it lands; the row is read from and written back to its
    // 128-byte-swizzled place (16-byte chunk c of row r at c ^ (r % 8)).
    const int r = (warp - 18) * 32 + lane;
    auto prep_row = [&](uint8_t* tile, int grow, const float* w) {
      uint8_t* rowp = tile + r * 128;
      const int sw = r & 7;
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(rowp + (c >> 3) * HALF_BYTES + (((c & 7) ^ sw) << 4));
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b2[e]);
          ss = fmaf(f.x, f.x, ss);
          ss = fmaf(f.y, f.y, ss);
        }
      }
      const float inv = rsqrtf(ss * (1.0f / 128.0f) + rope.eps);
      float p3[3] = {0.f, 0.f, 0.f};
      if (grow < L_pad) {
        p3[0] = rope.pos[(long)grow * 3 + 0];
        p3[1] = rope.pos[(long)grow * 3 + 1];
        p3[2] = rope.pos[(long)grow * 3 + 2];
      }
#pragma unroll 2
      for (int c = 0; c < 16; ++c) {
        uint4* addr = reinterpret_cast<uint4*>(rowp + (c >> 3) * HALF_BYTES + (((c & 7) ^ sw) << 4));
        uint4 u = *addr;
        __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int d = c * 8 + e * 2;  // the pair (d, d + 1), pair index d / 2
          const float2 f = __bfloat1622float2(b2[e]);
          const float a = f.x * inv * w[d], bb = f.y * inv * w[d + 1];
          const int ax = pro_axis[d >> 1];
          const float pa = ax == 0 ? p3[0] : (ax == 1 ? p3[1] : p3[2]);
          float sn, cs;
          rope_sincos(pa * pro_freq[d >> 1], &sn, &cs);
          b2[e] = __floats2bfloat162_rn(a * cs - bb * sn, a * sn + bb * cs);
        }
        *addr = u;
      }
    };
    bool ok = mbar_wait_warp(q_full, 0);
    if (ok) {
      for (int t = 0; t < nt; ++t) prep_row(sQ + t * QK_TILE, (t == 0 ? qt0 : qt1) * TILE + r, pro_qw);
      fence_proxy_async_smem();  // the MMAs read these rows through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    for (int j = 0; j < nkv && ok; ++j) {
      const int st = j & 1;
      if (!mbar_wait_warp(&k_full[st], (j >> 1) & 1)) break;
      prep_row(sK + st * QK_TILE, j * TILE + r, pro_kw);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&k_ready[st]);
    }
  } else if (((warp - 2) >> 3) < nt) {
    const int t = (warp - 2) >> 3;         // query tile
    const int hf = ((warp - 2) >> 2) & 1;  // key half of every key tile
    const int qw = warp & 3;               // TMEM lane quarter
    const int r = qw * 32 + lane;          // query row inside the tile
    const uint32_t tS = tmem + ((uint32_t)(qw * 32) << 16) + t * 256;
    const uint32_t tH = tS + hf * 64;      // this warp's 64 score columns; its P goes to the first 32
    const uint32_t tO = tS + 128;
    // QK8: the dequantisation of S folds into the scale; an all-zero norm
    // weight (every code 0, S = 0) is raised to a tiny positive scale so
    // masked keys (-inf) still give 0 and not 0 * inf = NaN
    const float sl2 = QK8 ? fmaxf(scale_log2 * *qk_scale, 1e-30f) : scale_log2;
    const uint64_t sc2 = f2_pack(sl2, sl2);
    const uint64_t nb2 = f2_pack(-B, -B);
    float l_part = 0.f;
    bool bad = false;
    bool ok = true;
    // p = 2^(s scale_log2 - B) for 32 scores; their bf16 pairs into pk[16];
    // returns their sum (masked keys, -inf, give 0)
    // QK8 with H3_ATTN_SPLIT_QK8_POLY: that many of every 16 exponentials on
    // the FMA pipe (exp2_fma2), where the e4m3 S leaves the tensor pipe slack
    // and the MUFU unit is the busier one; never on the last key tile (its
    // masked keys must give exactly 0)
    constexpr int kPoly = QK8 ? H3_ATTN_SPLIT_QK8_POLY : 0;
    const float pa = sl2 * (1.0f / 252.0f), pb = (125.0f - B) * (1.0f / 252.0f);
    (void)pa;
    (void)pb;
    auto exp32 = [&](const float* s, uint32_t* pk, auto poly_tag) {
      constexpr int kP = decltype(poly_tag)::value;
      uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float p0, p1;
        if (kP > 0 && (c & 15) < kP) {
          f2_unpack(exp2_fma2(s[c], s[c + 1], pa, pb), p0, p1);
        } else {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sc2, nb2), x0, x1);
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        acc[(c >> 1) & 1] = f2_add(acc[(c >> 1) & 1], f2_pack(p0, p1));
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      float a0, a1, a2, a3;
      f2_unpack(acc[0], a0, a1);
      f2_unpack(acc[1], a2, a3);
      return (a0 + a1) + (a2 + a3);
    };
    using NoPoly = std::integral_constant<int, 0>;
    using Poly = std::integral_constant<int, kPoly>;
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait_warp(&s_full[t], j & 1);
      if (!ok) break;
      tc_fence_after();
      const int valid = L - j * TILE - hf * 64;  // this half's keys [0, valid) are real
      float s[32];
      uint32_t pkA[16], pkB[16];
      tmem_ld32(tH, reinterpret_cast<uint32_t*>(s));
      tmem_wait_ld();
      if (valid < 32) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float hs;
      if constexpr (kPoly == 0)
        hs = exp32(s, pkA, NoPoly{});
      else
        hs = valid < 64 ? exp32(s, pkA, NoPoly{}) : exp32(s, pkA, Poly{});
      // P of keys [0, 32) of the half over its own first 16 score columns
      tmem_st16(tH, pkA);
      tmem_ld32(tH + 32, reinterpret_cast<uint32_t*>(s));
      tmem_wait_ld();
      if (valid < 64) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c + 32 >= valid) s[c] = -INFINITY;
      }
      if constexpr (kPoly == 0)
        hs += exp32(s, pkB, NoPoly{});
      else
        hs += valid < 64 ? exp32(s, pkB, NoPoly{}) : exp32(s, pkB, Poly{});
      // P of keys [32, 64) of the half over score columns [16, 32), already read
      tmem_st16(tH + 16, pkB);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
      bad |= !(hs <= HALF_SUM_LIMIT);
      l_part += hs;
    }
    // The CTA's verdict on the bound, in two rounds so that every warp
    // decides before any writes: (1) a key half summed past 2^32 (a score
    // far above the bound) and the half sums; (2) a row whose whole sum fell
    // below 2^-110 (every score far below the bound: p would flush)
    const int qt = t == 0 ? qt0 : qt1;
    const int grow = qt * TILE + r;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(cta_bad, 1);
    lsum[(t * 2 + hf) * 128 + r] = l_part;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sums_done[0]);
    ok = mbar_wait_warp(&sums_done[0], 0) && ok;
    const float l = lsum[(t * 2) * 128 + r] + lsum[(t * 2 + 1) * 128 + r];
    if (__any_sync(0xffffffffu, grow < L && !(l >= 7.7e-34f)) && lane == 0) atomicOr(cta_bad, 1);  // 2^-110
    __syncwarp();
    if (lane == 0) mbar_arrive(&sums_done[1]);
    if (ok) ok = mbar_wait_warp(&sums_done[1], 0) && mbar_wait_warp(&o_final[t], 0);
    if (ok) {
      tc_fence_after();
      const bool redo = *reinterpret_cast<volatile int*>(cta_bad) != 0;
      if (redo) {
        if (t == 0 && hf == 0 && r == 0) {
          *sentinel_ptr(out, grow, h) = __ushort_as_bfloat16((unsigned short)0x7FC0);
          if (PRO) atomicCAS(&g_h3_device_error, 0, 2);  // no launch recomputes it
        }
      } else {
        const float inv = (grow < L) ? 1.0f / l : 0.0f;
        bf16* dst = sentinel_ptr(out, grow, h);
        // this warp writes O columns [64 hf, 64 hf + 64) of its row
#pragma unroll 1
        for (int c = 2 * hf; c < 2 * hf + 2; ++c) {
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace attn_split

cudaError_t launch_attention_split(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                   const attn_detail::AttnOut& out, dim3 grid, int H, int L, int L_pad,
                                   float scale_log2, const bf16* qn_w, const bf16* kn_w, bool qk8,
                                   const attn_detail::AttnRope* rope, cudaStream_t stream) {
  using namespace attn_split;
  static unsigned long long attr_done[3] = {0, 0, 0};
  const attn_detail::AttnRope r = rope ? *rope : attn_detail::AttnRope{nullptr, 0, 0, 0, 0.f, 0.f};
  const int which = rope ? 2 : (qk8 ? 1 : 0);
  const void* kfn = which == 2 ? reinterpret_cast<const void*>(attention_split_kernel<false, true>)
                    : which == 1 ? reinterpret_cast<const void*>(attention_split_kernel<true, false>)
                                 : reinterpret_cast<const void*>(attention_split_kernel<false, false>);
  const int bytes = which == 2 ? SLayout<false, true>::BYTES
                    : which == 1 ? SLayout<true, false>::BYTES
                                 : SLayout<false, false>::BYTES;
  cudaError_t e = ensure_smem_attr(kfn, bytes, &attr_done[which]);
  if (e != cudaSuccess) return e;
  if (which == 2)
    attention_split_kernel<false, true><<<grid, SLayout<false, true>::THREADS, bytes, stream>>>(
        tq, tk, tv, out, H, L, L_pad, scale_log2, qn_w, kn_w, r);
  else if (which == 1)
    attention_split_kernel<true, false><<<grid, SLayout<true, false>::THREADS, bytes, stream>>>(
        tq, tk, tv, out, H, L, L_pad, scale_log2, qn_w, kn_w, r);
  else
    attention_split_kernel<false, false><<<grid, SLayout<false, false>::THREADS, bytes, stream>>>(
        tq, tk, tv, out, H, L, L_pad, scale_log2, qn_w, kn_w, r);
  return cudaGetLastError();
}

}  // namespace h3

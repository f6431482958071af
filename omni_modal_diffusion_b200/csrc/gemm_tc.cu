// Persistent tcgen05 GEMM, out = A[M,K] * B[N,K]^T (bf16 in, fp32 accumulate
// in TMEM), with the block's fused epilogues:
//   - input projections into the fp32 residual stream,
//   - modality-gated residual add (attention out-projection, FFN down),
//   - SiLU(gate) * up (FFN gate/up),
//   - per-head Q/K RMSNorm + 3-D RoPE with a head-major scatter (QKV),
//   - the video head's inverse patchify gather.
// Block structure per "MiniMax-H3: native joint audio-video generation"
// (note.shouss.top) §3 and §3.2; patch layout per "MiniMax-H3 paper reading"
// (gojay.top) §7.3.
//
// CTA = 6 warps.  Warp 0: TMA producer (one thread).  Warp 1: TMEM owner and
// MMA issuer (one thread).  Warps 2-5: epilogue, one accumulator row per
// thread (warp w may read TMEM lanes 32*(w%4) .. +31).  Tiles are 128 x 256
// with a 64-deep K step, 4 shared-memory stages (48 KB each) and two TMEM
// accumulators (2 x 256 columns) so the epilogue of one tile overlaps the
// MMAs of the next.
#include "h3_internal.cuh"
#include "ptx.cuh"

namespace h3 {

#ifndef H3_GEMM_HALF_N
#define H3_GEMM_HALF_N 1
#endif

namespace gemm_detail {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_STAGE_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
// The fp32 store epilogue transposes each 32 x 32 chunk of a warp's rows
// through shared memory (pitch 36 words: 16-byte rows, conflict-free for the
// 8-lane phases of 16-byte accesses both ways) so that every global store
// instruction writes four rows' 128 contiguous bytes each.
constexpr int EPI_PITCH = 36;
constexpr int EPI_STAGE_BYTES = 4 * 32 * EPI_PITCH * 4;
// [1 KB alignment slack][stages][512 B barriers, TMEM slot, RoPE tables][epilogue staging]
constexpr int MISC_BYTES = 512;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + MISC_BYTES + EPI_STAGE_BYTES;

__device__ __forceinline__ int modality_of(int row, const GemmEpilogue& e) {
#pragma unroll
  for (int m = 0; m < 3; ++m)
    if (row >= e.rstart[m] && row < e.rstart[m] + e.rcount[m]) return m;
  return -1;
}

// Tile t -> (row tile, column tile): bands of `group` row tiles sweep every
// column tile before the next band starts, so the band's A rows stay in L2
// while B streams past.
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int group, int& mt, int& nt) {
  const int per_group = group * n_tiles;
  const int g = t / per_group;
  const int first = g * group;
  const int gm = min(group, m_tiles - first);
  const int local = t - g * per_group;
  mt = first + local % gm;
  nt = local / gm;
}

__device__ __forceinline__ void ld_chunk(uint32_t taddr, float* v) {
  tmem_ld32(taddr, reinterpret_cast<uint32_t*>(v));
}

// e4m3 operands: the 32 accumulator columns of a chunk (B rows b0 .. b0 + 31)
// times a_scale[m] * b_scale[b]; B rows past the end scale to 0.  No-op for
// bf16 operands.
__device__ __forceinline__ void scale_chunk(const GemmEpilogue& e, float* v, int m, int b0) {
  if (e.a_scale == nullptr) return;
  const float sa = (m < e.a_rows) ? e.a_scale[m] : 0.f;
  if (b0 + 32 <= e.b_rows) {  // b0 is a multiple of 32 and b_scale 16-byte aligned
    const float4* bs = reinterpret_cast<const float4*>(e.b_scale + b0);
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 b = __ldg(bs + j / 4);
      v[j] *= sa * b.x;
      v[j + 1] *= sa * b.y;
      v[j + 2] *= sa * b.z;
      v[j + 3] *= sa * b.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int b = b0 + j;
      v[j] *= sa * (b < e.b_rows ? __ldg(e.b_scale + b) : 0.f);
    }
  }
}

// ------------------------------------------------------------ epilogues
// stage: this warp's [32][EPI_PITCH] fp32 buffer; lane = row m - m0 of the
// warp's 32 consecutive rows.
__device__ __forceinline__ void epi_store_f32(const GemmEpilogue& e, uint32_t tb, int m, int n0, float* stage) {
  const int lane = threadIdx.x & 31;
  const int m0 = m - lane;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    const int nc = n0 + c * 32;
    if (nc >= e.N) break;  // uniform across the CTA
    float v[32];
    ld_chunk(tb + c * 32, v);
    tmem_wait_ld();
    scale_chunk(e, v, m, nc);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(stage + lane * EPI_PITCH + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    __syncwarp();
    // lane l: row 4 i + l / 8, columns 4 (l % 8) .. + 3 of the chunk
    const int sub = lane >> 3, col = nc + 4 * (lane & 7);
    float* out = static_cast<float*>(e.out);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 4 * i + sub;
      if (m0 + r >= e.M) continue;
      const float4 w = *reinterpret_cast<const float4*>(stage + r * EPI_PITCH + 4 * (lane & 7));
      const long off = (long)(e.row_off + m0 + r) * e.ldo + col;
      float* dst = out + off;
      if (e.euler) {
        // one Euler step of the latent in out: out += dsigma * velocity
        const float wv[4] = {w.x, w.y, w.z, w.w};
        for (int k = 0; k < 4 && col + k < e.N; ++k) {
          const float a = fmaf(e.dsigma, wv[k], dst[k]);
          dst[k] = a;
          if (e.out_bf16) e.out_bf16[off + k] = __float2bfloat16_rn(a);
        }
      } else if (col + 4 <= e.N) {
        *reinterpret_cast<float4*>(dst) = w;
      } else {
        const float wv[4] = {w.x, w.y, w.z, w.w};
        for (int k = 0; k < 4 && col + k < e.N; ++k) dst[k] = wv[k];
      }
    }
  }
}

// Chunks [c_lo, c_hi) of 32 accumulator columns (all BN / 32 by default).
__device__ __forceinline__ void epi_gated_resid(const GemmEpilogue& e, uint32_t tb, int m, int n0, int c_lo = 0,
                                                int c_hi = BN / 32) {
  const int row = e.row_off + m;
  const int mod_id = (m < e.M) ? modality_of(row, e) : -1;
  const float* gate = e.mod + (long)((mod_id < 0 ? 0 : mod_id) * 6 + e.gate_slot) * e.D;
  float* xrow = static_cast<float*>(e.out) + (long)row * e.ldo;
#pragma unroll 1
  for (int c = c_lo; c < c_hi; ++c) {
    const int nc = n0 + c * 32;
    if (nc >= e.N) break;
    float v[32];
    ld_chunk(tb + c * 32, v);
    tmem_wait_ld();
    scale_chunk(e, v, m, nc);
    if (mod_id >= 0) {
      if (nc + 32 <= e.N) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 x = *reinterpret_cast<const float4*>(xrow + nc + j);
          const float4 g = __ldg(reinterpret_cast<const float4*>(gate + nc + j));
          x.x = fmaf(g.x, v[j], x.x);
          x.y = fmaf(g.y, v[j + 1], x.y);
          x.z = fmaf(g.z, v[j + 2], x.z);
          x.w = fmaf(g.w, v[j + 3], x.w);
          *reinterpret_cast<float4*>(xrow + nc + j) = x;
        }
      } else {
        for (int j = 0; j < 32 && nc + j < e.N; ++j) xrow[nc + j] = fmaf(gate[nc + j], v[j], xrow[nc + j]);
      }
    }
  }
}

__device__ __forceinline__ void epi_swiglu(const GemmEpilogue& e, uint32_t tb, int m, int nt, int c_lo = 0,
                                           int c_hi = 4) {
  // columns [0,128) of the accumulator hold gate, [128,256) hold up, for
  // output columns nt*128 + [0,128); chunks [c_lo, c_hi) of 32 of them
  bf16* dst = static_cast<bf16*>(e.out) + (long)m * e.ldo + (long)nt * 128;
#pragma unroll 1
  for (int c = c_lo; c < c_hi; ++c) {
    float g[32], u[32];
    ld_chunk(tb + c * 32, g);
    ld_chunk(tb + 128 + c * 32, u);
    tmem_wait_ld();
    scale_chunk(e, g, m, nt * 128 + c * 32);
    scale_chunk(e, u, m, e.N + nt * 128 + c * 32);
    if (m < e.M) {
      uint32_t packed[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float h0 = g[j] / (1.0f + __expf(-g[j])) * u[j];
        const float h1 = g[j + 1] / (1.0f + __expf(-g[j + 1])) * u[j + 1];
        packed[j / 2] = pack_bf16x2(h0, h1);
      }
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<uint4*>(dst + c * 32 + j * 2) =
            make_uint4(packed[j], packed[j + 1], packed[j + 2], packed[j + 3]);
    }
  }
}

// One warp: the e4m3 code scales of q and k, 448 / (sqrt(128) max|w|) for
// the norm weights w = qn_w, kn_w (RMSNorm then RoPE bound every element of
// a head row by sqrt(128) max|w|, so no code saturates).
__device__ __forceinline__ void qk_e4m3_inv_scales(const GemmEpilogue& e, float* qk_inv) {
  const int lane = threadIdx.x & 31;
  float mq = 0.f, mk = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mq = fmaxf(mq, fabsf(__bfloat162float(e.qn_w[lane * 4 + i])));
    mk = fmaxf(mk, fabsf(__bfloat162float(e.kn_w[lane * 4 + i])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
    mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
  }
  // an all-zero norm weight makes every q (k) element 0: inverse scale 0
  // (codes 0, no 0 * inf), and attention's scale product is 0 as well
  if (lane == 0) {
    qk_inv[0] = mq > 0.f ? 448.0f / (11.3137085f * mq) : 0.f;
    qk_inv[1] = mk > 0.f ? 448.0f / (11.3137085f * mk) : 0.f;
  }
}

// sin and cos of a RoPE angle on the MUFU unit.  The angle is first reduced
// to [-pi, pi] with 2 pi split into its nearest fp32 value H = 6.28318548...
// and the remainder T = 2 pi - H = -1.7484556e-7 (two-term Cody-Waite
// reduction: r = (a - k H) - k T, each step one fused multiply-add), which
// keeps |r - (a - 2 pi k)| within a few fp32 ulps of r for the angles here
// (|a| < 10^4); __sincosf is then accurate to ~2^-21 on [-pi, pi].  The
// library's accurate sincosf took twice as long over the whole QKV GEMM with
// e4m3 operands (the epilogue, not the MMAs, bounded it).
__device__ __forceinline__ void rope_sincos(float a, float* s, float* c) {
  const float k = rintf(a * 0.159154937f);  // a / (2 pi)
  float r = fmaf(-k, 6.28318548f, a);
  r = fmaf(-k, -1.74845553e-7f, r);
  __sincosf(r, s, c);
}

// Heads [h_lo, h_hi) of the tile's two 128-column heads.  Two passes over
// TMEM per head: the sum of squares of the 128 values, then chunk by chunk
// normalise, rotate and store (no 128-value array in registers).
__device__ __forceinline__ void epi_qkv(const GemmEpilogue& e, uint32_t tb, int m, int n0, const float* freq,
                                        const uint8_t* axis_of_pair, const float* qk_inv, int h_lo = 0,
                                        int h_hi = 2) {
  float p3[3] = {0.f, 0.f, 0.f};
  if (m < e.L_pad && !e.qk_raw) {  // raw q, k: pos is not read (it may be null)
    p3[0] = e.pos[(long)m * 3 + 0];
    p3[1] = e.pos[(long)m * 3 + 1];
    p3[2] = e.pos[(long)m * 3 + 2];
  }
#pragma unroll 1
  for (int half = h_lo; half < h_hi; ++half) {
    const int n = n0 + half * 128;
    if (n >= e.N) break;  // uniform
    const int part = n / e.I;
    const int h = (n % e.I) / 128;
    const uint32_t th = tb + half * 128;
    float inv = 1.0f;
    const bf16* w = part == 0 ? e.qn_w : e.kn_w;
    const bool norm_rope = part < 2 && !e.qk_raw;
    if (norm_rope) {
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        ld_chunk(th + c * 32, v);
        tmem_wait_ld();
        scale_chunk(e, v, m, n + c * 32);
#pragma unroll
        for (int d = 0; d < 32; ++d) ss = fmaf(v[d], v[d], ss);
      }
      inv = rsqrtf(ss * (1.0f / 128.0f) + e.eps_qk);
    }
    bf16* dst = nullptr;
    if (m < e.M) {
      if (e.sp_n > 0) {  // sequence parallel: straight into the head group's rank
        const int g = h / e.sp_heads, hl = h - g * e.sp_heads;
        bf16* base = part == 0 ? e.sp_q[g] : (part == 1 ? e.sp_k[g] : e.sp_v[g]);
        dst = base + ((long)hl * e.sp_L_total + e.sp_row0 + m) * 128;
      } else {
        bf16* base = part == 0 ? e.q : (part == 1 ? e.k : e.v);
        dst = base + ((long)h * e.L_pad + m) * 128;
      }
    }
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float v[32];
      ld_chunk(th + c * 32, v);
      tmem_wait_ld();
      scale_chunk(e, v, m, n + c * 32);
      if (norm_rope) {
#pragma unroll
        for (int d = 0; d < 32; d += 8) {
          const uint4 wv = __ldg(reinterpret_cast<const uint4*>(w + c * 32 + d));
          const bf16* wb = reinterpret_cast<const bf16*>(&wv);
#pragma unroll
          for (int j = 0; j < 8; ++j) v[d + j] = v[d + j] * inv * __bfloat162float(wb[j]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int ip = c * 16 + i;  // pair index within the head
          const int ax = axis_of_pair[ip];
          const float pa = ax == 0 ? p3[0] : (ax == 1 ? p3[1] : p3[2]);
          float sn, cs;
          rope_sincos(pa * freq[ip], &sn, &cs);
          const float a = v[2 * i], bb = v[2 * i + 1];
          v[2 * i] = a * cs - bb * sn;
          v[2 * i + 1] = a * sn + bb * cs;
        }
      }
      if (dst && part < 2 && e.qk_e4m3) {
        // e4m3 codes of v * 448 / (sqrt(128) max|w|): 32 bytes of the head's
        // 128-byte row
        const float inv = qk_inv[part];
        uint32_t w4[8];
#pragma unroll
        for (int d = 0; d < 32; d += 4)
          w4[d / 4] = cvt_e4m3x2(v[d] * inv, v[d + 1] * inv) | (cvt_e4m3x2(v[d + 2] * inv, v[d + 3] * inv) << 16);
        uint8_t* dst8;
        if (e.sp_n > 0) {  // sequence parallel: the codes go straight to the head group's rank
          const int g = h / e.sp_heads, hl = h - g * e.sp_heads;
          dst8 = reinterpret_cast<uint8_t*>(part == 0 ? e.sp_q[g] : e.sp_k[g]) +
                 ((long)hl * e.sp_L_total + e.sp_row0 + m) * 128 + c * 32;
        } else {
          dst8 = reinterpret_cast<uint8_t*>(part == 0 ? e.q : e.k) + ((long)h * e.L_pad + m) * 128 + c * 32;
        }
        reinterpret_cast<uint4*>(dst8)[0] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        reinterpret_cast<uint4*>(dst8)[1] = make_uint4(w4[4], w4[5], w4[6], w4[7]);
      } else if (dst) {
#pragma unroll
        for (int d = 0; d < 32; d += 8) {
          uint4 o;
          o.x = pack_bf16x2(v[d], v[d + 1]);
          o.y = pack_bf16x2(v[d + 2], v[d + 3]);
          o.z = pack_bf16x2(v[d + 4], v[d + 5]);
          o.w = pack_bf16x2(v[d + 6], v[d + 7]);
          *reinterpret_cast<uint4*>(dst + c * 32 + d) = o;
        }
      }
    }
  }
}

__device__ __forceinline__ void epi_unpatch(const GemmEpilogue& e, uint32_t tb, int m, int n0) {
  const int C = e.C_lat;
  const int t = m / (e.Ht * e.Wt), i = (m / e.Wt) % e.Ht, j = m % e.Wt;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    const int nc = n0 + c * 32;
    if (nc >= e.N) break;
    float v[32];
    ld_chunk(tb + c * 32, v);
    tmem_wait_ld();
    scale_chunk(e, v, m, nc);
    if (m < e.M) {
      for (int jj = 0; jj < 32 && nc + jj < e.N; ++jj) {
        const int f = nc + jj;
        const int ph = f / (2 * C), pw = (f / C) % 2, ch = f % C;
        const long dst = (((long)t * (2 * e.Ht) + 2 * i + ph) * (2 * e.Wt) + 2 * j + pw) * C + ch;
        float* o = static_cast<float*>(e.out) + dst;
        if (e.euler) {
          // one Euler step of the latent in out: out += dsigma * velocity
          const float a = fmaf(e.dsigma, v[jj], *o);
          *o = a;
          if (e.out_bf16) e.out_bf16[dst] = __float2bfloat16_rn(a);
        } else {
          *o = v[jj];
        }
      }
    }
  }
}

// F8: e4m3 operands (kind::f8f6f4), a K step of 128 one-byte elements; else
// bf16 (kind::f16), a K step of 64.  Both stage 128-byte rows.
template <bool F8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ GemmProblem p) {
  constexpr int KSTEP = F8 ? 2 * BK : BK;  // elements per stage
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* smA = smem;
  uint8_t* smB = smem + STAGES * A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  float* freq = reinterpret_cast<float*>(tmem_slot + 4);
  uint8_t* axis_of_pair = reinterpret_cast<uint8_t*>(freq + 64);
  float* qk_inv = reinterpret_cast<float*>(axis_of_pair + 64);
  float* epi_stage = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + MISC_BYTES);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const GemmEpilogue& e = p.epi;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (e.mode == EPI_QKV && threadIdx.x >= 64 && threadIdx.x < 128) {
    // rotation frequency of each of the 64 pairs: section t | h | w, pair i
    // of a section of width d turns by theta^(-2i/d) per unit position
    const int i = threadIdx.x - 64;
    const int pt = e.rope_t / 2, ph = e.rope_h / 2;
    int ax, i_sec, d_sec;
    if (i < pt) { ax = 0; i_sec = i; d_sec = e.rope_t; }
    else if (i < pt + ph) { ax = 1; i_sec = i - pt; d_sec = e.rope_h; }
    else { ax = 2; i_sec = i - pt - ph; d_sec = e.rope_w; }
    freq[i] = powf(e.theta, -2.0f * (float)i_sec / (float)d_sec);
    axis_of_pair[i] = (uint8_t)ax;
  }
  if (e.mode == EPI_QKV && e.qk_e4m3 && threadIdx.x >= 128 && threadIdx.x < 160) qk_e4m3_inv_scales(e, qk_inv);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int m_tiles = (p.M + BM - 1) / BM;
  const int num_tiles = m_tiles * p.n_tiles;
  const int num_kb = (p.K + KSTEP - 1) / KSTEP;
  const bool swiglu = e.mode == EPI_SWIGLU;
  // A narrow output (the heads: 96 or fewer columns) takes one 128-row B box
  // and N = 128 MMAs, half the tensor work of a 256-wide tile: these GEMMs
  // stream A from HBM and have no use for the other half
  const bool half_n = H3_GEMM_HALF_N && !F8 && p.n_tiles == 1 && p.N_b_rows <= 128 &&
                      (e.mode == EPI_STORE_F32 || e.mode == EPI_UNPATCH);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, m_tiles, p.n_tiles, p.group_m, mt, nt);
        const int b0 = nt * (swiglu ? 128 : 256);
        const int b1 = b0 + p.b_second_half_off;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], half_n ? STAGE_BYTES - B_STAGE_BYTES / 2 : STAGE_BYTES);
          tma_load_2d(smA + stage * A_STAGE_BYTES, &tmA, &full[stage], kb * KSTEP, mt * BM);
          tma_load_2d(smB + stage * B_STAGE_BYTES, &tmB, &full[stage], kb * KSTEP, b0);
          if (!half_n)
            tma_load_2d(smB + stage * B_STAGE_BYTES + B_STAGE_BYTES / 2, &tmB, &full[stage], kb * KSTEP, b1);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      drain_loads(full, STAGES, issued);
    }
  } else if (warp == 1) {
    // The whole warp runs the issue loop, converged; one elected lane issues.
    const uint32_t idesc = F8 ? idesc_e4m3_f32(BM, BN) : idesc_bf16_f32(BM, half_n ? 128 : BN, false);
    // descriptors computed once; per MMA only the start address moves
    // (16-byte units: a 32-byte K step is +2)
    const uint64_t a_desc0 = sdesc_sw128(smem_u32(smA), 16, 1024);
    const uint64_t b_desc0 = sdesc_sw128(smem_u32(smB), 16, 1024);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait_warp(&full[stage], phase)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = a_desc0 + (uint64_t)((stage * A_STAGE_BYTES) >> 4);
        const uint64_t bd = b_desc0 + (uint64_t)((stage * B_STAGE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {  // 4 MMAs of 32 bytes of K
          if constexpr (F8)
            umma_e4m3(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          else
            umma_bf16(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      umma_commit(&tfull[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    drain_mmas(drain);
  } else {
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(t, m_tiles, p.n_tiles, p.group_m, mt, nt);
      bool ok = mbar_wait(&tfull[acc], acc_phase);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int m = mt * BM + row_in_tile;
      switch (e.mode) {
        case EPI_STORE_F32: epi_store_f32(e, tb, m, nt * BN, epi_stage + q * 32 * EPI_PITCH); break;
        case EPI_GATED_RESID: epi_gated_resid(e, tb, m, nt * BN); break;
        case EPI_SWIGLU: epi_swiglu(e, tb, m, nt); break;
        case EPI_QKV: epi_qkv(e, tb, m, nt * BN, freq, axis_of_pair, qk_inv); break;
        case EPI_UNPATCH: epi_unpatch(e, tb, m, nt * BN); break;
        default: break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (cta_group::2): a cluster of two CTAs computes a 256 x 256
// tile; CTA r stages A rows [128 r, 128 r + 128) and B rows [128 r, 128 r + 128)
// of the tile (for SwiGLU: r = 0 the gate rows, r = 1 the up rows) in its own
// shared memory, and the leader CTA (rank 0) issues M = 256 MMAs that read
// both CTAs' operands and leave each CTA's 128 result rows in its own TMEM.
// Per CTA this stages 32 KB per 64-deep K step instead of 48 KB.
#ifndef H3_GEMM_PAIR_STAGES
#define H3_GEMM_PAIR_STAGES 6
#endif
constexpr int P_STAGES = H3_GEMM_PAIR_STAGES;
constexpr int P_A_BYTES = 128 * BK * 2;             // 16 KB
constexpr int P_B_BYTES = 128 * BK * 2;             // 16 KB (half of the 256 columns)
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + 1024 + MISC_BYTES;
// Warp 0 TMA, warp 1 MMA (leader CTA), warps 2-9 epilogue: two warps per TMEM
// lane quarter, each taking half of the tile's 256 columns, so that one
// warp's loads and stores overlap the other's arithmetic.  With e4m3 operands
// (half the MMA time per tile) one epilogue warp per quarter bounded the QKV
// GEMM (epilogue busy 20.3K of the MMAs' 21.5K SM clocks per tile) and the
// out-projection (34K against 29K).
constexpr int P_NUM_THREADS = 320;

template <bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_NUM_THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ GemmProblem p) {
  constexpr int KSTEP = F8 ? 2 * BK : BK;  // elements per stage
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* smA = smem;
  uint8_t* smB = smem + P_STAGES * P_A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES);
  uint64_t* empty = full + P_STAGES;
  uint64_t* tfull = empty + P_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  float* freq = reinterpret_cast<float*>(tmem_slot + 4);
  uint8_t* axis_of_pair = reinterpret_cast<uint8_t*>(freq + 64);
  float* qk_inv = reinterpret_cast<float*>(axis_of_pair + 64);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const GemmEpilogue& e = p.epi;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);    // the leader's producer arrives (+ both CTAs' bytes)
      mbar_init(&empty[s], 1);   // the leader's MMA commit, delivered to both CTAs
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);   // the leader's commit, delivered to both CTAs
      mbar_init(&tempty[a], 16);  // 8 epilogue warps in each CTA (leader's copy used)
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (e.mode == EPI_QKV && threadIdx.x >= 64 && threadIdx.x < 128) {
    const int i = threadIdx.x - 64;
    const int pt = e.rope_t / 2, ph = e.rope_h / 2;
    int ax, i_sec, d_sec;
    if (i < pt) { ax = 0; i_sec = i; d_sec = e.rope_t; }
    else if (i < pt + ph) { ax = 1; i_sec = i - pt; d_sec = e.rope_h; }
    else { ax = 2; i_sec = i - pt - ph; d_sec = e.rope_w; }
    freq[i] = powf(e.theta, -2.0f * (float)i_sec / (float)d_sec);
    axis_of_pair[i] = (uint8_t)ax;
  }
  if (e.mode == EPI_QKV && e.qk_e4m3 && threadIdx.x >= 128 && threadIdx.x < 160) qk_e4m3_inv_scales(e, qk_inv);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int m_pairs = (p.M + 255) / 256;
  const int num_tiles = m_pairs * p.n_tiles;
  const int num_kb = (p.K + KSTEP - 1) / KSTEP;
  const bool swiglu = e.mode == EPI_SWIGLU;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t leader_full0 = mapa_shared(smem_u32(&full[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += n_pairs) {
        int mt, nt;
        tile_coords(t, m_pairs, p.n_tiles, p.group_m, mt, nt);
        const int arow = mt * 256 + (int)rank * 128;
        const int brow = nt * (swiglu ? 128 : 256) + (int)rank * p.b_second_half_off;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * P_STAGE_BYTES);
          const uint32_t fb = leader_full0 + stage * 8;
          tma_load_2d_pair(smA + stage * P_A_BYTES, &tmA, fb, kb * KSTEP, arow);
          tma_load_2d_pair(smB + stage * P_B_BYTES, &tmB, fb, kb * KSTEP, brow);
          ++issued;
          if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // the leader's full barriers count both CTAs' bytes: the leader waits
      // for both, the peer CTA is held by the cluster barrier below
      if (leader) drain_loads(full, P_STAGES, issued);
    }
  } else if (warp == 1) {
    if (leader) {
      // The leader's whole warp runs the issue loop, converged; one elected lane issues.
      const uint32_t idesc = F8 ? idesc_e4m3_f32(256, 256) : idesc_bf16_f32(256, 256, false);
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(smA), 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(smB), 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += n_pairs) {
        if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_warp(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = a_desc0 + (uint64_t)((stage * P_A_BYTES) >> 4);
          const uint64_t bd = b_desc0 + (uint64_t)((stage * P_B_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {  // 4 MMAs of 32 bytes of K
            if constexpr (F8)
              umma_e4m3_pair(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc,
                             (kb | kk) != 0 ? 1u : 0u);
            else
              umma_bf16_pair(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc,
                             (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&empty[stage]);
          if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
        }
        umma_commit_pair(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      umma_commit_pair(drain);
      mbar_wait(drain, 0);
    }
  } else {
    const int q = warp & 3;     // TMEM lane quarter
    const int sub = (warp - 2) >> 2;  // which half of the tile's columns
    const int row_in_tile = q * 32 + lane;
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < num_tiles; t += n_pairs) {
      int mt, nt;
      tile_coords(t, m_pairs, p.n_tiles, p.group_m, mt, nt);
      bool ok = mbar_wait(&tfull[acc], acc_phase);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int m = mt * 256 + (int)rank * 128 + row_in_tile;
      switch (e.mode) {  // the modes the launcher routes here
        case EPI_GATED_RESID:
          // the fp32 residual read-modify-write: split between the two
          // warps only where the MMAs of a tile are short, e4m3 operands and
          // K <= 8192 (out-projection 0.244 -> 0.236 ms at 7,904 tokens;
          // split, the e4m3 FFN down-projection took 3.6% more cycles and the
          // bf16 out-projection 0.416 -> 0.427 ms); else one warp per quarter
          // takes all 256 columns
          if (F8 && p.K <= 8192)
            epi_gated_resid(e, tb, m, nt * BN, sub * 4, sub * 4 + 4);
          else if (sub == 0)
            epi_gated_resid(e, tb, m, nt * BN);
          break;
        case EPI_SWIGLU: epi_swiglu(e, tb, m, nt, sub * 2, sub * 2 + 2); break;
        case EPI_QKV: epi_qkv(e, tb, m, nt * BN, freq, axis_of_pair, qk_inv, sub, sub + 1); break;
        default: break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + acc * 8);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no MMA of the pair is in flight and no remote arrival pending
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace gemm_detail
using namespace gemm_detail;

// 2-D tensor map with 128-byte inner boxes (64 bf16 or 128 one-byte
// elements) and 128-byte swizzle; out-of-range elements read as zero.
static bool make_tmap_128b(CUtensorMap* map, CUtensorMapDataType dt, uint32_t elem_bytes, const void* base,
                           uint64_t rows, uint64_t cols, uint64_t row_stride_elems, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {row_stride_elems * elem_bytes};
  cuuint32_t box[2] = {128 / elem_bytes, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                    uint32_t box_rows) {
  return make_tmap_128b(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, row_stride_elems, box_rows);
}

bool make_tmap_e4m3(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                    uint32_t box_rows) {
  return make_tmap_128b(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, rows, cols, row_stride_elems, box_rows);
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned long long* done_mask) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const unsigned long long bit = 1ull << (dev & 63);
  if (*done_mask & bit) return cudaSuccess;
  err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess) *done_mask |= bit;
  return err;
}

cudaError_t launch_gemm(const GemmProblem& p, cudaStream_t stream) {
  if (p.M <= 0) return cudaSuccess;
  const bool f8 = p.f8 != 0;
  if (f8 && (p.a_scale == nullptr || p.b_scale == nullptr)) return cudaErrorInvalidValue;
  static unsigned long long attr_done[2] = {0, 0};
  const void* k1 = f8 ? reinterpret_cast<const void*>(gemm_tc_kernel<true>)
                      : reinterpret_cast<const void*>(gemm_tc_kernel<false>);
  cudaError_t aerr = ensure_smem_attr(k1, gemm_detail::SMEM_BYTES, &attr_done[f8 ? 1 : 0]);
  if (aerr != cudaSuccess) return aerr;
  CUtensorMap tmA, tmB;
  auto make = f8 ? make_tmap_e4m3 : make_tmap_bf16;
  if (!make(&tmA, p.A, (uint64_t)p.M, (uint64_t)p.K, (uint64_t)p.lda, 128)) return cudaErrorInvalidValue;
  if (!make(&tmB, p.B, (uint64_t)p.N_b_rows, (uint64_t)p.K, (uint64_t)p.ldb, 128)) return cudaErrorInvalidValue;
  const int m_tiles = (p.M + gemm_detail::BM - 1) / gemm_detail::BM;
  const int tiles = m_tiles * p.n_tiles;
  GemmProblem q = p;
  q.epi.a_scale = f8 ? p.a_scale : nullptr;
  q.epi.b_scale = f8 ? p.b_scale : nullptr;
  q.epi.a_rows = p.M;
  q.epi.b_rows = p.N_b_rows;
  if (q.group_m <= 0) {
    // A band of row tiles whose A panel (128 rows x K bf16 each) takes about
    // 24 MB of L2, so it stays resident while B streams past.  Measured on
    // B200 (FFN / QKV / out-projection at 32,160 tokens): 11.2 / 5.2 / 2.0 ms
    // with 24 MB bands against 14.5 / 6.8 / 2.4 ms with one band of all row
    // tiles (which re-read the whole A panel from DRAM every wave).
#ifndef H3_GEMM_BAND_BYTES
#define H3_GEMM_BAND_BYTES (24ll << 20)
#endif
    const long long panel = 128ll * p.K * (f8 ? 1 : 2);
    long long g = H3_GEMM_BAND_BYTES / (panel > 0 ? panel : 1);
    q.group_m = (int)(g < 1 ? 1 : (g > m_tiles ? m_tiles : g));
  }
#ifndef H3_GEMM_PAIR
#define H3_GEMM_PAIR 1
#endif
  // The block's four GEMMs use the pair kernel.  Measured on B200 at 7,904 /
  // 32,160 tokens: out-projection 0.49 / 1.96 -> 0.45 / 1.79 ms, QKV 1.30 /
  // 5.33 -> 1.27 / 5.24 ms; FFN gate/up and down 7% / 13% and 6% / 12% fewer
  // SM cycles (ncu, clock-independent).  The input projections and the heads
  // (small M or N) stay on the one-CTA kernel.
  const bool pair_mode = p.epi.mode == EPI_QKV || p.epi.mode == EPI_GATED_RESID || p.epi.mode == EPI_SWIGLU;
  if (H3_GEMM_PAIR && p.pair == 1 && p.M > 128 && pair_mode) {
    static unsigned long long attr2_done[2] = {0, 0};
    const void* k2 = f8 ? reinterpret_cast<const void*>(gemm_detail::gemm_tc2_kernel<true>)
                        : reinterpret_cast<const void*>(gemm_detail::gemm_tc2_kernel<false>);
    cudaError_t err2 = ensure_smem_attr(k2, gemm_detail::P_SMEM_BYTES, &attr2_done[f8 ? 1 : 0]);
    if (err2 != cudaSuccess) return err2;
    const int m_pairs = (p.M + 255) / 256;
    GemmProblem q2 = q;
    // bands of as many 256-row pairs as the one-CTA kernel takes 128-row
    // tiles (48 MB of A): measured on the FFN GEMMs, 14-16% less DRAM read
    // and slightly fewer cycles than bands of the same rows
    if (p.group_m <= 0) q2.group_m = q.group_m > 0 ? q.group_m : 1;
    if (q2.group_m > m_pairs) q2.group_m = m_pairs;
    const int pair_tiles = m_pairs * p.n_tiles;
    const int max_pairs = num_sms() / 2;
    const int pairs = pair_tiles < max_pairs ? pair_tiles : max_pairs;
    if (f8)
      gemm_detail::gemm_tc2_kernel<true><<<2 * pairs, gemm_detail::P_NUM_THREADS, gemm_detail::P_SMEM_BYTES, stream>>>(
          tmA, tmB, q2);
    else
      gemm_detail::gemm_tc2_kernel<false><<<2 * pairs, gemm_detail::P_NUM_THREADS, gemm_detail::P_SMEM_BYTES,
                                            stream>>>(tmA, tmB, q2);
    return cudaGetLastError();
  }
  const int grid = tiles < num_sms() ? tiles : num_sms();
  if (f8)
    gemm_tc_kernel<true><<<grid, gemm_detail::NUM_THREADS, gemm_detail::SMEM_BYTES, stream>>>(tmA, tmB, q);
  else
    gemm_tc_kernel<false><<<grid, gemm_detail::NUM_THREADS, gemm_detail::SMEM_BYTES, stream>>>(tmA, tmB, q);
  return cudaGetLastError();
}

}  // namespace h3

// Memory-bound kernels of the block step: packing/patchify, LayerNorm with
// range-selected modulation, and the flow-sampler Euler update.
#include "h3_internal.cuh"
#include "ptx.cuh"

namespace h3 {

namespace ew_detail {

__device__ __forceinline__ int range_of(int row, const int* rs, const int* rc) {
#pragma unroll
  for (int m = 0; m < 3; ++m)
    if (row >= rs[m] && row < rs[m] + rc[m]) return m;
  return -1;
}

struct RangeArgs {
  int start[3], count[3];
};

// ------------------------------------------------------------ packing
// One thread per 8-byte (4 x bf16) piece of a patch row: a video token
// (t, i, j) takes latent pixels (t, 2i+ph, 2j+pw), ph/pw in {0,1}, in the
// order f = (ph*2 + pw)*C + c ("MiniMax-H3 paper reading" (gojay.top) §4,
// §7.3: 1x2x2 patchify over (t, h, w), time untouched).
__global__ void patchify_kernel(const bf16* __restrict__ video, int T, int Hl, int Wl, int C,
                                bf16* __restrict__ patches) {
  const int Ht = Hl / 2, Wt = Wl / 2;
  const long n_tok = (long)T * Ht * Wt;
  const int pieces_per_tok = C;  // 4*C elements = C pieces of 4
  const long total = n_tok * pieces_per_tok;
  for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const long r = idx / pieces_per_tok;
    const int f = (int)(idx % pieces_per_tok) * 4;
    const int q = f / C, c = f % C;  // q = ph*2 + pw
    const int ph = q >> 1, pw = q & 1;
    const int t = (int)(r / (Ht * Wt)), i = (int)((r / Wt) % Ht), j = (int)(r % Wt);
    const long src = (((long)t * Hl + 2 * i + ph) * Wl + 2 * j + pw) * C + c;
    *reinterpret_cast<uint2*>(patches + r * 4 * C + f) = *reinterpret_cast<const uint2*>(video + src);
  }
}

// Positions, modality ids and zeroed padding rows.  Video token (t, i, j)
// sits at (t, i, j); audio latent k of either channel at (6k/40, 0, 0) so
// that 40 Hz audio and 24/4 = 6 Hz video latents share one time axis with
// h = w = 0 for audio ("MiniMax-H3 paper reading" §7.4); text at (0, 0, 0).
__global__ void positions_kernel(RangeArgs rg, int Ht, int Wt, int n_audio, int L, int L_pad, float* __restrict__ pos,
                                 uint8_t* __restrict__ mod_ids) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= L_pad) return;
  float p0 = 0.f, p1 = 0.f, p2 = 0.f;
  int m = row < L ? range_of(row, rg.start, rg.count) : -1;
  if (m == 1) {
    const int k = (row - rg.start[1]) % n_audio;
    p0 = __fdiv_rn((float)(6 * k), 40.0f);
  } else if (m == 2) {
    const int r = row - rg.start[2];
    p0 = (float)(r / (Ht * Wt));
    p1 = (float)((r / Wt) % Ht);
    p2 = (float)(r % Wt);
  }
  pos[row * 3 + 0] = p0;
  pos[row * 3 + 1] = p1;
  pos[row * 3 + 2] = p2;
  mod_ids[row] = m < 0 ? (uint8_t)255 : (uint8_t)m;
}

__global__ void zero_rows_kernel(float* __restrict__ x, long first, long last, int D) {
  const long n = (last - first) * D;
  float* base = x + first * D;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) base[i] = 0.f;
}

// ------------------------------------------------------------ LN + modulate
// One CTA per row; thread i keeps float4 elements i, i + T, i + 2T, ... of the
// row in registers (up to LN_VPT of them).  Two-pass mean/variance in fp32
// (biased variance), h = (x - mu) / sqrt(var + eps), out = h * (1 + scale_m) +
// shift_m with m the modality of the row's token range ("MiniMax-H3: native
// joint audio-video generation" (note.shouss.top) §3, §3.1).  mod == nullptr:
// plain LN.  Stores are 8 bytes (4 bf16) per float4 read.
#ifndef H3_LN_THREADS
#define H3_LN_THREADS 256
#endif
constexpr int LN_THREADS = H3_LN_THREADS;
constexpr int LN_VPT = (2048 + LN_THREADS - 1) / LN_THREADS;  // up to 8192 columns

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < (LN_THREADS + 31) / 32; ++i) t += red[i];
  return t;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < (LN_THREADS + 31) / 32; ++i) t = fmaxf(t, red[i]);
  return t;
}

// Per-row e4m3 scaling (OFP8 e4m3, saturating round-to-nearest-even): for a
// row with amax = max |y| > 0, rscale = 448 / amax and scale = amax / 448 (both
// IEEE fp32 divisions), code = e4m3(y * rscale) with the product rounded to
// fp32; a zero row has rscale = scale = 0.
__device__ __forceinline__ void e4m3_row_scales(float amax, float& rscale, float& scale) {
  rscale = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
}
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d, float rs) {
  return cvt_e4m3x2(__fmul_rn(a, rs), __fmul_rn(b, rs)) | (cvt_e4m3x2(__fmul_rn(c, rs), __fmul_rn(d, rs)) << 16);
}

// E4M3 = false: out is bf16 [L_pad][D].  E4M3 = true: out is e4m3 codes
// [L_pad][D] (bytes) with one fp32 scale per row in out_scale, quantised
// from the fp32 values of the modulated row.
template <bool E4M3>
__global__ void __launch_bounds__(LN_THREADS) ln_modulate_kernel(const float* __restrict__ x,
                                                                  const float* __restrict__ mod, int branch,
                                                                  RangeArgs rg, int L, int D, float eps,
                                                                  void* __restrict__ out,
                                                                  float* __restrict__ out_scale) {
  __shared__ float red[(LN_THREADS + 31) / 32];
  const int row = blockIdx.x;
  const int nv = D / 4;
  bf16* orow = static_cast<bf16*>(out) + (long)row * D;
  uint8_t* qrow = static_cast<uint8_t*>(out) + (long)row * D;
  if (row >= L) {
    for (int i = threadIdx.x; i < nv; i += LN_THREADS) {
      if (E4M3)
        *reinterpret_cast<uint32_t*>(qrow + 4 * i) = 0u;
      else
        *reinterpret_cast<uint2*>(orow + 4 * i) = make_uint2(0, 0);
    }
    if (E4M3 && threadIdx.x == 0) out_scale[row] = 0.f;
    return;
  }
  const float4* xr = reinterpret_cast<const float4*>(x + (long)row * D);
  float4 v[LN_VPT];
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < LN_VPT; ++k) {
    const int i = threadIdx.x + k * LN_THREADS;
    if (i < nv) {
      v[k] = __ldcs(xr + i);
      s += (v[k].x + v[k].y) + (v[k].z + v[k].w);
    }
  }
  const float mu = block_sum(s, red) / (float)D;
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < LN_VPT; ++k) {
    const int i = threadIdx.x + k * LN_THREADS;
    if (i < nv) {
      const float a = v[k].x - mu, b = v[k].y - mu, c = v[k].z - mu, d = v[k].w - mu;
      ss += (a * a + b * b) + (c * c + d * d);
    }
  }
  const float var = block_sum(ss, red) / (float)D;
  const float inv = rsqrtf(var + eps);
  const int m = range_of(row, rg.start, rg.count);
  const float4* shift = mod ? reinterpret_cast<const float4*>(mod + (long)(m * 6 + 3 * branch + 0) * D) : nullptr;
  const float4* scale = mod ? reinterpret_cast<const float4*>(mod + (long)(m * 6 + 3 * branch + 1) * D) : nullptr;
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < LN_VPT; ++k) {
    const int i = threadIdx.x + k * LN_THREADS;
    if (i < nv) {
      float a = (v[k].x - mu) * inv, b = (v[k].y - mu) * inv, c = (v[k].z - mu) * inv, d = (v[k].w - mu) * inv;
      if (mod) {
        const float4 sh = __ldg(shift + i), sc = __ldg(scale + i);
        a = fmaf(a, 1.f + sc.x, sh.x);
        b = fmaf(b, 1.f + sc.y, sh.y);
        c = fmaf(c, 1.f + sc.z, sh.z);
        d = fmaf(d, 1.f + sc.w, sh.w);
      }
      if (E4M3) {
        v[k] = make_float4(a, b, c, d);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d))));
      } else {
        *reinterpret_cast<uint2*>(orow + 4 * i) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
      }
    }
  }
  if (E4M3) {
    float rs, sc;
    e4m3_row_scales(block_max(amax, red), rs, sc);
    if (threadIdx.x == 0) out_scale[row] = sc;
#pragma unroll
    for (int k = 0; k < LN_VPT; ++k) {
      const int i = threadIdx.x + k * LN_THREADS;
      if (i < nv) *reinterpret_cast<uint32_t*>(qrow + 4 * i) = e4m3x4(v[k].x, v[k].y, v[k].z, v[k].w, rs);
    }
  }
}

// ------------------------------------------------------------ row quantiser
// One CTA per row of a bf16 matrix: amax over the row, then codes with the
// row scaling above.  cols, ld_in and ld_q are multiples of 8.
__global__ void __launch_bounds__(LN_THREADS) quantize_rows_e4m3_kernel(const bf16* __restrict__ in, long ld_in,
                                                                         int cols, uint8_t* __restrict__ q,
                                                                         long ld_q, float* __restrict__ scale) {
  __shared__ float red[(LN_THREADS + 31) / 32];
  const int row = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(in + (long)row * ld_in);
  const int n8 = cols / 8;
  float amax = 0.f;
  for (int i = threadIdx.x; i < n8; i += LN_THREADS) {
    const uint4 w = __ldg(src + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  float rs, sc;
  e4m3_row_scales(block_max(amax, red), rs, sc);
  if (threadIdx.x == 0) scale[row] = sc;
  uint2* dst = reinterpret_cast<uint2*>(q + (long)row * ld_q);
  for (int i = threadIdx.x; i < n8; i += LN_THREADS) {
    const uint4 w = __ldg(src + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
    const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
    const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
    dst[i] = make_uint2(e4m3x4(f0.x, f0.y, f1.x, f1.y, rs), e4m3x4(f2.x, f2.y, f3.x, f3.y, rs));
  }
}

// ------------------------------------------------------------ Euler
// lat += (sigma_next - sigma) * vel  ("MiniMax-H3: native joint audio-video
// generation" §6: RF velocity, Euler update on the generation targets).
__global__ void euler_kernel(float* __restrict__ lat, const float* __restrict__ vel, long long n, float dsigma) {
  const long long nv = n / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  float4* l4 = reinterpret_cast<float4*>(lat);
  const float4* v4 = reinterpret_cast<const float4*>(vel);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nv; i += stride) {
    float4 a = l4[i];
    const float4 b = __ldcs(v4 + i);
    a.x = fmaf(dsigma, b.x, a.x);
    a.y = fmaf(dsigma, b.y, a.y);
    a.z = fmaf(dsigma, b.z, a.z);
    a.w = fmaf(dsigma, b.w, a.w);
    l4[i] = a;
  }
  for (long long i = nv * 4 + blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += stride)
    lat[i] = fmaf(dsigma, vel[i], lat[i]);
}

// Euler update that also writes the bf16 copy the next step's packing reads.
__global__ void euler_bf16_kernel(float* __restrict__ lat, const float* __restrict__ vel, long long n, float dsigma,
                                  bf16* __restrict__ out) {
  const long long nv = n / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  float4* l4 = reinterpret_cast<float4*>(lat);
  const float4* v4 = reinterpret_cast<const float4*>(vel);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nv; i += stride) {
    float4 a = l4[i];
    const float4 b = __ldcs(v4 + i);
    a.x = fmaf(dsigma, b.x, a.x);
    a.y = fmaf(dsigma, b.y, a.y);
    a.z = fmaf(dsigma, b.z, a.z);
    a.w = fmaf(dsigma, b.w, a.w);
    l4[i] = a;
    *reinterpret_cast<uint2*>(out + 4 * i) = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
  for (long long i = nv * 4 + blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += stride) {
    const float a = fmaf(dsigma, vel[i], lat[i]);
    lat[i] = a;
    out[i] = __float2bfloat16_rn(a);
  }
}

// One thread waits on an mbarrier that nothing arrives on: the bounded wait
// gives up after limit_ns and records its error code, like any stalled
// pipeline wait in the tensor-core kernels.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait_limit(&bar, 0, limit_ns);
}

// a[i] = bf16(SiLU(c[i])) = bf16(c / (1 + e^-c)): the conditioning vectors
// of the AdaLN producer, as the A operand of its GEMM
__global__ void silu_bf16_kernel(const float* __restrict__ c, long long n, bf16* __restrict__ a) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = c[i];
    a[i] = __float2bfloat16_rn(v / (1.0f + expf(-v)));
  }
}

}  // namespace ew_detail
using namespace ew_detail;

cudaError_t launch_silu_bf16(const float* c, long long n, bf16* a, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  long long blocks = (n + 255) / 256;
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  silu_bf16_kernel<<<(int)blocks, 256, 0, stream>>>(c, n, a);
  return cudaGetLastError();
}

cudaError_t launch_pack(const bf16* video, int T, int Hl, int Wl, int C_lat, int n_audio, int audio_channels,
                        const int* rstart, const int* rcount, int L, int L_pad, bf16* patches, float* pos,
                        uint8_t* mod_ids, float* x, int D, cudaStream_t stream) {
  (void)audio_channels;
  RangeArgs rg;
  for (int m = 0; m < 3; ++m) {
    rg.start[m] = rstart[m];
    rg.count[m] = rcount[m];
  }
  const long n_tok = (long)T * (Hl / 2) * (Wl / 2);
  if (n_tok > 0) {
    const long total = n_tok * C_lat;
    const int threads = 256;
    long blocks = (total + threads - 1) / threads;
    if (blocks > 148L * 16) blocks = 148L * 16;
    patchify_kernel<<<(int)blocks, threads, 0, stream>>>(video, T, Hl, Wl, C_lat, patches);
  }
  positions_kernel<<<(L_pad + 255) / 256, 256, 0, stream>>>(rg, Hl / 2, Wl / 2, n_audio > 0 ? n_audio : 1, L, L_pad,
                                                            pos, mod_ids);
  if (L_pad > L) {
    long n = (long)(L_pad - L) * D;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    zero_rows_kernel<<<blocks, 256, 0, stream>>>(x, L, L_pad, D);
  }
  return cudaGetLastError();
}

cudaError_t launch_ln_modulate(const float* x, const float* mod, int branch, const int* rstart, const int* rcount,
                               int L, int L_pad, int D, float eps, bf16* out, cudaStream_t stream) {
  RangeArgs rg;
  for (int m = 0; m < 3; ++m) {
    rg.start[m] = rstart[m];
    rg.count[m] = rcount[m];
  }
  ln_modulate_kernel<false><<<L_pad, LN_THREADS, 0, stream>>>(x, mod, branch, rg, L, D, eps, out, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_ln_modulate_e4m3(const float* x, const float* mod, int branch, const int* rstart,
                                    const int* rcount, int L, int L_pad, int D, float eps, uint8_t* out,
                                    float* out_scale, cudaStream_t stream) {
  RangeArgs rg;
  for (int m = 0; m < 3; ++m) {
    rg.start[m] = rstart[m];
    rg.count[m] = rcount[m];
  }
  ln_modulate_kernel<true><<<L_pad, LN_THREADS, 0, stream>>>(x, mod, branch, rg, L, D, eps, out, out_scale);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_e4m3(const bf16* in, long ld_in, int rows, int cols, uint8_t* q, long ld_q,
                                      float* scale, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  quantize_rows_e4m3_kernel<<<rows, LN_THREADS, 0, stream>>>(in, ld_in, cols, q, ld_q, scale);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 1, 0, stream>>>(limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_euler_bf16(float* lat, const float* vel, long long n, float dsigma, bf16* out,
                              cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  long long blocks = (n / 4 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  euler_bf16_kernel<<<(int)blocks, 256, 0, stream>>>(lat, vel, n, dsigma, out);
  return cudaGetLastError();
}

cudaError_t launch_euler(float* lat, const float* vel, long long n, float dsigma, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  long long blocks = (n / 4 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  euler_kernel<<<(int)blocks, 256, 0, stream>>>(lat, vel, n, dsigma);
  return cudaGetLastError();
}

}  // namespace h3

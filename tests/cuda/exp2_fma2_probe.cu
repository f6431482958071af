// Test-only probe (not part of libh3.so): the attention softmax's FMA-pipe
// exponential exp2_fma2 applied elementwise, y[i] = 2^(k s[i] + c) with the
// operands in the form the softmax passes them (a = k / 252,
// b = (125 + c) / 252; the exponent clamped to [-125, 127]), so that a test
// can hold it against its error bound.  Built by
// omni_modal_diffusion_b200/build.py (build_probe).
#include "../../omni_modal_diffusion_b200/csrc/ptx.cuh"

namespace {
// y[i] = exp2_fma2 of s[i] with the softmax's operands a = k / 252,
// b = (125 + c) / 252, i.e. 2^(k s + c) clamped to [2^-125, 2^127]
__global__ void exp2_fma2_kernel(const float* __restrict__ s, float* __restrict__ y, long long n, float a, float b) {
  const long long pairs = (n + 1) / 2;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < pairs;
       i += (long long)gridDim.x * blockDim.x) {
    const long long i0 = 2 * i, i1 = (2 * i + 1 < n) ? 2 * i + 1 : 2 * i;
    float y0, y1;
    h3::f2_unpack(h3::exp2_fma2(s[i0], s[i1], a, b), y0, y1);
    y[i0] = y0;
    if (i1 != i0) y[i1] = y1;
  }
}
}  // namespace

// s, y: device arrays of n fp32 values; returns a cudaError_t code.
extern "C" int exp2_fma2_probe(const float* s, float* y, long long n, float k, float c, void* stream) {
  if (n <= 0) return 0;
  long long blocks = ((n + 1) / 2 + 255) / 256;
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  exp2_fma2_kernel<<<(int)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(s, y, n, k * (1.0f / 252.0f),
                                                                                (125.0f + c) * (1.0f / 252.0f));
  return (int)cudaGetLastError();
}

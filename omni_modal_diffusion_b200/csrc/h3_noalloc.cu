// h3_ffn_swiglu_noalloc: the gated SwiGLU FFN with its intermediate
// workspace held in a fixed, file-scope device array instead of a buffer the
// caller passes in.  For callers that own only their inputs and outputs and
// cannot obtain device memory for scratch: a plugin or operator interface
// that hands over tensors but no workspace, a host process whose device
// memory is entirely reserved by another allocator, or a serving loop that
// must not allocate on its hot path.  This variant has no counterpart on the
// pages; it computes exactly what h3_ffn_swiglu computes.
//
// The array is H3_FFN_STATIC_WS_BYTES (32 MiB) on every GPU that loads the
// library, held until the process exits.  In host code the name of a
// __device__ array is only a host-side stand-in, never a device address, so
// the device address is obtained once per device with cudaGetSymbolAddress
// (with that device current) and passed to the kernels.
//
// Included into h3_api.cu (one translation unit): it uses that file's
// argument checks and the GEMM launcher.

#include <mutex>

namespace {

constexpr size_t kStaticWsBytes = (size_t)H3_FFN_STATIC_WS_BYTES;

// Workspace of h3_ffn_swiglu_noalloc: SiLU(gate) * up, bf16 [L_pad][F].
static __device__ __align__(256) unsigned char g_ffn_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 256;
std::mutex g_static_ws_mu;
void* g_static_ws_addr[kMaxDevices] = {};

// Device address of g_ffn_static_ws on the current device, looked up on the
// first call for that device and cached.
int static_ws_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(H3_ERR_CUDA, "h3_ffn_swiglu_noalloc: device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_static_ws_mu);
  if (!g_static_ws_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ffn_static_ws);
    if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu_noalloc: cudaGetSymbolAddress");
    if (!p) return fail(H3_ERR_CUDA, "h3_ffn_swiglu_noalloc: cudaGetSymbolAddress returned NULL");
    g_static_ws_addr[dev] = p;
  }
  *out = g_static_ws_addr[dev];
  return H3_OK;
}

}  // namespace

extern "C" int h3_ffn_swiglu_noalloc(const h3_dims* dims, const h3_ranges* ranges, float* x, const h3_bf16* xm,
                                     const h3_bf16* Wgu, const h3_bf16* Wd, const float* mod, void* stream) {
  H3_TRACE();
  H3_CHECK(check_dims(dims, __func__));
  H3_CHECK(check_ranges(ranges, __func__));
  H3_REQUIRE_PTR(x);
  H3_REQUIRE_PTR(xm);
  H3_REQUIRE_PTR(Wgu);
  H3_REQUIRE_PTR(Wd);
  H3_REQUIRE_PTR(mod);
  const int F = dims->F, Lp = ranges->L_pad;
  const size_t need = (size_t)Lp * (size_t)F * 2;
  if (need > kStaticWsBytes)
    return fail(H3_ERR_SHAPE,
                "%s: L_pad * F * 2 = %zu bytes of workspace needed, the static workspace holds %zu bytes "
                "(L_pad * F must be at most %zu); use h3_ffn_swiglu with a caller workspace instead",
                __func__, need, kStaticWsBytes, kStaticWsBytes / 2);
  void* ws = nullptr;
  H3_CHECK(static_ws_address(&ws));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // gate/up GEMM writes every element [0, L_pad) x [0, F) of the workspace
  // that the down GEMM then reads, so nothing in it needs to start at zero.
  GemmProblem p1 = swiglu_problem(dims, Lp, xm, Wgu, ws);
  cudaError_t e = launch_gemm(p1, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu_noalloc: gate/up");
  GemmProblem p2 = gated_problem(dims, ranges, x, ws, F, Wd, mod, 5);
  e = launch_gemm(p2, st);
  if (e != cudaSuccess) return cuda_fail(e, "h3_ffn_swiglu_noalloc: down");
  return ok();
}

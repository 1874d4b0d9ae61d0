// noalloc.cu -- hsa_context_kv_noalloc: the context key/value projection for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine, torch's caching
// allocator included) at the point where they need this projection -- for example a
// host runtime whose memory budget was fixed at start-up, or code running where an
// allocation would synchronise the device.  hsa_context_kv asks them for a scratch
// buffer of L x 2D floats; this variant uses a buffer that lives inside the library
// instead: the file-scope array g_ctx_scratch below, 8 MiB, which every GPU that loads
// libhsa holds until the process exits.
//
// Host code must not pass g_ctx_scratch itself to a kernel: in host code that name is a
// host-side stand-in, not a device address.  The device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the first call
// made on it; that first call should therefore come before any stream capture.
#include <mutex>

#include "common.cuh"

namespace hsa {

constexpr size_t kCtxScratchBytes = size_t(8) << 20;   // 8 MiB: L x 2D x 4 bytes must fit
static __device__ __align__(256) uint8_t g_ctx_scratch[kCtxScratchBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

// Device address of g_ctx_scratch on the current device (looked up once per device).
int ctx_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(HSA_ECUDA, std::string("context_kv_noalloc: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return set_error(HSA_ECUDA, "context_kv_noalloc: device index out of range");
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ctx_scratch);
    if (e != cudaSuccess || !p)
      return set_error(HSA_ECUDA, std::string("context_kv_noalloc: cudaGetSymbolAddress failed: ") +
                                      cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HSA_OK;
}
}  // namespace

}  // namespace hsa

extern "C" size_t hsa_context_kv_noalloc_max_bytes(void) { return hsa::kCtxScratchBytes; }

extern "C" int hsa_context_kv_noalloc(const void* d_ctx, int L, int D, int dtype, const void* d_w_kv2,
                                      const float* d_b_kv2, const float* d_g_k2, void* d_k2, void* d_v2,
                                      void* stream) {
  using namespace hsa;
  if (L <= 0 || D <= 0) return set_error(HSA_EINVAL, "context_kv_noalloc: need L > 0 and D > 0");
  const size_t need = hsa_context_kv_workspace_size(L, D);
  if (need > kCtxScratchBytes)
    return set_error(HSA_EINVAL, "context_kv_noalloc: L x 2D x 4 bytes exceeds the 8 MiB built-in scratch; "
                                 "use hsa_context_kv with a caller workspace");
  void* scratch = nullptr;
  const int rc = ctx_scratch_address(&scratch);
  if (rc != HSA_OK) return rc;
  // The projection writes every scratch element it later reads, so nothing needs clearing.
  return hsa_context_kv(d_ctx, L, D, dtype, d_w_kv2, d_b_kv2, d_g_k2, d_k2, d_v2, scratch, need, stream);
}

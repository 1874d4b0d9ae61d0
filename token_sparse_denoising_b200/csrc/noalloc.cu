// noalloc.cu -- hsa_context_kv_noalloc: the context key/value projection for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine, torch's caching
// allocator included) at the point where they need this projection -- for example a
// host runtime whose memory budget was fixed at start-up, or code running where an
// allocation would synchronise the device.  hsa_context_kv asks them for a scratch
// buffer of L x 2D elements; this variant uses a buffer that lives inside the library
// instead: the file-scope array g_ctx_scratch below, 8 MiB, which every GPU that loads
// libhsa holds until the process exits.
//
// Host code must not pass g_ctx_scratch itself to a kernel: in host code that name is a
// host-side stand-in, not a device address.  The device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the first call
// made on it (and again on the first call after the device's context has been replaced,
// e.g. by cudaDeviceReset, which reloads the module); that first call should therefore
// come before any stream capture.
#include "common.cuh"

namespace hsa {

constexpr size_t kCtxScratchBytes = size_t(8) << 20;   // 8 MiB: L x 2D elements must fit
static __device__ __align__(256) uint8_t g_ctx_scratch[kCtxScratchBytes];

size_t context_kv_scratch_bytes(int L, int D, int dtype);

namespace {
PerContextOnce g_scratch_addr;

// Device address of g_ctx_scratch in the current device's context.
int ctx_scratch_address(void** out) {
  return g_scratch_addr.ensure(
      [](void** p) {
        const cudaError_t e = cudaGetSymbolAddress(p, g_ctx_scratch);
        if (e != cudaSuccess || !*p)
          return set_error(HSA_ECUDA, std::string("context_kv_noalloc: cudaGetSymbolAddress failed: ") +
                                          cudaGetErrorString(e));
        return (int)HSA_OK;
      },
      out);
}
}  // namespace

}  // namespace hsa

extern "C" size_t hsa_context_kv_noalloc_max_bytes(void) { return hsa::kCtxScratchBytes; }

extern "C" int hsa_context_kv_noalloc(const void* d_ctx, int L, int D, int dtype, const void* d_w_kv2,
                                      const float* d_b_kv2, const float* d_g_k2, void* d_k2, void* d_v2,
                                      void* stream) {
  using namespace hsa;
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "context_kv_noalloc: unknown dtype");
  if (L <= 0 || D <= 0) return set_error(HSA_EINVAL, "context_kv_noalloc: need L > 0 and D > 0");
  const size_t need = context_kv_scratch_bytes(L, D, dtype);
  if (need > kCtxScratchBytes)
    return set_error(HSA_EINVAL, "context_kv_noalloc: L x 2D elements of the dtype exceed the 8 MiB built-in "
                                 "scratch; use hsa_context_kv with a caller workspace");
  void* scratch = nullptr;
  const int rc = ctx_scratch_address(&scratch);
  if (rc != HSA_OK) return rc;
  // The projection writes every scratch element it later reads, so nothing needs clearing.
  return hsa_context_kv(d_ctx, L, D, dtype, d_w_kv2, d_b_kv2, d_g_k2, d_k2, d_v2, scratch, need, stream);
}

// runtime.h -- host-only declarations shared by the entry-point files of libhsa.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>
#include <utility>

#include "../../include/hsa.h"

namespace hsa {

int set_error(int code, const std::string& msg);
int check_launch(const char* what);
void count_launch(int n);
int num_sms();

// Identity of the current CUDA context, unique for the life of the process (cuCtxGetId): a
// device reset or a new primary context gives a new value.  0 when no context is current yet
// or the driver cannot say.
uint64_t current_context_id();

// Host set-up that must run once per CUDA context of a device -- a kernel attribute, the
// device address of a __device__ symbol -- shared by every host thread.  ensure(setup, &v)
// calls setup(&v) under a lock when the current device's context is not the one the last
// successful set-up ran in (after cudaDeviceReset, for instance), or when the context's
// identity cannot be read; otherwise it returns the value that set-up stored.
class PerContextOnce {
 public:
  template <typename F>
  int ensure(F&& setup, void** out = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
      return set_error(HSA_ECUDA, "no usable current CUDA device");
    const uint64_t id = current_context_id();
    std::lock_guard<std::mutex> g(mu_);
    if (id == 0 || ctx_[dev] != id) {
      void* v = nullptr;
      const int rc = setup(&v);
      if (rc != HSA_OK) return rc;
      ctx_[dev] = id;
      value_[dev] = v;
    }
    if (out) *out = value_[dev];
    return HSA_OK;
  }

 private:
  static constexpr int kMaxDevices = 64;
  std::mutex mu_;
  uint64_t ctx_[kMaxDevices] = {};
  void* value_[kMaxDevices] = {};
};

// 2-D tiled tensor map over a row-major matrix of `outer` rows x `inner` elements
// (bf16 or f32), rows `row_stride_bytes` apart, boxes of box_outer x box_inner.
int make_tmap_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                 uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128);
// Same with the 64-byte swizzle (boxes whose inner extent is 64 bytes).
int make_tmap_2d_sw64(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);

// Records a CUDA event pair around the launches made while it is alive, when
// timing is enabled (hsa_timing_enable); otherwise does nothing.
class ScopedTiming {
 public:
  ScopedTiming(int kclass, cudaStream_t st);
  ~ScopedTiming();
  ScopedTiming(const ScopedTiming&) = delete;
  ScopedTiming& operator=(const ScopedTiming&) = delete;

 private:
  int kclass_;
  cudaStream_t st_;
  cudaEvent_t a_ = nullptr;
};

// Launches `kernel` on `st` with programmatic stream serialization allowed, so its CTAs may
// be scheduled while the kernel ahead of it finishes (each kernel's pdl_prologue keeps the
// memory order).  A launch error is left for check_launch to report.
template <typename... P, typename... A>
void launch(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, A&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// The same with the grid in clusters of `cluster_x` CTAs (x only).
template <typename... P, typename... A>
void launch_cluster(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, unsigned cluster_x,
                    A&&... args) {
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace hsa

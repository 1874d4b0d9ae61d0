// runtime.cu -- host side of libhsa: error text, the device status word, launch
// counting, per-class kernel timing and TMA tensor-map encoding; plus the one-warp
// kernel behind hsa_selftest_wait_timeout, which checks the bounded-wait failure path.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "runtime.h"

namespace hsa {

static thread_local std::string t_last_error = "no error";
static std::atomic<uint64_t> g_launches{0};

int set_error(int code, const std::string& msg) {
  t_last_error = msg;
  return code;
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(HSA_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return HSA_OK;
}

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int num_sms() {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

uint64_t current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id);
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

static int make_tmap_2d_impl(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                             CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(HSA_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (!aligned16(base) || (row_stride_bytes & 15u))
    return set_error(HSA_EINVAL, "tensor map base and row stride must be 16-byte aligned");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d): dims %llu x %llu, box %u x %u", (int)r,
             (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
    return set_error(HSA_ECUDA, buf);
  }
  return HSA_OK;
}

int make_tmap_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                 uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  return make_tmap_2d_impl(map, base, bf16, inner, outer, row_stride_bytes, box_inner, box_outer,
                           swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

int make_tmap_2d_sw64(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  return make_tmap_2d_impl(map, base, bf16, inner, outer, row_stride_bytes, box_inner, box_outer,
                           CU_TENSOR_MAP_SWIZZLE_64B);
}

// ------------------------------------------------------------------ per-kernel timing
namespace {
struct TimingRec {
  cudaEvent_t a, b;
  int kclass;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

ScopedTiming::ScopedTiming(int kclass, cudaStream_t st) : kclass_(kclass), st_(st) {
  std::lock_guard<std::mutex> g(g_tmu);
  if (!g_timing) return;
  a_ = take_event();
  if (a_) cudaEventRecord(a_, st_);
}

ScopedTiming::~ScopedTiming() {
  if (!a_) return;
  std::lock_guard<std::mutex> g(g_tmu);
  cudaEvent_t b = take_event();
  if (!b) {
    g_pool.push_back(a_);
    return;
  }
  cudaEventRecord(b, st_);
  g_recs.push_back({a_, b, kclass_});
}

}  // namespace hsa

// ------------------------------------------------------------------ C ABI
extern "C" int hsa_timing_enable(int on) {
  std::lock_guard<std::mutex> g(hsa::g_tmu);
  hsa::g_timing = on != 0;
  return HSA_OK;
}

extern "C" int hsa_timing_read(int kclass, double* total_ms, int* launches) {
  if (kclass < 0 || kclass >= HSA_KCLASS_COUNT || !total_ms || !launches)
    return hsa::set_error(HSA_EINVAL, "timing_read: bad class or null output");
  std::lock_guard<std::mutex> g(hsa::g_tmu);
  double ms = 0.0;
  int n = 0;
  for (const auto& r : hsa::g_recs) {
    if (r.kclass != kclass) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return hsa::check_launch("timing_read: event sync");
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return hsa::check_launch("timing_read: elapsed");
    ms += t;
    ++n;
  }
  *total_ms = ms;
  *launches = n;
  return HSA_OK;
}

extern "C" int hsa_timing_reset(void) {
  std::lock_guard<std::mutex> g(hsa::g_tmu);
  for (auto& r : hsa::g_recs) {
    cudaEventSynchronize(r.b);
    hsa::g_pool.push_back(r.a);
    hsa::g_pool.push_back(r.b);
  }
  hsa::g_recs.clear();
  return HSA_OK;
}
extern "C" const char* hsa_last_error_string(void) { return hsa::t_last_error.c_str(); }

extern "C" uint64_t hsa_launch_count(void) { return hsa::g_launches.load(); }

// One warp waits on a shared-memory mbarrier that no thread ever arrives at: every lane's
// bounded wait gives up after kWaitLimitNs, the first one records HSA_ETIMEOUT and raises the
// abort flag, and the kernel returns.  Checks the failure path without a GPU fault.
__global__ void k_wait_never() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    hsa::mbar_init(&bar, 1);
    hsa::fence_mbar_init();
  }
  __syncthreads();
  (void)hsa::mbar_wait(&bar, 0);
}

extern "C" int hsa_selftest_wait_timeout(void* stream) {
  k_wait_never<<<1, 32, 0, hsa::as_stream(stream)>>>();
  hsa::count_launch(1);
  return hsa::check_launch("selftest wait launch");
}

extern "C" int hsa_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(hsa::as_stream(stream));
  if (e != cudaSuccess) return hsa::set_error(HSA_ECUDA, std::string("stream sync: ") + cudaGetErrorString(e));
  int status = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&status, hsa::g_hsa_status, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(hsa::g_hsa_status, &zero, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(hsa::g_hsa_abort, &zero, sizeof(int));
  if (e != cudaSuccess) return hsa::set_error(HSA_ECUDA, std::string("status word: ") + cudaGetErrorString(e));
  if (status == HSA_EINDEX) hsa::set_error(status, "a kernel met a token index outside [0, N)");
  if (status == HSA_ETIMEOUT) hsa::set_error(status, "a kernel's bounded pipeline wait ran out");
  return status;
}

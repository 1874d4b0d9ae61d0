// select.cu -- dynamic token selection (HSA summary §2.1): split the N tokens into
// K groups of fixed sizes by the L1 relative change of their velocity, so the
// slowest-changing tokens get the fewest denoising steps.
//
// Total order: (score descending, token index ascending); scores compare as
// float32 with NaN ranking as +inf and values <= 0 as 0.  Group k holds ranks
// [c_{k-1}, c_k) with c_k = n_1 + ... + n_k.  The result is unique, so the GPU
// output is compared bit for bit.
//
// One 1024-thread CTA (the work is a few passes over N floats):
//   1. for each boundary c_k (k < K): radix-select, over the 32-bit order key,
//      the element of rank c_k - 1 (4 passes of 8 bits with a shared-memory
//      histogram), then the right index among the equal keys by a block scan;
//   2. each token's group = number of boundaries it ranks at or after;
//   3. the groups' lists, each ascending by index, by per-thread chunk counts
//      and one block scan per group; group k starts at c_{k-1}.
#include "common.cuh"

namespace hsa {

constexpr int kSelectThreads = 1024;
constexpr int kMaxGroups = 16;

struct SelectArgs {
  int K;
  int cum[kMaxGroups + 1];  // cum[0] = 0, cum[k] = n_1 + ... + n_k
};

__device__ __forceinline__ uint32_t score_key(float s) {
  if (isnan(s)) return 0x7F800000u;
  if (!(s > 0.f)) return 0u;
  return __float_as_uint(s);
}

// Exclusive prefix sum over the block; *total gets the block sum.
__device__ int block_exclusive_scan(int v, int* total, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s - w;  // exclusive
    if (lane == 31) warp_sums[32] = s;
  }
  __syncthreads();
  const int out = warp_sums[warp] + x - v;
  *total = warp_sums[32];
  __syncthreads();
  return out;
}

__global__ void __launch_bounds__(kSelectThreads, 1)
    k_select(const float* __restrict__ score, int N, SelectArgs a, int8_t* __restrict__ group,
             int* __restrict__ order) {
  __shared__ uint32_t hist[256];
  __shared__ int warp_sums[33];
  __shared__ uint32_t s_thr_key[kMaxGroups];
  __shared__ int s_thr_idx[kMaxGroups];
  __shared__ uint32_t s_prefix;
  __shared__ int s_rank;

  const int tid = threadIdx.x;
  const int chunk = (N + kSelectThreads - 1) / kSelectThreads;
  const int lo = min(N, tid * chunk), hi = min(N, lo + chunk);

  // ---- 1. threshold element of every inner boundary
  for (int b = 1; b < a.K; ++b) {
    const int c = a.cum[b];
    if (c <= 0 || c >= N) continue;  // empty prefix or everything: no threshold needed
    // ascending order of ik = ~key is descending score order
    uint32_t prefix = 0, mask = 0;
    int rank = c - 1;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelectThreads) hist[i] = 0;
      __syncthreads();
      // warp-aggregated histogram: lanes with the same bin add once (scores share few
      // exponent bytes, so plain per-lane atomics would serialise on one address)
      const int lane = tid & 31;
      for (int base = 0; base < N; base += kSelectThreads) {
        const int n = base + tid;
        uint32_t bin = 256u + (uint32_t)lane;          // unique non-bin value when inactive
        if (n < N) {
          const uint32_t ik = ~score_key(score[n]);
          if ((ik & mask) == prefix) bin = (ik >> shift) & 255u;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
      }
      __syncthreads();
      if (tid == 0) {
        int r = rank, d = 0;
        for (; d < 255; ++d) {
          if (r < (int)hist[d]) break;
          r -= (int)hist[d];
        }
        s_prefix = prefix | ((uint32_t)d << shift);
        s_rank = r;
      }
      __syncthreads();
      prefix = s_prefix;
      rank = s_rank;
      mask |= 255u << shift;
      __syncthreads();
    }
    // the rank-th smallest token index among keys equal to the target
    int cnt = 0;
    for (int n = lo; n < hi; ++n) cnt += (~score_key(score[n]) == prefix);
    int total;
    const int excl = block_exclusive_scan(cnt, &total, warp_sums);
    if (rank >= excl && rank < excl + cnt) {
      int seen = excl;
      for (int n = lo; n < hi; ++n) {
        if (~score_key(score[n]) == prefix) {
          if (seen == rank) {
            s_thr_idx[b] = n;
            s_thr_key[b] = ~prefix;
            break;
          }
          ++seen;
        }
      }
    }
    __syncthreads();
  }

  // ---- 2. group of each token in this thread's chunk; local counts per group
  int cnt[kMaxGroups];
#pragma unroll
  for (int k = 0; k < kMaxGroups; ++k) cnt[k] = 0;
  for (int n = lo; n < hi; ++n) {
    const uint32_t key = score_key(score[n]);
    int g = 0;
    for (int b = 1; b < a.K; ++b) {
      const int c = a.cum[b];
      if (c <= 0) {
        ++g;
      } else if (c < N) {
        const uint32_t kt = s_thr_key[b];
        if (key < kt || (key == kt && n > s_thr_idx[b])) ++g;
      }
    }
    group[n] = (int8_t)g;
#pragma unroll
    for (int k = 0; k < kMaxGroups; ++k) cnt[k] += (g == k);
  }

  // ---- 3. ascending per-group lists, group k starting at cum[k]
  int off[kMaxGroups];
  for (int k = 0; k < a.K; ++k) {
    int total;
    off[k] = a.cum[k] + block_exclusive_scan(cnt[k], &total, warp_sums);
  }
  for (int n = lo; n < hi; ++n) {
    const int g = group[n];
#pragma unroll
    for (int k = 0; k < kMaxGroups; ++k)
      if (k == g) order[off[k]++] = n;
  }
}

}  // namespace hsa

extern "C" size_t hsa_select_tokens_workspace_size(int N, int K) {
  (void)N;
  (void)K;
  return 0;
}

extern "C" int hsa_select_tokens(const float* d_score, int N, int K, const int* h_group_sizes, int8_t* d_group,
                                 int32_t* d_order, void* d_ws, size_t ws_bytes, void* stream) {
  using namespace hsa;
  (void)d_ws;
  (void)ws_bytes;
  if (N < 0 || K < 1 || K > kMaxGroups || !h_group_sizes)
    return set_error(HSA_EINVAL, "select: need N >= 0 and 1 <= K <= 16 group sizes");
  if (N > 0 && (!d_score || !d_group || !d_order))
    return set_error(HSA_EINVAL, "select: null device pointer");
  SelectArgs a{};
  a.K = K;
  long long c = 0;
  for (int k = 0; k < K; ++k) {
    if (h_group_sizes[k] < 0) return set_error(HSA_EINVAL, "select: negative group size");
    c += h_group_sizes[k];
    a.cum[k + 1] = (int)c;
  }
  if (c != N) return set_error(HSA_EINVAL, "select: group sizes must sum to N");
  if (N == 0) return HSA_OK;
  ScopedTiming timing(HSA_KCLASS_OTHER, as_stream(stream));
  k_select<<<1, kSelectThreads, 0, as_stream(stream)>>>(d_score, N, a, d_group, d_order);
  count_launch(1);
  return check_launch("select launch");
}

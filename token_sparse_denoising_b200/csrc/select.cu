// select.cu -- dynamic token selection (HSA summary §2.1): split the N tokens into
// K groups of fixed sizes by the L1 relative change of their velocity, so the
// slowest-changing tokens get the fewest denoising steps.
//
// Total order: (score descending, token index ascending); scores compare as
// float32 with NaN ranking as +inf and values <= 0 as 0.  Optionally a set of
// pinned tokens (image-to-video: the conditioning frame's tokens) ranks ahead of
// every other token, pinned tokens among themselves by index, so they fill G_1
// first whatever their score.  Group k holds ranks
// [c_{k-1}, c_k) with c_k = n_1 + ... + n_k.  The result is unique, so the GPU
// output is compared bit for bit.
//
// One cluster of 8 CTAs of 1024 threads (one CTA below 4096 tokens, where the cluster's barriers
// cost more than they save).  CTA r of the cluster owns a contiguous range of token indices, and
// warp w of a CTA a contiguous sub-range:
//   1. for each boundary c_k (k < K): radix-select, over the 32-bit order key,
//      the element of rank c_k - 1 (4 passes of 8 bits; per-warp private
//      shared-memory histograms, since scores share few exponent bytes, summed
//      per CTA and then over the cluster through distributed shared memory, so
//      every CTA takes the same decision).  The top-digit pass is shared by all
//      boundaries, and each later pass serves two boundaries at once: their key
//      subsets are disjoint or identical, so one sweep fills both histograms.
//      Then the right index among the equal keys by a scan over the warps and the
//      CTAs; the CTA holding it publishes it to all;
//   2. each token's group = number of boundaries it ranks at or after;
//   3. the groups' lists, each ascending by index: each warp walks its range 32
//      consecutive indices at a time (bank-conflict-free shared-memory reads,
//      coalesced writes); per-group warp counts come from ballots, a scan over the
//      warps and one over the CTAs give each warp its offsets, and a lane's
//      position is the number of lower lanes in its group.  Group k starts at
//      c_{k-1}.
// Every CTA runs the same sequence of cluster barriers whatever the data, and the last
// one keeps every CTA's shared memory alive until its peers have read it.
// Up to 36864 keys per CTA are first staged in shared memory, so the passes do not wait
// on L2 latency for every element.
//
// Also here: k_active_rows, which builds A_i from the group lists when the active
// groups are not a prefix of the order (non-nested budgets).
#include "common.cuh"

namespace hsa {

constexpr int kSelectThreads = 1024;
constexpr int kSelectCluster = 8;          // CTAs per cluster from kSelectClusterMinN tokens on
constexpr int kSelectClusterMinN = 4096;   // below it one CTA (measured: N = 1024 13 us alone, 19 in a cluster)
constexpr int kMaxGroups = 16;

// Most keys one CTA stages in shared memory (4 bytes each, on top of ~70 KB of histograms);
// a CTA with a longer range reads the scores from global memory on every pass.
constexpr int kSelectStagedMax = 36864;

struct SelectArgs {
  int K;
  int staged;               // 1: each CTA's keys staged in dynamic shared memory
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

// One radix pass over the keys that match `prefix` on `mask`: histogram of the 8-bit
// digit at `shift` (per-warp private copies, then summed), and the digit holding the
// element of rank `rank` among them.  Returns (digit, rank within that digit) through
// shared memory.  Every thread of the block calls it.
// Inverted order key of token n (ascending = descending score): ~score_key, or 0 for a
// pinned token (score_key never exceeds 0x7F800000, so ~0xFFFFFFFF = 0 ranks before every
// score).  Read from the keys staged in shared memory when the kernel has them, else from
// the scores (and pin mask) in global memory.
__device__ __forceinline__ uint32_t inverted_key(const float* __restrict__ score, const uint8_t* __restrict__ pinned,
                                                 int n) {
  return (pinned && pinned[n]) ? 0u : ~score_key(score[n]);
}
struct KeySource {
  const float* __restrict__ score;
  const uint8_t* __restrict__ pinned;  // nullable
  const uint32_t* ikeys;               // shared memory (this CTA's range from index lo), or nullptr
  int lo;
  __device__ __forceinline__ uint32_t operator()(int n) const {
    return ikeys ? ikeys[n - lo] : inverted_key(score, pinned, n);
  }
};

constexpr int kHistStride = 513;   // per-warp histogram row: 2 x 256 bins, odd stride

// One warp finds, in bins[0, 256), the digit holding the element of rank `rank` and the rank within
// it: lane l owns bins [8l, 8l+8) (local sums, warp exclusive scan, the owning lane walks its bins).
__device__ __forceinline__ void scan_bins(const uint32_t* bins, int rank, int* out_digit, int* out_rank) {
  const int lane = threadIdx.x & 31;
  uint32_t v[8], s = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    v[e] = bins[8 * lane + e];
    s += v[e];
  }
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - s;
  if ((uint32_t)rank >= excl && (uint32_t)rank < incl) {
    uint32_t r = (uint32_t)rank - excl;
    int d = 0;
    for (; d < 7; ++d) {
      if (r < v[d]) break;
      r -= v[d];
    }
    *out_digit = 8 * lane + d;
    *out_rank = (int)r;
  }
}

// One radix pass for nt <= 2 targets t, each a (prefix, mask) of the keys already fixed and the rank
// sought among them: the histogram of the 8-bit digit at `shift` of every target's keys (per-warp
// private copies over this CTA's indices [lo, hi), summed into hpub, then summed over the cluster's
// CTAs into hist), then, by warp t, target t's digit and the rank within that digit.
// Two targets select either disjoint key sets (different prefixes: bins [0,256) and [256,512)) or the
// same one (equal prefix and mask: both read bins [0,256)), so one sweep over the keys serves both.
// Every thread of every CTA of the cluster calls it with the same targets; hist keeps the summed bins
// for the caller.  Consecutive passes alternate between two hpub buffers: the cluster barrier of
// the next pass keeps any CTA from rewriting a buffer its peers are still reading.  NT is a template
// parameter so the single-target pass carries no second-target test per key.
template <int NT>
__device__ void radix_pass2(KeySource key, int lo, int hi, const uint32_t* prefix, const uint32_t* mask,
                            const int* rank, int shift, uint32_t (*hw)[kHistStride], uint32_t* hpub,
                            uint32_t* hist, int* out_digit, int* out_rank) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int nt = NT;
  const bool shared_keys = NT == 2 && prefix[0] == prefix[1] && mask[0] == mask[1];
  const bool two = NT == 2 && !shared_keys;
  const int nbins = two ? 512 : 256;
  const uint32_t p0 = prefix[0], m0 = mask[0];
  const uint32_t p1 = two ? prefix[1] : 0u, m1 = two ? mask[1] : 0u;
  for (int i = lane; i < nbins; i += 32) hw[warp][i] = 0;
  __syncwarp();
  // Keys of similar scores share their top bytes, so most lanes of a warp often carry the
  // same bin: the lanes equal to lane 0's bin add with one atomic, the rest one each.
  for (int base = lo; base < hi; base += kSelectThreads) {
    const int n = base + tid;
    uint32_t bin = 0xFFFFu;                         // no contribution
    if (n < hi) {
      const uint32_t ik = key(n);
      if ((ik & m0) == p0) bin = (ik >> shift) & 255u;
      else if (two && (ik & m1) == p1) bin = 256u + ((ik >> shift) & 255u);
    }
    const uint32_t lead = __shfl_sync(0xffffffffu, bin, 0);
    const unsigned same = __ballot_sync(0xffffffffu, bin == lead);
    if (lane == 0 && lead != 0xFFFFu) atomicAdd(&hw[warp][lead], (uint32_t)__popc(same));
    if (bin != lead && bin != 0xFFFFu) atomicAdd(&hw[warp][bin], 1u);
  }
  __syncthreads();
  if (tid < nbins) {
    uint32_t t = 0;
#pragma unroll 8
    for (int w = 0; w < kSelectThreads / 32; ++w) t += hw[w][tid];
    hpub[tid] = t;
  }
  cluster_sync();
  if (tid < nbins) {
    uint32_t t = 0;
    const int nc = (int)cluster_size();
    for (int q = 0; q < nc; ++q) t += ld_peer(peer_smem(hpub + tid, (uint32_t)q));
    hist[tid] = t;
  }
  __syncthreads();
  if (warp < nt) scan_bins(hist + (two && warp == 1 ? 256 : 0), rank[warp], out_digit + warp, out_rank + warp);
  __syncthreads();
}

__global__ void __launch_bounds__(kSelectThreads, 1)
    k_select(const float* __restrict__ score, const uint8_t* __restrict__ pinned, int N, SelectArgs a,
             int8_t* __restrict__ group, int* __restrict__ order) {
  pdl_prologue();
  __shared__ uint32_t hist[512];
  __shared__ uint32_t hpub[2][512];                        // this CTA's pass histogram, for its peers
  __shared__ int warp_sums[33];
  __shared__ int s_wcnt[kMaxGroups][kSelectThreads / 32];   // per group, per warp: count, then offset
  __shared__ int s_tcnt[kMaxGroups];                        // per boundary: this CTA's matching keys
  __shared__ int s_gcnt[kMaxGroups];                        // per group: this CTA's tokens
  __shared__ uint32_t s_thr_key[kMaxGroups];
  __shared__ int s_thr_idx[kMaxGroups];
  __shared__ uint32_t s_pref[kMaxGroups], s_mask[kMaxGroups];   // per inner boundary (compacted list)
  __shared__ int s_rank[kMaxGroups], s_bnd[kMaxGroups];
  __shared__ int s_digit2[2], s_rank2[2];
  // dynamic shared memory: the per-warp private histograms, then this CTA's staged keys when the
  // launch provides them
  extern __shared__ uint32_t s_dyn[];
  uint32_t (*hw)[kHistStride] = reinterpret_cast<uint32_t (*)[kHistStride]>(s_dyn);
  uint32_t* s_ikeys = s_dyn + (kSelectThreads / 32) * kHistStride;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kSelectThreads / 32;
  const int r = (int)cluster_rank(), nc = (int)cluster_size();
  // CTA r owns indices [lo, hi), warp w [wlo, whi) within them: multiples of 32 per warp, walked
  // 32 consecutive at a time
  const int per_cta = ((N + nc * kWarps * 32 - 1) / (nc * kWarps * 32)) * kWarps * 32;
  const int lo = min(N, r * per_cta), hi = min(N, lo + per_cta);
  const int per_warp = per_cta / kWarps;
  const int wlo = min(hi, lo + warp * per_warp), whi = min(hi, wlo + per_warp);
  const unsigned lanes_below = (1u << lane) - 1u;
  KeySource key{score, pinned, nullptr, lo};
  if (a.staged) {
    for (int n = lo + tid; n < hi; n += kSelectThreads) s_ikeys[n - lo] = inverted_key(score, pinned, n);
    __syncthreads();
    key.ikeys = s_ikeys;
  }
  int pass = 0;                                            // alternates the hpub buffers

  // ---- 1. threshold element of every inner boundary.  Ascending order of ik = ~key is descending
  // score order; boundary c_b needs the element of rank c_b - 1.  Boundaries with c_b <= 0 or
  // c_b >= N need no threshold.
  int nb = 0;
  for (int b = 1; b < a.K; ++b) {
    const int c = a.cum[b];
    if (c > 0 && c < N) {
      if (tid == 0) {
        s_bnd[nb] = b;
        s_rank[nb] = c - 1;
        s_pref[nb] = 0u;
        s_mask[nb] = 0u;
      }
      ++nb;
    }
  }
  __syncthreads();
  if (nb > 0) {
    // top byte: one histogram serves every boundary
    radix_pass2<1>(key, lo, hi, s_pref, s_mask, s_rank, 24, hw, hpub[pass++ & 1], hist, s_digit2, s_rank2);
    if (warp == 0) {
      for (int i = 0; i < nb; ++i) {
        scan_bins(hist, s_rank[i], s_digit2, s_rank2);
        __syncwarp();
        if (lane == 0) {
          s_pref[i] = (uint32_t)s_digit2[0] << 24;
          s_mask[i] = 255u << 24;
          s_rank[i] = s_rank2[0];
        }
        __syncwarp();
      }
    }
    __syncthreads();
  }
  for (int i0 = 0; i0 < nb; i0 += 2) {
    const int nt = nb - i0 < 2 ? nb - i0 : 2;
    for (int shift = 16; shift >= 0; shift -= 8) {
      uint32_t* hp = hpub[pass++ & 1];
      if (nt == 2)
        radix_pass2<2>(key, lo, hi, s_pref + i0, s_mask + i0, s_rank + i0, shift, hw, hp, hist, s_digit2, s_rank2);
      else
        radix_pass2<1>(key, lo, hi, s_pref + i0, s_mask + i0, s_rank + i0, shift, hw, hp, hist, s_digit2, s_rank2);
      if (tid < nt) {
        s_pref[i0 + tid] |= (uint32_t)s_digit2[tid] << shift;
        s_mask[i0 + tid] |= 255u << shift;
        s_rank[i0 + tid] = s_rank2[tid];
      }
      __syncthreads();
    }
    for (int t = 0; t < nt; ++t) {
      const int i = i0 + t;
      const uint32_t prefix = s_pref[i];
      const int rank = s_rank[i], b = s_bnd[i];
      // the rank-th smallest token index among keys equal to the target: per-warp counts of
      // matches, scans over the warps and over the CTAs, then the warp holding that rank finds the
      // lane and hands the threshold to every CTA of the cluster
      int cnt = 0;
      for (int base = wlo; base < whi; base += 32) {
        const int n = base + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, n < whi && key(n) == prefix));
      }
      if (lane == 0) warp_sums[warp] = cnt;
      __syncthreads();
      if (warp == 0) {
        const int v = warp_sums[lane];
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        warp_sums[lane] = incl - v;
        if (lane == 31) s_tcnt[i] = incl;                  // this CTA's matches
      }
      cluster_sync();
      int cta_excl = 0;
      for (int q = 0; q < r; ++q) cta_excl += (int)ld_peer(peer_smem(s_tcnt + i, (uint32_t)q));
      const int excl = cta_excl + warp_sums[warp];
      if (rank >= excl && rank < excl + cnt) {      // warp-uniform
        int seen = excl;
        for (int base = wlo; base < whi; base += 32) {
          const int n = base + lane;
          const bool m = n < whi && key(n) == prefix;
          const unsigned mk = __ballot_sync(0xffffffffu, m);
          if (rank < seen + __popc(mk)) {
            if (m && seen + __popc(mk & lanes_below) == rank) {
              for (int q = 0; q < nc; ++q) {
                st_peer(peer_smem(s_thr_idx + b, (uint32_t)q), (uint32_t)n);
                st_peer(peer_smem(s_thr_key + b, (uint32_t)q), ~prefix);
              }
            }
            break;
          }
          seen += __popc(mk);
        }
      }
      cluster_sync();
    }
  }

  // ---- 2. group of each token; per-warp counts per group.  Loops over groups are unrolled to
  // kMaxGroups with a K guard, so the counters stay in registers (warp-uniform values).
  int cnt[kMaxGroups];
#pragma unroll
  for (int k = 0; k < kMaxGroups; ++k) cnt[k] = 0;
  for (int base = wlo; base < whi; base += 32) {
    const int n = base + lane;
    const bool valid = n < whi;
    int g = -1;
    if (valid) {
      const uint32_t kn = ~key(n);
      g = 0;
#pragma unroll
      for (int b = 1; b < kMaxGroups; ++b) {
        if (b < a.K) {
          const int c = a.cum[b];
          if (c <= 0) {
            ++g;
          } else if (c < N) {
            const uint32_t kt = s_thr_key[b];
            if (kn < kt || (kn == kt && n > s_thr_idx[b])) ++g;
          }
        }
      }
      group[n] = (int8_t)g;
      if (key.ikeys) s_ikeys[n - lo] = (uint32_t)g;   // this lane's own slot: it now holds the group
    }
#pragma unroll
    for (int k = 0; k < kMaxGroups; ++k)
      if (k < a.K) cnt[k] += __popc(__ballot_sync(0xffffffffu, g == k));
  }
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < kMaxGroups; ++k)
      if (k < a.K) s_wcnt[k][warp] = cnt[k];
  }
  __syncthreads();
  // ---- 3. offsets: warp k scans group k's counts over the warps (ascending index ranges), then
  // adds the counts of the CTAs with lower index ranges
  int incl_k = 0, v_k = 0;
  if (warp < a.K) {
    v_k = s_wcnt[warp][lane];
    incl_k = v_k;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl_k, o);
      if (lane >= o) incl_k += y;
    }
    if (lane == 31) s_gcnt[warp] = incl_k;               // this CTA's tokens of group `warp`
  }
  cluster_sync();
  if (warp < a.K) {
    int cta_off = 0;
    for (int q = 0; q < r; ++q) cta_off += (int)ld_peer(peer_smem(s_gcnt + warp, (uint32_t)q));
    s_wcnt[warp][lane] = a.cum[warp] + cta_off + incl_k - v_k;
  }
  __syncthreads();
  int off[kMaxGroups];
#pragma unroll
  for (int k = 0; k < kMaxGroups; ++k) off[k] = (k < a.K) ? s_wcnt[k][warp] : 0;
  for (int base = wlo; base < whi; base += 32) {
    const int n = base + lane;
    const int g = n < whi ? (key.ikeys ? (int)s_ikeys[n - lo] : (int)group[n]) : -1;
#pragma unroll
    for (int k = 0; k < kMaxGroups; ++k) {
      if (k < a.K) {
        const unsigned mk = __ballot_sync(0xffffffffu, g == k);
        if (g == k) order[off[k] + __popc(mk & lanes_below)] = n;
        off[k] += __popc(mk);
      }
    }
  }
  // no CTA leaves while a peer may still read its shared memory
  cluster_sync();
}

}  // namespace hsa

extern "C" size_t hsa_select_tokens_workspace_size(int N, int K) {
  (void)N;
  (void)K;
  return 0;
}

extern "C" int hsa_select_tokens_pinned(const float* d_score, const uint8_t* d_pinned, int N, int K,
                                        const int* h_group_sizes, int8_t* d_group, int32_t* d_order, void* d_ws,
                                        size_t ws_bytes, void* stream) {
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
  // cluster size, and each CTA's index range as the kernel computes it
  const int nc = N < kSelectClusterMinN ? 1 : kSelectCluster;
  const int per_cta = (N + nc * kSelectThreads - 1) / (nc * kSelectThreads) * kSelectThreads;
  a.staged = per_cta <= kSelectStagedMax ? 1 : 0;
  constexpr size_t kHistBytes = (size_t)(kSelectThreads / 32) * kHistStride * sizeof(uint32_t);
  const size_t dyn = kHistBytes + (a.staged ? (size_t)per_cta * sizeof(uint32_t) : 0);
  static PerContextOnce attr;
  const int arc = attr.ensure([](void**) {
    if (cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kHistBytes + kSelectStagedMax * (int)sizeof(uint32_t)) != cudaSuccess)
      return check_launch("select: shared-memory attribute");
    return (int)HSA_OK;
  });
  if (arc) return arc;
  ScopedTiming timing(HSA_KCLASS_OTHER, as_stream(stream));
  if (nc == 1)   // a lone CTA is a cluster of one: its cluster barriers and peer accesses stay in the CTA
    launch(k_select, 1, kSelectThreads, dyn, as_stream(stream), d_score, d_pinned, N, a, d_group, d_order);
  else
    launch_cluster(k_select, nc, kSelectThreads, dyn, as_stream(stream), (unsigned)nc, d_score, d_pinned, N, a,
                   d_group, d_order);
  count_launch(1);
  return check_launch("select launch");
}

extern "C" int hsa_select_tokens(const float* d_score, int N, int K, const int* h_group_sizes, int8_t* d_group,
                                 int32_t* d_order, void* d_ws, size_t ws_bytes, void* stream) {
  return hsa_select_tokens_pinned(d_score, nullptr, N, K, h_group_sizes, d_group, d_order, d_ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ A_i from the group lists (§2.1)
namespace hsa {
struct RowSegments {
  int n;                                   // active groups
  int src[kMaxGroups], dst[kMaxGroups + 1];  // start in order / in A_i; dst[n] = M
};

// A_i = the active groups' lists of `order`, concatenated in group order.  Grid-stride over the
// M output positions; each finds its segment among at most 16.
__global__ void __launch_bounds__(256) k_active_rows(const int32_t* __restrict__ order, RowSegments seg,
                                                     int32_t* __restrict__ idx) {
  pdl_prologue();
  const int M = seg.dst[seg.n];
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < M; r += gridDim.x * blockDim.x) {
    int k = 0;
    while (k + 1 < seg.n && r >= seg.dst[k + 1]) ++k;
    idx[r] = order[seg.src[k] + (r - seg.dst[k])];
  }
}
}  // namespace hsa

extern "C" int hsa_active_rows(const int32_t* d_order, int N, int K, const int* h_group_sizes,
                               const uint8_t* h_active, int32_t* d_idx, int* h_M, void* stream) {
  using namespace hsa;
  if (N < 0 || K < 1 || K > kMaxGroups || !h_group_sizes || !h_active)
    return set_error(HSA_EINVAL, "active_rows: need N >= 0, 1 <= K <= 16, group sizes and the active mask");
  RowSegments seg{};
  long long start = 0;
  int pos = 0;
  for (int k = 0; k < K; ++k) {
    if (h_group_sizes[k] < 0) return set_error(HSA_EINVAL, "active_rows: negative group size");
    if (h_active[k] && h_group_sizes[k] > 0) {
      seg.src[seg.n] = (int)start;
      seg.dst[seg.n] = pos;
      ++seg.n;
      pos += h_group_sizes[k];
    }
    start += h_group_sizes[k];
  }
  if (start != N) return set_error(HSA_EINVAL, "active_rows: group sizes must sum to N");
  seg.dst[seg.n] = pos;
  if (h_M) *h_M = pos;
  if (pos == 0) return HSA_OK;
  if (!d_order || !d_idx) return set_error(HSA_EINVAL, "active_rows: null device pointer");
  const int blocks = (pos + 255) / 256 < 4 * num_sms() ? (pos + 255) / 256 : 4 * num_sms();
  launch(k_active_rows, blocks, 256, 0, as_stream(stream), d_order, seg, d_idx);
  count_launch(1);
  return check_launch("active_rows launch");
}

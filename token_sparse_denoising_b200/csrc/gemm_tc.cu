// gemm_tc.cu -- bf16 GEMM on the 5th-generation tensor cores for the linear
// layers of the HSA block on the compacted active rows (HSA summary §2.2: only
// A_i runs the projections and the feed-forward).
//
//   y[M x Nout] = epilogue(x[M x K] * W[Nout x K]^T + b)
//
// Two kernels share the epilogue (store_chunk):
//   k_gemm_pair  outputs 256-column multiples with more than 128 rows (every GEMM of the block):
//                a cluster of two CTAs on two SMs computes 256 x 256 tiles with one stream of
//                tcgen05.mma.cta_group::2 issued by CTA 0; each CTA loads its own 128 rows of A and
//                128 of the 256 weight rows per k-block, so each SM moves half the weight bytes per
//                FLOP (details above the kernel);
//   k_gemm_tc    everything else: one CTA per 128 x BN tile.
// Both are persistent (one CTA, or pair, per SM walks the output tiles).  Warp roles:
//   warp 0      TMA producer: A (128 x 64) and B (BN x 64, or 128 x 64 per CTA of a pair)
//               k-blocks into a ring of shared-memory slots, 128-byte swizzled;
//   warp 1      allocates the TMEM accumulators (two, so the epilogue of one tile overlaps the
//               mainloop of the next); the warp runs the loop converged and one elected lane
//               issues tcgen05.mma (M=128 or 256, N=BN, K=16) and releases each shared-memory
//               slot with tcgen05.commit;
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane quarter, bias, GELU / residual gate.
//               Thread = output row.  Each warp stages 32 x 32 sub-tiles of the output in shared
//               memory and hands them to the TMA: bf16 and fp32 outputs by tensor stores, the
//               fp32 residual update y += gate * (acc + b) by a tensor reduce-add done in L2, so
//               the epilogue never waits on a global load.
// Rows beyond M are zero-filled by TMA and never stored.  No load is multicast.
#include "tcgen05.cuh"

namespace hsa {

enum : int { EPI_STORE = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_F32 = 3 };

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmThreads = 192;

template <int BN>
struct GemmCfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;   // 16 KB
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // epilogue staging: 4 warps x 2 buffers x one 32 x 32 sub-tile (fp32: 4 KB; bf16 uses 2 KB of it)
  static constexpr int kStageOutBytes = 4 * 2 * 4096;
  static constexpr int kSmem = kStages * kStageBytes + kStageOutBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(2 * BN <= 512, "double-buffered accumulator must fit TMEM");
  static_assert(kSmem <= 232448, "GEMM shared memory above the 227 KB per-CTA limit");
};

// GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).  The tanh is the hardware
// tanh.approx.f32 (one MUFU op, relative error about 2^-11); the result is rounded to bf16, whose
// step is 2^-8 relative, so the approximation is below the output's own rounding.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
  const float hx = 0.5f * x;
  return fmaf(hx, tanh_approx(u), hx);
}

// Epilogue of one 32 x 32 output sub-tile held by a warp (lane = row, r = its 32 accumulator
// columns): bias, GELU or residual gate, staged in shared memory (sb, one of the warp's two
// buffers) and handed to the TMA: a tensor store, or for the fp32 residual update y += gate (acc +
// b) a tensor reduce-add done in L2.  Rows beyond M are clipped by the tensor map.
template <int EPI>
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], uint8_t* sb, int lane, int col0, int row0,
                                            const float* __restrict__ bias, const float* __restrict__ gate,
                                            const CUtensorMap* tmY) {
  constexpr bool kF32Out = (EPI == EPI_RESID || EPI == EPI_F32);
  if (lane == 0) bulk_wait_group_read<1>();   // the copy that last read sb is done
  __syncwarp();
  if constexpr (kF32Out) {
    // fp32 rows of 128 bytes, 128-byte swizzle: chunk k of row r at k ^ (r & 7)
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      v[j] = __uint_as_float(r[j]) + (bias ? __ldg(bias + col0 + j) : 0.f);
      if (EPI == EPI_RESID && gate) v[j] *= __ldg(gate + col0 + j);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
      *reinterpret_cast<float4*>(sb + lane * 128 + ((k ^ (lane & 7)) << 4)) =
          make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  } else {
    // bf16 rows of 64 bytes, 64-byte swizzle: chunk k of row r at k ^ ((r >> 1) & 3)
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float v0 = __uint_as_float(r[2 * j]) + (bias ? __ldg(bias + col0 + 2 * j) : 0.f);
      float v1 = __uint_as_float(r[2 * j + 1]) + (bias ? __ldg(bias + col0 + 2 * j + 1) : 0.f);
      if (EPI == EPI_GELU) {
        v0 = gelu_tanh_f(v0);
        v1 = gelu_tanh_f(v1);
      }
      w[j] = pack_bf16x2(v0, v1);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<uint4*>(sb + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)) =
          make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if constexpr (EPI == EPI_RESID)
      tma_reduce_add_2d(tmY, sb, col0, row0);
    else
      tma_store_2d(tmY, sb, col0, row0);
    bulk_commit_group();
  }
}

// Persistent: CTA c handles output tiles c, c + gridDim.x, ... (n fastest, so the
// CTAs running together share A row-tiles and the weights stay in L2).  The TMEM
// accumulator is double-buffered (2 x BN columns): the epilogue of one tile runs
// while the MMA warp accumulates the next.
template <int BN, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmY, int M, int Nout, int K, const float* __restrict__ bias,
              const float* __restrict__ gate, void* __restrict__ out) {
  pdl_prologue();
  using Cfg = GemmCfg<BN>;
  constexpr int S = Cfg::kStages;
  constexpr bool kF32Out = (EPI == EPI_RESID || EPI == EPI_F32);
  constexpr int kChunkBytes = kF32Out ? 4096 : 2048;   // one staged 32 x 32 output sub-tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_out = smem + S * Cfg::kStageBytes;   // 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(stage_out + Cfg::kStageOutBytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;     // [2]
  uint64_t* acc_empty = acc_full + 2; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = K / kGemmBK;
  const int n_tiles = Nout / BN;
  const int tiles = n_tiles * ((M + kGemmBM - 1) / kGemmBM);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t keep = policy_evict_last();   // weights are re-read by every row tile
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int n0 = (t % n_tiles) * BN, m0 = (t / n_tiles) * kGemmBM;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) { ok = false; break; }
          uint8_t* a = smem + s * Cfg::kStageBytes;
          mbar_expect_tx(&full[s], Cfg::kStageBytes);
          tma_load_2d(a, &tmA, &full[s], kb * kGemmBK, m0);
          tma_load_2d_hint(a + Cfg::kABytes, &tmB, &full[s], kb * kGemmBK, n0, keep);
        }
      }
    }
  } else if (warp == 1) {
    // the whole warp runs the loop and waits (warp-uniform values); one elected lane issues.
    // Against a loop run by lane 0 alone: QKV 0.342 -> 0.335 ms, FFN1 0.692-0.713 -> 0.667-0.690,
    // FFN2 0.722-0.769 -> 0.701-0.727, O-projection 0.179-0.183 -> 0.174-0.178 (outputs identical).
    {
      const bool leader = elect_one();
      constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, BN, false);
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tc) {
        const int buf = tc & 1;
        if (!__shfl_sync(0xffffffffu, mbar_wait(&acc_empty[buf], ((tc >> 1) & 1) ^ 1), 0)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          if (!__shfl_sync(0xffffffffu, mbar_wait(&full[s], (it / S) & 1), 0)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * Cfg::kStageBytes);
          const uint32_t b = a + Cfg::kABytes;
          if (leader) {
#pragma unroll
            for (int k = 0; k < kGemmBK / 16; ++k)
              umma_ss(acc, sdesc_sw128(a + 32 * k, 16, 1024), sdesc_sw128(b + 32 * k, 16, 1024), idesc,
                      (kb | k) != 0);
            umma_commit(&empty[s]);
          }
          __syncwarp();
        }
        if (leader) umma_commit(&acc_full[buf]);
        __syncwarp();
      }
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows of that quarter
    const int quarter = warp & 3;
    uint8_t* my_out = stage_out + (warp - 2) * 2 * kChunkBytes;   // this warp's two sub-tile buffers
    int tc = 0, nchunk = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
      const int n0 = (t % n_tiles) * BN, m0 = (t / n_tiles) * kGemmBM;
      const int buf = tc & 1;
      const bool ok = mbar_wait(&acc_full[buf], (tc >> 1) & 1);
      __syncwarp();
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c, ++nchunk) {
        uint32_t r[32];
        __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the guarded stores
        tmem_ld32(base + (uint32_t)(c * 32), r);
        tmem_ld_wait();
        if (c == BN / 32 - 1) {  // accumulator fully read: the MMA warp may reuse it
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
        }
        store_chunk<EPI>(r, my_out + (nchunk & 1) * kChunkBytes, lane, n0 + c * 32, m0 + quarter * 32, bias, gate,
                         &tmY);
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// ------------------------------------------------------------------ pair variant (cta_group::2)
// A cluster of two CTAs computes 256 x 256 output tiles with one stream of tcgen05 MMAs (M = 256,
// N = 256, K = 16) issued by CTA 0.  Per 64-deep k-block, CTA r loads rows [m0 + 128 r, +128) of A
// and weight rows [n0 + 128 r, +128) of B into its own shared memory: each CTA moves half the
// weight bytes that a 128 x 256 tile of one CTA needs, and one MMA instruction covers both SMs.
// Each CTA's TMEM holds its 128 rows x 256 columns of the accumulator (double-buffered, 512
// columns), and each CTA's epilogue writes its own rows.  Barriers:
//   full[s]       CTA 0's counts the pair's bytes: CTA 0's producer arms it with both CTAs' bytes,
//                 and both CTAs' loads complete on it (CTA 1's through its cluster address);
//   empty[s]      in both CTAs, signalled by CTA 0's commit (multicast to the pair);
//   acc_full[b]   in both CTAs, the same way;
//   acc_empty[b]  CTA 0's, one arrival per epilogue warp of either CTA (8).
// No load is multicast: each CTA reads only its own rows of A and B.
struct GemmPairCfg {
  static constexpr int kStages = 6;
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;   // 16 KB: this CTA's 128 rows of A
  static constexpr int kBBytes = 128 * kGemmBK * 2;       // 16 KB: this CTA's 128 weight rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStageOutBytes = 4 * 2 * 4096;
  static constexpr int kSmem = kStages * kStageBytes + kStageOutBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kSmem <= 232448, "GEMM shared memory above the 227 KB per-CTA limit");
};

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, int M, int Nout, int K, const float* __restrict__ bias,
                const float* __restrict__ gate, void* __restrict__ out) {
  pdl_prologue();
  using Cfg = GemmPairCfg;
  constexpr int S = Cfg::kStages, BN = 256;
  constexpr bool kF32Out = (EPI == EPI_RESID || EPI == EPI_F32);
  constexpr int kChunkBytes = kF32Out ? 4096 : 2048;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_out = smem + S * Cfg::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(stage_out + Cfg::kStageOutBytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;     // [2]
  uint64_t* acc_empty = acc_full + 2; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const uint32_t rank = cluster_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = K / kGemmBK;
  const int n_tiles = Nout / BN;
  const int tiles = n_tiles * ((M + 2 * kGemmBM - 1) / (2 * kGemmBM));
  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);
    }
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * BN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers exist before any load or arrival crosses the pair
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t keep = policy_evict_last();   // weights are re-read by every row tile
      const uint32_t full0 = peer_smem(full, 0);   // CTA 0's full[0]; full[s] is 8 s bytes on
      int it = 0;
      bool ok = true;
      for (int t = pair; ok && t < tiles; t += npairs) {
        const int n0 = (t % n_tiles) * BN + (int)rank * 128, m0 = (t / n_tiles) * 2 * kGemmBM + (int)rank * kGemmBM;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) { ok = false; break; }
          uint8_t* a = smem + s * Cfg::kStageBytes;
          if (rank == 0) mbar_expect_tx(&full[s], 2 * Cfg::kStageBytes);
          tma_load_2d_pair(a, &tmA, full0 + 8u * (uint32_t)s, kb * kGemmBK, m0);
          tma_load_2d_pair_hint(a + Cfg::kABytes, &tmB, full0 + 8u * (uint32_t)s, kb * kGemmBK, n0, keep);
        }
      }
      // the last commits of CTA 0 arrive on this CTA's empty barriers: wait for them before exit
      for (int j = it - S < 0 ? 0 : it - S; ok && j < it; ++j) ok = mbar_wait(&empty[j % S], (j / S) & 1);
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // the whole warp runs the loop and waits (warp-uniform values); one elected lane issues
      const bool leader = elect_one();
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kGemmBM, BN, false);
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = pair; ok && t < tiles; t += npairs, ++tc) {
        const int buf = tc & 1;
        if (!__shfl_sync(0xffffffffu, mbar_wait(&acc_empty[buf], ((tc >> 1) & 1) ^ 1), 0)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          if (!__shfl_sync(0xffffffffu, mbar_wait(&full[s], (it / S) & 1), 0)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * Cfg::kStageBytes);
          const uint32_t b = a + Cfg::kABytes;
          if (leader) {
#pragma unroll
            for (int k = 0; k < kGemmBK / 16; ++k)
              umma_ss_pair(acc, sdesc_sw128(a + 32 * k, 16, 1024), sdesc_sw128(b + 32 * k, 16, 1024), idesc,
                           (kb | k) != 0);
            umma_commit_pair(&empty[s], 3);
          }
          __syncwarp();
        }
        if (leader) umma_commit_pair(&acc_full[buf], 3);
        __syncwarp();
      }
    }
  } else {
    // epilogue of this CTA's 128 rows: warp w reads TMEM lanes 32*(w%4) .. +31
    const int quarter = warp & 3;
    uint8_t* my_out = stage_out + (warp - 2) * 2 * kChunkBytes;
    const uint32_t acc_empty0 = peer_smem(acc_empty, 0);   // CTA 0's acc_empty[0]; [b] is 8 b bytes on
    int tc = 0, nchunk = 0;
    for (int t = pair; t < tiles; t += npairs, ++tc) {
      const int n0 = (t % n_tiles) * BN, m0 = (t / n_tiles) * 2 * kGemmBM + (int)rank * kGemmBM;
      const int buf = tc & 1;
      const bool ok = mbar_wait(&acc_full[buf], (tc >> 1) & 1);
      __syncwarp();
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c, ++nchunk) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(base + (uint32_t)(c * 32), r);
        tmem_ld_wait();
        if (c == BN / 32 - 1) {  // this warp's rows of the accumulator are read: CTA 0 may reuse it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * (uint32_t)buf);
        }
        store_chunk<EPI>(r, my_out + (nchunk & 1) * kChunkBytes, lane, n0 + c * 32, m0 + quarter * 32, bias, gate,
                         &tmY);
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // neither CTA leaves while the pair's MMAs or arrivals may still reach it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 2 * BN);
  }
}

template <int BN, int EPI>
static int launch_gemm_bn(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty, int M, int Nout,
                          int K, const float* bias, const float* gate, void* out, cudaStream_t st) {
  auto kern = k_gemm_tc<BN, EPI>;
  static PerContextOnce attr;
  const int arc = attr.ensure([&](void**) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<BN>::kSmem) != cudaSuccess)
      return check_launch("gemm: shared-memory attribute");
    return (int)HSA_OK;
  });
  if (arc) return arc;
  const int tiles = (Nout / BN) * ((M + kGemmBM - 1) / kGemmBM);
  dim3 grid(tiles < num_sms() ? tiles : num_sms());
  ScopedTiming timing(HSA_KCLASS_GEMM, st);
  launch(kern, grid, kGemmThreads, GemmCfg<BN>::kSmem, st, ta, tb, ty, M, Nout, K, bias, gate, out);
  count_launch(1);
  return check_launch("gemm_tc launch");
}

template <int EPI>
static int launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty, int M, int Nout,
                            int K, const float* bias, const float* gate, void* out, cudaStream_t st) {
  auto kern = k_gemm_pair<EPI>;
  // per context: the shared-memory attribute, and how many clusters of two fit at once
  static PerContextOnce attr;
  void* fit = nullptr;
  const int arc = attr.ensure([&](void** v) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmPairCfg::kSmem) != cudaSuccess)
      return check_launch("gemm (pair): shared-memory attribute");
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * num_sms());
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = GemmPairCfg::kSmem;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1)
      return check_launch("gemm (pair): cluster occupancy");
    *v = reinterpret_cast<void*>(static_cast<intptr_t>(n));
    return (int)HSA_OK;
  }, &fit);
  if (arc) return arc;
  const int pairs_fit = static_cast<int>(reinterpret_cast<intptr_t>(fit));
  const int tiles = (Nout / 256) * ((M + 2 * kGemmBM - 1) / (2 * kGemmBM));
  const int pairs = tiles < pairs_fit ? tiles : pairs_fit;
  ScopedTiming timing(HSA_KCLASS_GEMM, st);
  launch_cluster(kern, dim3(2 * pairs), dim3(kGemmThreads), GemmPairCfg::kSmem, st, 2u, ta, tb, ty, M, Nout, K, bias,
                 gate, out);
  count_launch(1);
  return check_launch("gemm_tc (pair) launch");
}

template <int EPI>
static int launch_gemm_epi(const void* A, int M, int K, const void* W, int Nout, const float* bias,
                           const float* gate, void* out, cudaStream_t st) {
  const int BN = (Nout % 256 == 0) ? 256 : (Nout % 128 == 0 ? 128 : 64);
  CUtensorMap ta, tb;
  int rc = make_tmap_2d(&ta, A, true, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, kGemmBK, kGemmBM, true);
  if (rc) return rc;
  rc = make_tmap_2d(&tb, W, true, (uint64_t)K, (uint64_t)Nout, (uint64_t)K * 2, kGemmBK, (uint32_t)BN, true);
  if (rc) return rc;
  CUtensorMap ty;   // the output, in 32 x 32 boxes: bf16 with 64-byte swizzle, fp32 with 128-byte swizzle
  if (EPI == EPI_STORE || EPI == EPI_GELU)
    rc = make_tmap_2d_sw64(&ty, out, true, (uint64_t)Nout, (uint64_t)M, (uint64_t)Nout * 2, 32, 32);
  else
    rc = make_tmap_2d(&ty, out, false, (uint64_t)Nout, (uint64_t)M, (uint64_t)Nout * 4, 32, 32, true);
  if (rc) return rc;
  if (BN == 256 && M > kGemmBM) {
    // pair tiles of 256 x 256 over two SMs (cta_group::2): each CTA loads 128 of the 256 weight rows
    CUtensorMap tb2;
    rc = make_tmap_2d(&tb2, W, true, (uint64_t)K, (uint64_t)Nout, (uint64_t)K * 2, kGemmBK, 128, true);
    if (rc) return rc;
    return launch_gemm_pair<EPI>(ta, tb2, ty, M, Nout, K, bias, gate, out, st);
  }
  if (BN == 256) return launch_gemm_bn<256, EPI>(ta, tb, ty, M, Nout, K, bias, gate, out, st);
  if (BN == 128) return launch_gemm_bn<128, EPI>(ta, tb, ty, M, Nout, K, bias, gate, out, st);
  return launch_gemm_bn<64, EPI>(ta, tb, ty, M, Nout, K, bias, gate, out, st);
}

// Host entry used by every bf16 linear layer.  Shapes are validated here.
int gemm_bf16(const void* A, int M, int K, const void* W, int Nout, const float* bias, int epi, const float* gate,
              void* out, cudaStream_t st) {
  if (M <= 0) return HSA_OK;
  if (K <= 0 || K % kGemmBK || Nout <= 0 || Nout % 64)
    return set_error(HSA_EINVAL, "bf16 linear: need K % 64 == 0 and Nout % 64 == 0");
  if (!A || !W || !out || !aligned16(A) || !aligned16(W) || !aligned16(out))
    return set_error(HSA_EINVAL, "bf16 linear: null or misaligned pointer");
  switch (epi) {
    case EPI_STORE: return launch_gemm_epi<EPI_STORE>(A, M, K, W, Nout, bias, gate, out, st);
    case EPI_GELU: return launch_gemm_epi<EPI_GELU>(A, M, K, W, Nout, bias, gate, out, st);
    case EPI_RESID: return launch_gemm_epi<EPI_RESID>(A, M, K, W, Nout, bias, gate, out, st);
    case EPI_F32: return launch_gemm_epi<EPI_F32>(A, M, K, W, Nout, bias, gate, out, st);
  }
  return set_error(HSA_EINVAL, "linear: unknown epilogue");
}

}  // namespace hsa

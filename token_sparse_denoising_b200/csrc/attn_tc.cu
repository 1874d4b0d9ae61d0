// attn_tc.cu -- full-context attention of the active queries against the whole
// per-layer KV cache on the 5th-generation tensor cores (HSA summary §2.2:
// active tokens query the complete cached K, V -- fresh rows for active tokens,
// stale but valid rows for skipped ones -- at O(|A_i| N) cost).
//
//   o = softmax(q K^T / sqrt(128)) V, per head; q: M x 128H compacted rows,
//   K, V: L x 128H cache rows, o: M x 128H.  Non-causal.
//
// One CTA = one head x 128 queries, streaming 128-key tiles of K and V.
//   warp 0      TMA producer: Q once; K_j into a 3-slot ring, V_j into a 2-slot ring
//   warp 1      TMEM owner (512 columns) and MMA issuer:
//                 S_j = Q K_j^T        (SS: both K-major, 128 x 128 x 128)
//                 O  += P_j V_j        (TS: P from TMEM, V MN-major)
//               S_{j+1} is issued before waiting for P_j, so QK^T of the next
//               tile overlaps the softmax of this one.
//   warps 2..9  softmax: two threads per query row, each owning 64 of the 128 key
//               columns of a tile (warps 2-5 the left half, 6-9 the right half;
//               warp w reads TMEM lane quarter w % 4).  The two halves of a row
//               agree on the row max through shared memory and a named barrier per
//               lane quarter.  p = 2^(t - m) goes back to TMEM as bf16.  O is
//               rescaled in TMEM only when the max grew by more than 2^8
//               (otherwise the stale max keeps p <= 256, safe in fp32).
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P0 [384,448) P1 [448,512).
// Key rows beyond L are zero-filled by TMA and masked to -inf; query rows beyond
// M are computed on zeros and never stored.
#include "tcgen05.cuh"

namespace hsa {

constexpr int kAttnBM = 128;
constexpr int kAttnBN = 128;
constexpr int kKSlots = 3;
constexpr int kVSlots = 2;
constexpr int kAttnThreads = 320;                 // 2 control warps + 8 softmax warps
constexpr int kTileBytes = 128 * 128 * 2;         // one 128 x 128 bf16 operand tile (two 64-column boxes)
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
// Exponentials computed with the polynomial instead of the MUFU unit: the columns c
// of a thread's 64 with (c % 8) >= 8 - kPolyPer8.  Measured at the Wan-1.3B shape
// (attention alone, 32760 x 32760, 12 heads): 0 of 8 -> 6.44 ms, 2 of 8 -> 7.04 ms,
// 4 of 8 -> 7.63 ms, so the MUFU path alone is the default.
#ifndef HSA_ATTN_POLY_PER8
#define HSA_ATTN_POLY_PER8 0
#endif
constexpr int kPolyPer8 = HSA_ATTN_POLY_PER8;

struct AttnShared {
  uint64_t q_full;
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t v_full[kVSlots], v_empty[kVSlots];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint32_t tmem;
  float xmax[2][2][128];  // [tile parity][column half][row]: row-max exchange
  float xsum[2][128];     // [column half][row]: final row-sum exchange
};
constexpr int kAttnSmem = kTileBytes * (1 + kKSlots + kVSlots) + 1024 + (int)sizeof(AttnShared);

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe for x <= 8: x = n + f with n = round(x), f in [-1/2, 1/2]
// (Cody-Waite style split through the 1.5 * 2^23 rounding constant); 2^f from a
// degree-3 polynomial fitted here by weighted least squares on relative error
// (max relative error 7.7e-5, below the bf16 rounding of p); 2^n is added to the
// exponent field.  Inputs below -125 return about 2^-125 (p is stored as bf16;
// such terms vanish against the row sum).
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;
  const float n = t - 12582912.0f;
  const float f = x - n;
  const float p = fmaf(fmaf(fmaf(0.055181004f, f, 0.24263437f), f, 0.69326127f), f, 0.99992621f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// Packed fp32 pairs (two lanes of work per instruction on sm_100): d = a * b + c and d = a + b,
// each component rounded like fmaf / __fadd_rn.
__device__ __forceinline__ uint64_t as_u64(float2 v) {
  return (uint64_t)__float_as_uint(v.x) | ((uint64_t)__float_as_uint(v.y) << 32);
}
__device__ __forceinline__ float2 as_f2(uint64_t v) {
  return make_float2(__uint_as_float((uint32_t)v), __uint_as_float((uint32_t)(v >> 32)));
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(as_u64(a)), "l"(as_u64(b)), "l"(as_u64(c)));
  return as_f2(d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(as_u64(a)), "l"(as_u64(b)));
  return as_f2(d);
}
// max(a, b, c) in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, int M, int L, int H, __nv_bfloat16* __restrict__ O) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;                       // slot s at s * kTileBytes
  uint8_t* sV = sK + kKSlots * kTileBytes;
  AttnShared* sh = reinterpret_cast<AttnShared*>(sV + kVSlots * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kAttnBM, h = blockIdx.y;
  const int nj = (L + kAttnBN - 1) / kAttnBN;

  if (threadIdx.x == 0) {
    mbar_init(&sh->q_full, 1);
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(&sh->k_full[s], 1);
      mbar_init(&sh->k_empty[s], 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(&sh->v_full[s], 1);
      mbar_init(&sh->v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->s_full[b], 1);
      mbar_init(&sh->s_free[b], 256);
      mbar_init(&sh->p_full[b], 256);
      mbar_init(&sh->pv_done[b], 1);
    }
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = sh->tmem;

  if (warp == 0) {
    if (lane == 0) {
      const int x0 = h * 128;
      mbar_expect_tx(&sh->q_full, kTileBytes);
      tma_load_2d(sQ, &tmQ, &sh->q_full, x0, m0);
      tma_load_2d(sQ + kTileBytes / 2, &tmQ, &sh->q_full, x0 + 64, m0);
      for (int j = 0; j < nj; ++j) {
        const int sk = j % kKSlots, sv = j % kVSlots;
        if (!mbar_wait(&sh->k_empty[sk], ((j / kKSlots) & 1) ^ 1)) break;
        uint8_t* k = sK + sk * kTileBytes;
        mbar_expect_tx(&sh->k_full[sk], kTileBytes);
        tma_load_2d(k, &tmK, &sh->k_full[sk], x0, j * kAttnBN);
        tma_load_2d(k + kTileBytes / 2, &tmK, &sh->k_full[sk], x0 + 64, j * kAttnBN);
        if (!mbar_wait(&sh->v_empty[sv], ((j / kVSlots) & 1) ^ 1)) break;
        uint8_t* v = sV + sv * kTileBytes;
        mbar_expect_tx(&sh->v_full[sv], kTileBytes);
        tma_load_2d(v, &tmV, &sh->v_full[sv], x0, j * kAttnBN);
        tma_load_2d(v + kTileBytes / 2, &tmV, &sh->v_full[sv], x0 + 64, j * kAttnBN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(&sh->q_full, 0);
      auto issue_qk = [&](int j) -> bool {
        const int sk = j % kKSlots, b = j & 1;
        if (!mbar_wait(&sh->k_full[sk], (j / kKSlots) & 1)) return false;
        if (j >= 2 && !mbar_wait(&sh->s_free[b], ((j - 2) >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + sk * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
          umma_ss(tm + kColS + b * 128, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                  idesc_s, kk > 0);
        }
        umma_commit(&sh->s_full[b]);
        umma_commit(&sh->k_empty[sk]);          // K_j is free once S_j is computed
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < nj; ++j) {
        if (j + 1 < nj && !issue_qk(j + 1)) break;
        const int b = j & 1, sv = j % kVSlots;
        if (!mbar_wait(&sh->p_full[b], (j >> 1) & 1)) break;
        if (!mbar_wait(&sh->v_full[sv], (j / kVSlots) & 1)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + sv * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // V tile: key rows of 128 B (64 channels) per box; 16 keys = two 1024-byte atoms
          umma_ts(tm + kColO, tm + kColP + b * 64 + kk * 8, sdesc_sw128(v_addr + kk * 2048, kTileBytes / 2, 1024),
                  idesc_o, (j > 0 || kk > 0));
        }
        umma_commit(&sh->pv_done[b]);
        umma_commit(&sh->v_empty[sv]);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;               // key-column half of the tile this thread owns
    const int row = quarter * 32 + lane;
    const int bar_id = 1 + quarter;                 // named barrier of the two warps of this quarter
    const uint32_t lane_base = tm + ((uint32_t)(quarter * 32) << 16);
    const float sc = 0.12751743074680484f;          // log2(e) / sqrt(128)
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < nj; ++j) {
      const int b = j & 1;
      mbar_wait(&sh->s_full[b], (j >> 1) & 1);
      __syncwarp();
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(lane_base + kColS + b * 128 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(lane_base + kColS + b * 128 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&sh->s_free[b]);

      if ((j + 1) * kAttnBN > L) {  // ragged last tile only: keys beyond L get -inf
        const int valid = L - j * kAttnBN - half * 64;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 8; c < 64; c += 2)
        mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
      const float mloc = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // both halves of the row take the same max (double-buffered by tile parity)
      sh->xmax[b][half][row] = mloc;
      named_bar_sync(bar_id, 64);
      const float m_tile = sc * fmaxf(mloc, sh->xmax[b][half ^ 1][row]);
      if (j == 0) {
        m = m_tile;
      } else {
        const bool need = m_tile > m + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold PV_{j-1} before it is rescaled; each half rescales its 64 columns of O
          mbar_wait(&sh->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1);
          __syncwarp();
          tc_fence_after();
          const float corr = need ? ex2_approx(m - m_tile) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + half * 64 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
            tmem_st32(lane_base + kColO + half * 64 + c * 32, o);
          }
          tmem_st_wait();
          if (need) {
            l *= corr;
            m = m_tile;
          }
        }
      }
      const float neg_m = -m;
      const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(neg_m, neg_m);
      uint32_t pk[32];
      float2 rs4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float2 x = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2);
        const bool poly = (c & 7) >= 8 - kPolyPer8;  // compile-time per unrolled column pair
        const float p0 = poly ? ex2_poly(x.x) : ex2_approx(x.x);
        const float p1 = poly ? ex2_poly(x.y) : ex2_approx(x.y);
        rs4[(c >> 1) & 3] = fadd2(rs4[(c >> 1) & 3], make_float2(p0, p1));
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l += ((rs4[0].x + rs4[0].y) + (rs4[1].x + rs4[1].y)) + ((rs4[2].x + rs4[2].y) + (rs4[3].x + rs4[3].y));
      // P buffer b was last read by PV_{j-2}
      if (j >= 2) mbar_wait(&sh->pv_done[b], ((j - 2) >> 1) & 1);
      __syncwarp();
      tc_fence_after();
      tmem_st32(lane_base + kColP + b * 64 + half * 32, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sh->p_full[b]);
    }
    // ---------------------------------------------------------------- epilogue
    sh->xsum[half][row] = l;
    named_bar_sync(bar_id, 64);
    const float inv_l = 1.0f / (l + sh->xsum[half ^ 1][row]);
    mbar_wait(&sh->pv_done[(nj - 1) & 1], ((nj - 1) >> 1) & 1);
    __syncwarp();
    tc_fence_after();
    const int grow = m0 + row;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t o[32];
      __syncwarp();  // reconverge after the guarded stores before the warp-collective load
      tmem_ld32(lane_base + kColO + half * 64 + c * 32, o);
      tmem_ld_wait();
      if (grow < M) {
        __nv_bfloat16* dst = O + (size_t)grow * (H * 128) + h * 128 + half * 64 + c * 32;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
          u.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
          u.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
          u.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
          *reinterpret_cast<uint4*>(dst + e) = u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

int attention_bf16(const void* Q, int M, const void* K, const void* V, int L, int H, void* O, cudaStream_t st) {
  if (M <= 0) return HSA_OK;
  if (L <= 0 || H <= 0) return set_error(HSA_EINVAL, "attention: need L > 0 and H > 0");
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return set_error(HSA_EINVAL, "attention: null or misaligned pointer");
  const uint64_t D = (uint64_t)H * 128;
  CUtensorMap tq, tk, tv;
  int rc = make_tmap_2d(&tq, Q, true, D, (uint64_t)M, D * 2, 64, kAttnBM, true);
  if (!rc) rc = make_tmap_2d(&tk, K, true, D, (uint64_t)L, D * 2, 64, kAttnBN, true);
  if (!rc) rc = make_tmap_2d(&tv, V, true, D, (uint64_t)L, D * 2, 64, kAttnBN, true);
  if (rc) return rc;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return set_error(HSA_ECUDA, "attention: device index out of range");
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem) != cudaSuccess)
      return check_launch("attention: shared-memory attribute");
    attr_done[dev] = true;
  }
  ScopedTiming timing(HSA_KCLASS_ATTENTION, st);
  dim3 grid((M + kAttnBM - 1) / kAttnBM, H);
  k_attn_tc<<<grid, kAttnThreads, kAttnSmem, st>>>(tq, tk, tv, M, L, H, reinterpret_cast<__nv_bfloat16*>(O));
  count_launch(1);
  return check_launch("attn_tc launch");
}

}  // namespace hsa

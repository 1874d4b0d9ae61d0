// attn_tc.cu -- full-context attention of the active queries against the whole
// per-layer KV cache on the 5th-generation tensor cores (HSA summary §2.2:
// active tokens query the complete cached K, V -- fresh rows for active tokens,
// stale but valid rows for skipped ones -- at O(|A_i| N) cost).
//
//   o = softmax(q K^T / sqrt(128)) V, per head; q: M x 128H compacted rows,
//   K, V: L x 128H cache rows, o: M x 128H.  Non-causal.
//
// One CTA = one head x 128 queries, streaming 128-key tiles of K and V.
//   warp 0      TMA producer: Q once; K_j, V_j into a 3-slot ring
//   warp 1      TMEM owner (512 columns) and MMA issuer:
//                 S_j = Q K_j^T         (SS: both K-major, 128 x 128 x 128)
//                 O  += P_j V_j         (TS: P from TMEM, V MN-major)
//               S_{j+1} is issued before waiting for P_j, so QK^T of the next
//               tile overlaps the softmax of this one.
//   warps 2..5  softmax, thread = query row: S row from TMEM, running max in
//               the log2 domain, p = 2^(t - m) as bf16 back into TMEM; O is
//               rescaled in TMEM only when the max grew by more than 2^8
//               (otherwise the stale max keeps p <= 256, safe in fp32).
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P0 [384,448) P1 [448,512).
// Key rows beyond L are zero-filled by TMA and masked to -inf; query rows beyond
// M are computed on zeros and never stored.
#include "tcgen05.cuh"

namespace hsa {

constexpr int kAttnBM = 128;
constexpr int kAttnBN = 128;
constexpr int kAttnStages = 3;
constexpr int kAttnThreads = 192;
constexpr int kTileBytes = 128 * 128 * 2;       // one 128 x 128 bf16 operand tile (two 64-column boxes)
constexpr int kAttnSmem = kTileBytes * (1 + 2 * kAttnStages) + 1024 + 256;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct AttnBars {
  uint64_t q_full;
  uint64_t k_full[kAttnStages], v_full[kAttnStages], kv_empty[kAttnStages];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint32_t tmem;
};

__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, int M, int L, int H, __nv_bfloat16* __restrict__ O) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kTileBytes;  // slot s: K at s*2*kTileBytes, V right after
  AttnBars* bars = reinterpret_cast<AttnBars*>(smem + kTileBytes * (1 + 2 * kAttnStages));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kAttnBM, h = blockIdx.y;
  const int nj = (L + kAttnBN - 1) / kAttnBN;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], 128);
      mbar_init(&bars->p_full[b], 128);
      mbar_init(&bars->pv_done[b], 1);
    }
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = bars->tmem;

  if (warp == 0) {
    if (lane == 0) {
      const int x0 = h * 128;
      mbar_expect_tx(&bars->q_full, kTileBytes);
      tma_load_2d(sQ, &tmQ, &bars->q_full, x0, m0);
      tma_load_2d(sQ + kTileBytes / 2, &tmQ, &bars->q_full, x0 + 64, m0);
      for (int j = 0; j < nj; ++j) {
        const int s = j % kAttnStages;
        if (!mbar_wait(&bars->kv_empty[s], ((j / kAttnStages) & 1) ^ 1)) break;
        uint8_t* k = sKV + s * 2 * kTileBytes;
        uint8_t* v = k + kTileBytes;
        mbar_expect_tx(&bars->k_full[s], kTileBytes);
        tma_load_2d(k, &tmK, &bars->k_full[s], x0, j * kAttnBN);
        tma_load_2d(k + kTileBytes / 2, &tmK, &bars->k_full[s], x0 + 64, j * kAttnBN);
        mbar_expect_tx(&bars->v_full[s], kTileBytes);
        tma_load_2d(v, &tmV, &bars->v_full[s], x0, j * kAttnBN);
        tma_load_2d(v + kTileBytes / 2, &tmV, &bars->v_full[s], x0 + 64, j * kAttnBN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(&bars->q_full, 0);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % kAttnStages, b = j & 1;
        if (!mbar_wait(&bars->k_full[s], (j / kAttnStages) & 1)) return false;
        if (j >= 2 && !mbar_wait(&bars->s_free[b], ((j - 2) >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sKV + s * 2 * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
          umma_ss(tm + kColS + b * 128, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                  idesc_s, kk > 0);
        }
        umma_commit(&bars->s_full[b]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < nj; ++j) {
        if (j + 1 < nj && !issue_qk(j + 1)) break;
        const int s = j % kAttnStages, b = j & 1;
        if (!mbar_wait(&bars->p_full[b], (j >> 1) & 1)) break;
        if (!mbar_wait(&bars->v_full[s], (j / kAttnStages) & 1)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sKV + s * 2 * kTileBytes + kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // V tile: key rows of 128 B (64 channels) per box; 16 keys = two 1024-byte atoms
          umma_ts(tm + kColO, tm + kColP + b * 64 + kk * 8, sdesc_sw128(v_addr + kk * 2048, kTileBytes / 2, 1024),
                  idesc_o, (j > 0 || kk > 0));
        }
        umma_commit(&bars->pv_done[b]);
        umma_commit(&bars->kv_empty[s]);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tm + ((uint32_t)(quarter * 32) << 16);
    const float sc = 0.12751743074680484f;  // log2(e) / sqrt(128)
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < nj; ++j) {
      const int b = j & 1;
      mbar_wait(&bars->s_full[b], (j >> 1) & 1);
      __syncwarp();
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + kColS + b * 128 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * c));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->s_free[b]);

      const int valid = min(kAttnBN, L - j * kAttnBN);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float v = __uint_as_float(sr[c]);
        if (c >= valid) v = -INFINITY;
        sr[c] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      const float m_tile = mx * sc;
      if (j == 0) {
        m = m_tile;
      } else {
        const bool need = m_tile > m + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold PV_{j-1} before it is rescaled
          mbar_wait(&bars->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1);
          __syncwarp();
          tc_fence_after();
          const float corr = need ? ex2_approx(m - m_tile) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
            tmem_st32(lane_base + kColO + c * 32, o);
          }
          tmem_st_wait();
          if (need) {
            l *= corr;
            m = m_tile;
          }
        }
      }
      const float neg_m = -m;
      uint32_t pk[64];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c]), sc, neg_m));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c + 1]), sc, neg_m));
        rs += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l += rs;
      // P buffer b was last read by PV_{j-2}
      if (j >= 2) mbar_wait(&bars->pv_done[b], ((j - 2) >> 1) & 1);
      __syncwarp();
      tc_fence_after();
      tmem_st32(lane_base + kColP + b * 64, pk);
      tmem_st32(lane_base + kColP + b * 64 + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[b]);
    }
    // ---------------------------------------------------------------- epilogue
    mbar_wait(&bars->pv_done[(nj - 1) & 1], ((nj - 1) >> 1) & 1);
    __syncwarp();
    tc_fence_after();
    const float inv_l = 1.0f / l;
    const int grow = m0 + row;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      __syncwarp();  // reconverge after the guarded stores before the warp-collective load
      tmem_ld32(lane_base + kColO + c * 32, o);
      tmem_ld_wait();
      if (grow < M) {
        __nv_bfloat16* dst = O + (size_t)grow * (H * 128) + h * 128 + c * 32;
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
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem) != cudaSuccess)
      return check_launch("attention: shared-memory attribute");
    attr_done[dev] = true;
  }
  dim3 grid((M + kAttnBM - 1) / kAttnBM, H);
  ScopedTiming timing(HSA_KCLASS_ATTENTION, st);
  k_attn_tc<<<grid, kAttnThreads, kAttnSmem, st>>>(tq, tk, tv, M, L, H, reinterpret_cast<__nv_bfloat16*>(O));
  count_launch(1);
  return check_launch("attn_tc launch");
}

}  // namespace hsa

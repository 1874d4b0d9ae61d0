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

      if ((j + 1) * kAttnBN > L) {  // ragged last tile only: keys beyond L get -inf
        const int valid = L - j * kAttnBN;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
      }
      // row max with 8 independent chains (a single chain would serialise 128 dependent ops)
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(sr[c]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
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
      float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c]), sc, neg_m));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c + 1]), sc, neg_m));
        rs8[(c >> 1) & 7] += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l += ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
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

// ---------------------------------------------------------------------------------------------
// k_attn_tc2: two 128-query tiles per CTA (256 queries share every K/V tile).
//   warp 0      TMA producer: Q0, Q1 once; then K_0, V_0, K_1, V_1, ... into a 5-slot ring
//   warp 1      MMA issuer:  S_t = Q_t K_j^T for t = 0, 1, then O_t += P_t V_j for t = 0, 1
//   warps 2..5  softmax of tile 0, warps 6..9 softmax of tile 1 (thread = query row)
// TMEM (512 columns): tile t owns S_t = [256t, 256t+128) and O_t = [256t+128, 256t+256);
// P_t (bf16) is written over the first 64 columns of S_t once the row has been read.
// S_t(j+1) is issued only after PV_t(j) has completed (it overwrites P_t(j)), so by the
// time a softmax thread sees S_t(j) the previous O_t update is done and O_t may be
// rescaled without waiting.
constexpr int kAttn2Threads = 320;
constexpr int kRingSlots = 5;
constexpr int kAttn2Smem = kTileBytes * (2 + kRingSlots) + 1024 + 512;

struct Attn2Bars {
  uint64_t q_full;
  uint64_t full[kRingSlots], empty[kRingSlots];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint32_t tmem;
};

__global__ void __launch_bounds__(kAttn2Threads, 1)
    k_attn_tc2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, int M, int L, int H, __nv_bfloat16* __restrict__ O) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                           // Q0 then Q1
  uint8_t* sRing = smem + 2 * kTileBytes;       // slot s at s * kTileBytes
  Attn2Bars* bars = reinterpret_cast<Attn2Bars*>(smem + kTileBytes * (2 + kRingSlots));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 2 * kAttnBM, h = blockIdx.y;
  const int nj = (L + kAttnBN - 1) / kAttnBN;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kRingSlots; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
      mbar_init(&bars->pv_done[t], 1);
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
      mbar_expect_tx(&bars->q_full, 2 * kTileBytes);
      for (int t = 0; t < 2; ++t) {
        tma_load_2d(sQ + t * kTileBytes, &tmQ, &bars->q_full, x0, m0 + t * kAttnBM);
        tma_load_2d(sQ + t * kTileBytes + kTileBytes / 2, &tmQ, &bars->q_full, x0 + 64, m0 + t * kAttnBM);
      }
      for (int q = 0; q < 2 * nj; ++q) {
        const int s = q % kRingSlots;
        if (!mbar_wait(&bars->empty[s], ((q / kRingSlots) & 1) ^ 1)) break;
        const CUtensorMap* map = (q & 1) ? &tmV : &tmK;
        uint8_t* dst = sRing + s * kTileBytes;
        const int y = (q >> 1) * kAttnBN;
        mbar_expect_tx(&bars->full[s], kTileBytes);
        tma_load_2d(dst, map, &bars->full[s], x0, y);
        tma_load_2d(dst + kTileBytes / 2, map, &bars->full[s], x0 + 64, y);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
      bool ok = mbar_wait(&bars->q_full, 0);
      for (int j = 0; ok && j < nj; ++j) {
        const int qk = 2 * j, qv = 2 * j + 1;
        const int sk = qk % kRingSlots, sv = qv % kRingSlots;
        if (!mbar_wait(&bars->full[sk], (qk / kRingSlots) & 1)) break;
        const uint32_t k_addr = smem_u32(sRing + sk * kTileBytes);
        for (int t = 0; t < 2; ++t) {
          // S_t(j) overwrites P_t(j-1): PV_t(j-1) must have completed
          if (j > 0 && !mbar_wait(&bars->pv_done[t], (j - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(sQ + t * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
            umma_ss(tm + 256 * t, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                    idesc_s, kk > 0);
          }
          umma_commit(&bars->s_full[t]);
        }
        if (!ok) break;
        umma_commit(&bars->empty[sk]);          // K_j is free once both S tiles are done
        if (!mbar_wait(&bars->full[sv], (qv / kRingSlots) & 1)) break;
        const uint32_t v_addr = smem_u32(sRing + sv * kTileBytes);
        for (int t = 0; t < 2; ++t) {
          if (!mbar_wait(&bars->p_full[t], j & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tm + 256 * t + 128, tm + 256 * t + kk * 8,
                    sdesc_sw128(v_addr + kk * 2048, kTileBytes / 2, 1024), idesc_o, (j > 0 || kk > 0));
          umma_commit(&bars->pv_done[t]);
        }
        umma_commit(&bars->empty[sv]);          // V_j is free once both O updates are done
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    const int t = (warp - 2) >> 2;               // query tile of this warpgroup
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tm + ((uint32_t)(quarter * 32) << 16) + 256 * t;
    const float sc = 0.12751743074680484f;       // log2(e) / sqrt(128)
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < nj; ++j) {
      mbar_wait(&bars->s_full[t], j & 1);
      __syncwarp();
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lane_base + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * c));
      tmem_ld_wait();
      if ((j + 1) * kAttnBN > L) {
        const int valid = L - j * kAttnBN;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(sr[c]));
      const float m_tile = sc * fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                      fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      if (j == 0) {
        m = m_tile;
      } else {
        const bool need = m_tile > m + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          // PV_t(j-1) completed before S_t(j) was issued: O_t is stable here
          const float corr = need ? ex2_approx(m - m_tile) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + 128 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
            tmem_st32(lane_base + 128 + c * 32, o);
          }
          if (need) {
            l *= corr;
            m = m_tile;
          }
        }
      }
      const float neg_m = -m;
      uint32_t pk[64];
      float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c]), sc, neg_m));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c + 1]), sc, neg_m));
        rs8[(c >> 1) & 7] += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l += ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      tmem_st32(lane_base, pk);
      tmem_st32(lane_base + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[t]);
    }
    // ---------------------------------------------------------------- epilogue
    mbar_wait(&bars->pv_done[t], (nj - 1) & 1);
    __syncwarp();
    tc_fence_after();
    const float inv_l = 1.0f / l;
    const int grow = m0 + t * kAttnBM + row;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      __syncwarp();
      tmem_ld32(lane_base + 128 + c * 32, o);
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
    if (cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem) != cudaSuccess ||
        cudaFuncSetAttribute(k_attn_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttn2Smem) != cudaSuccess)
      return check_launch("attention: shared-memory attribute");
    attr_done[dev] = true;
  }
  ScopedTiming timing(HSA_KCLASS_ATTENTION, st);
  if (M > kAttnBM) {
    dim3 grid((M + 2 * kAttnBM - 1) / (2 * kAttnBM), H);
    k_attn_tc2<<<grid, kAttn2Threads, kAttn2Smem, st>>>(tq, tk, tv, M, L, H, reinterpret_cast<__nv_bfloat16*>(O));
  } else {
    dim3 grid(1, H);
    k_attn_tc<<<grid, kAttnThreads, kAttnSmem, st>>>(tq, tk, tv, M, L, H, reinterpret_cast<__nv_bfloat16*>(O));
  }
  count_launch(1);
  return check_launch("attn_tc launch");
}

}  // namespace hsa

// attn_tc.cu -- full-context attention of the active queries against the whole
// per-layer KV cache on the 5th-generation tensor cores (HSA summary §2.2:
// active tokens query the complete cached K, V -- fresh rows for active tokens,
// stale but valid rows for skipped ones -- at O(|A_i| N) cost).
//
//   o = softmax(q K^T / sqrt(128)) V, per head; q: M x 128H compacted rows,
//   K, V: L x 128H cache rows, o: M x 128H.  Non-causal.
//
// One CTA = one head x 128 queries, streaming 128-key tiles of K and V.  Two variants share the
// code: k_attn_tc<2> (two tile parities, one CTA per SM) for long key ranges, k_attn_tc<1> (one
// parity, two CTAs per SM) for short ones.  k_attn_tc<2>:
//   warp 0      TMA producer (the warp waits, one elected lane copies): Q once; K_j into a
//               3-slot ring, V_j into a 2-slot ring, in the order the MMA warp consumes
//               them (K0 K1 V0 K2 V1 K3 ...).  V_j and K_{j+2} complete on the barriers
//               that also count the softmax warps' P stores of tile j, so the MMA warp
//               waits twice per tile.
//   warp 1      TMEM owner (512 columns) and MMA issuer (the warp runs the loop with
//               warp-uniform descriptors, one elected lane issues):
//                 S_b = Q K_j^T          (SS: both K-major, 128 x 128 x 128), b = j % 2
//                 O_b += P_j V_j         (TS: P from TMEM, V MN-major), in two halves of
//                                        64 keys, each issued as soon as its P is stored
//               QK^T of tile j+2 is issued right after PV of tile j, so the tensor
//               pipe alternates between the two parities.
//   warps 2..9  softmax, one thread per query row and all 128 key columns of a tile:
//               warps 2-5 take the even tiles, warps 6-9 the odd tiles (warp w reads
//               TMEM lane quarter w % 4).  Each parity keeps its own running max, sum
//               and O accumulator, so the two warps of a sub-partition never wait for
//               each other and one's exponentials overlap the other's loads, max and
//               stores.  p = 2^(t - m) goes back to TMEM as bf16 over the first 64
//               columns of the S buffer it came from; the first half of the keys is
//               released to the MMA warp while the second half's exponentials are
//               computed.  O_b is rescaled in TMEM only when the max grew by more than
//               2^8 (the stale max keeps p <= 256).
//               The epilogue merges the two parities: O = (a0 O_0 + a1 O_1) / (a0 l_0
//               + a1 l_1) with a_b = 2^(m_b - max(m_0, m_1)).
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P_b aliases the
// first 64 columns of S_b.  QK^T of tile j+2 overwrites S_b only after PV of tile j
// has read P_b: both are issued by the one MMA thread, whose tcgen05.mma operations
// execute in issue order.
// k_attn_tc<1> runs the same steps with one parity: warps 2..5 take every tile, TMEM holds S
// [0,128) and O [128,256), K and V have one slot each, and QK^T of tile j+1 follows PV of tile
// j.  A CTA's chain of tiles is then serial, but it needs half the shared memory, TMEM and
// threads, so two CTAs share an SM and one's tiles overlap the other's.  The CTAs are persistent:
// each walks units blockIdx.x, blockIdx.x + gridDim.x, ..., with Q of the next unit loaded once
// the last QK^T of the current one is done, and the K of the next unit's first tile bundled with
// the current unit's last P, so the next unit's first QK^T follows the last PV at once.  The
// epilogue stages O in the V slot (the next unit's first V waits for it) and releases O to the
// next unit's first PV as soon as it is in registers.  With a few key tiles per unit (the
// cross-attention's 512-row context) CTA set-up, Q latency and the epilogue were most of a
// unit's time when every unit was a CTA of its own.
// Key rows beyond L are zero-filled by TMA and masked to -inf; query rows beyond
// M are computed on zeros and never stored.
//
// Work units are (128-query tile, head) pairs, one per CTA, in blockIdx.x order.  The
// units of the complete waves run whole.  When a workspace is given, the units of an
// incomplete last wave are each split over S ranges of key tiles (S chosen so the split
// CTAs fill the last wave).  A split CTA writes its unnormalised O (fp32) with its row
// max and sum, and k_attn_combine merges the S parts into the bf16 output.
#include "tcgen05.cuh"

namespace hsa {

constexpr int kAttnBM = 128;
constexpr int kAttnBN = 128;
// Key ranges of at most this many 128-key tiles run the one-parity kernel (k_attn_tc<1>), two
// CTAs per SM; longer ones the two-parity kernel (k_attn_tc<2>), one CTA per SM
constexpr int kShortMaxTiles = 8;
constexpr int kTileBytes = 128 * 128 * 2;         // one 128 x 128 bf16 operand tile (two 64-column boxes)
constexpr uint32_t kColS = 0;
// Exponentials computed with the polynomial instead of the MUFU unit: the columns c
// of a thread's 128 with (c % 8) >= 8 - kPolyPer8.  Every measurement at the Wan-1.3B
// shape (attention alone, 32760 x 32760, 12 heads) found the MUFU path faster: with two
// softmax threads per row 0 / 2 / 4 of 8 took 6.44 / 7.04 / 7.63 ms, and with the tile
// parities 6.05 / 6.35 / 7.52 ms at the power cap.  So the MUFU path alone is the default.
#ifndef HSA_ATTN_POLY_PER8
#define HSA_ATTN_POLY_PER8 0
#endif
constexpr int kPolyPer8 = HSA_ATTN_POLY_PER8;
// The one-parity kernel of short key ranges measured the same way at the cross-attention shape
// (32760 x 512, 12 heads): 0 / 2 / 4 of 8 took 0.132 / 0.133 / 0.143 ms, so it uses the MUFU path too.
// P goes to the MMA warp in two halves of 64 keys; PV of the first half starts while the
// softmax warps compute the exponentials of the second.  Measured at the Wan-1.3B shape
// (attention alone): one release per tile 5.40 ms, halves 5.21 ms, quarters 5.47 ms.

struct AttnShared {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[3];    // k_full: the first tile of each parity only
  uint64_t v_empty[2];
  // p_full[b][h]: P of keys [64 h, 64 h + 64) of tile t (b = t % kPar) stored by the 128 softmax
  // threads of parity b, plus one producer arrival with the bytes of the next operand the MMA
  // warp needs: V_t for h = 0, K_{t+kPar} for h = 1 (a plain arrival when there is no such tile)
  uint64_t s_full[2], p_full[2][2], o_done;
  // one-parity kernel, which walks several units: Q reusable (last QK^T of a unit done), O read
  // out by the epilogue, staging area (the V slot) read back by the epilogue
  uint64_t q_empty, o_free, stage_free;
  uint32_t tmem;
  float xm[2][128], xl[2][128];  // [parity][row]: running max and sum, merged in the epilogue
};

// The two variants.  kPar = 2: 2 control warps + 8 softmax warps, TMEM S0 S1 O0 O1 (512
// columns), a 3-slot K ring and a 2-slot V ring, one CTA per SM.  kPar = 1: 2 control warps + 4
// softmax warps, TMEM S O (256 columns), one K and one V slot, two CTAs per SM, so one CTA's
// fill and drain overlap the other's tiles.
template <int kPar>
struct AttnCfg {
  static constexpr int kThreads = 64 + 128 * kPar;
  static constexpr int kKSlots = kPar == 2 ? 3 : 1;
  static constexpr int kVSlots = kPar == 2 ? 2 : 1;
  static constexpr uint32_t kCols = 256 * kPar;
  static constexpr uint32_t kColO = 128 * kPar;
  static constexpr int kSmem = kTileBytes * (1 + kKSlots + kVSlots) + 1024 + (int)sizeof(AttnShared);
};
static_assert(2 * AttnCfg<1>::kSmem <= 227 * 1024, "two one-parity CTAs must fit one SM's shared memory");

// Unit -> CTA map: units u < u_full are whole; unit u_full + t / s_tail, key range t % s_tail,
// for the split tail.  part_o / part_ml hold the split CTAs' partial results, slot t.
struct AttnGrid {
  int QT;          // query tiles per head
  int u_full;      // units run whole
  int s_tail;      // key-range splits of each tail unit (1: no split)
  float* part_o;   // [slots][128][128] unnormalised O
  float2* part_ml; // [slots][128] (row max in log2 units, row sum)
};

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

template <int kPar>
__global__ void __launch_bounds__(AttnCfg<kPar>::kThreads, 3 - kPar)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, int M, int L, int H, __nv_bfloat16* __restrict__ O,
              const AttnGrid grid) {
  pdl_prologue();
  using Cfg = AttnCfg<kPar>;
  constexpr int KS = Cfg::kKSlots, VS = Cfg::kVSlots;
  constexpr uint32_t kColO = Cfg::kColO;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;                       // slot s at s * kTileBytes
  uint8_t* sV = sK + KS * kTileBytes;
  AttnShared* sh = reinterpret_cast<AttnShared*>(sV + VS * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // kPar == 1 walks units blockIdx.x, blockIdx.x + gridDim.x, ... (all whole); kPar == 2 takes one
  const int n_units = kPar == 1 ? (grid.u_full - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 1;
  int u = blockIdx.x, split = 0, n_split = 1, slot = -1;
  if (u >= grid.u_full) {
    const int t = u - grid.u_full;
    u = grid.u_full + t / grid.s_tail;
    split = t % grid.s_tail;
    n_split = grid.s_tail;
    if (n_split > 1) slot = t;
  }
  const int m0 = (u % grid.QT) * kAttnBM, h = u / grid.QT;
  // this CTA's key tiles [j0, j0 + nt): loops, ring slots and parities use the local index
  const int nj_all = (L + kAttnBN - 1) / kAttnBN;
  const int j0 = split * nj_all / n_split;
  const int nt = (split + 1) * nj_all / n_split - j0;

  if (threadIdx.x == 0) {
    mbar_init(&sh->q_full, 1);
    for (int s = 0; s < KS; ++s) mbar_init(&sh->k_empty[s], 1);
    for (int b = 0; b < kPar; ++b) mbar_init(&sh->k_full[b], 1);
    for (int s = 0; s < VS; ++s) mbar_init(&sh->v_empty[s], 1);
    for (int b = 0; b < kPar; ++b) {
      mbar_init(&sh->s_full[b], 1);
      mbar_init(&sh->p_full[b][0], 129);   // the parity's 128 softmax threads + the producer
      mbar_init(&sh->p_full[b][1], 129);
    }
    mbar_init(&sh->o_done, 1);
    if (kPar == 1) {
      mbar_init(&sh->q_empty, 1);
      mbar_init(&sh->o_free, 128);
      mbar_init(&sh->stage_free, 128);
    }
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem, Cfg::kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = sh->tmem;

  if (warp == 0 && kPar == 1) {
    // TMA producer of the one-parity kernel, unit after unit (T counts this CTA's tiles over all
    // of its units): Q of unit i once the last QK^T of unit i-1 is done, so it arrives while
    // that unit finishes; K and V of every tile in order, the K of tile T + 1 (the next unit's
    // first at a unit's end) completing with the second half of P_T.  The V slot doubles as the
    // epilogue's staging area, so the first V of a unit also waits until the previous unit's
    // output has been read back out of it.
    const bool leader = elect_one();
    const int ntot = n_units * nt;
    auto unit_of = [&](int i) { return (int)blockIdx.x + i * (int)gridDim.x; };
    auto load_k = [&](int T, uint64_t* bar) -> bool {
      const bool ok = __shfl_sync(0xffffffffu, mbar_wait(&sh->k_empty[0], (T & 1) ^ 1), 0);
      __syncwarp();
      if (ok && leader) {
        const int x0 = unit_of(T / nt) / grid.QT * 128, row = (T % nt) * kAttnBN;
        mbar_expect_tx(bar, kTileBytes);
        tma_load_2d(sK, &tmK, bar, x0, row);
        tma_load_2d(sK + kTileBytes / 2, &tmK, bar, x0 + 64, row);
      }
      return ok;
    };
    bool ok = true;
    for (int i = 0; ok && i < n_units; ++i) {
      const int ui = unit_of(i), x0 = ui / grid.QT * 128;
      if (i > 0) {
        ok = __shfl_sync(0xffffffffu, mbar_wait(&sh->q_empty, (i - 1) & 1), 0);
        __syncwarp();
        if (!ok) break;
      }
      if (leader) {
        const int row = ui % grid.QT * kAttnBM;
        mbar_expect_tx(&sh->q_full, kTileBytes);
        tma_load_2d(sQ, &tmQ, &sh->q_full, x0, row);
        tma_load_2d(sQ + kTileBytes / 2, &tmQ, &sh->q_full, x0 + 64, row);
      }
      __syncwarp();
      if (i == 0) ok = load_k(0, &sh->k_full[0]);
      for (int t = 0; ok && t < nt; ++t) {
        const int T = i * nt + t;
        ok = __shfl_sync(0xffffffffu, mbar_wait(&sh->v_empty[0], (T & 1) ^ 1), 0);
        if (ok && t == 0 && i > 0) ok = __shfl_sync(0xffffffffu, mbar_wait(&sh->stage_free, (i - 1) & 1), 0);
        __syncwarp();
        if (!ok) break;
        if (leader) {
          mbar_expect_tx(&sh->p_full[0][0], kTileBytes);
          tma_load_2d(sV, &tmV, &sh->p_full[0][0], x0, t * kAttnBN);
          tma_load_2d(sV + kTileBytes / 2, &tmV, &sh->p_full[0][0], x0 + 64, t * kAttnBN);
        }
        if (T + 1 < ntot) {
          ok = load_k(T + 1, &sh->p_full[0][1]);
        } else {
          if (leader) mbar_arrive(&sh->p_full[0][1]);
          __syncwarp();
        }
      }
    }
  } else if (warp == 0) {
    // TMA producer: the whole warp runs the loop and waits; one elected lane issues the copies
    const int x0 = h * 128;
    const bool leader = elect_one();
    if (leader) {
      mbar_expect_tx(&sh->q_full, kTileBytes);
      tma_load_2d(sQ, &tmQ, &sh->q_full, x0, m0);
      tma_load_2d(sQ + kTileBytes / 2, &tmQ, &sh->q_full, x0 + 64, m0);
    }
    // K of tile j into its ring slot, completing on `bar`
    auto load_k = [&](int j, uint64_t* bar) -> bool {
      const int sk = j % KS;
      const bool ok = __shfl_sync(0xffffffffu, mbar_wait(&sh->k_empty[sk], ((j / KS) & 1) ^ 1), 0);
      __syncwarp();
      if (ok && leader) {
        uint8_t* k = sK + sk * kTileBytes;
        mbar_expect_tx(bar, kTileBytes);
        tma_load_2d(k, &tmK, bar, x0, (j0 + j) * kAttnBN);
        tma_load_2d(k + kTileBytes / 2, &tmK, bar, x0 + 64, (j0 + j) * kAttnBN);
      }
      return ok;
    };
    bool ok = load_k(0, &sh->k_full[0]);
    if (kPar == 2 && ok && nt > 1) ok = load_k(1, &sh->k_full[1]);
    // Phase order of the p_full arrivals: the producer arrives on phase (t / kPar) of
    // p_full[t % kPar][*] only after waiting for a ring slot that the MMA warp releases after it
    // waited on the previous phase of the same barrier, so no arrival lands a phase early
    for (int t = 0; ok && t < nt; ++t) {
      const int b = t % kPar, sv = t % VS;
      ok = __shfl_sync(0xffffffffu, mbar_wait(&sh->v_empty[sv], ((t / VS) & 1) ^ 1), 0);
      __syncwarp();
      if (!ok) break;
      if (leader) {
        uint8_t* v = sV + sv * kTileBytes;
        mbar_expect_tx(&sh->p_full[b][0], kTileBytes);
        tma_load_2d(v, &tmV, &sh->p_full[b][0], x0, (j0 + t) * kAttnBN);
        tma_load_2d(v + kTileBytes / 2, &tmV, &sh->p_full[b][0], x0 + 64, (j0 + t) * kAttnBN);
      }
      if (t + kPar < nt) {
        ok = load_k(t + kPar, &sh->p_full[b][1]);
      } else {
        if (leader) mbar_arrive(&sh->p_full[b][1]);
        __syncwarp();
      }
    }
  } else if (warp == 1 && kPar == 1) {
    // MMA issuer of the one-parity kernel, unit after unit: S = Q K_T^T, then P_T V_T in two
    // halves into O, then the next QK^T.  A unit's first PV overwrites O, so it waits until the
    // epilogue has read the previous unit's O out of TMEM; the unit's last QK^T frees Q.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
    const bool leader = elect_one();
    const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t k_desc = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t v_desc = sdesc_sw128(smem_u32(sV), kTileBytes / 2, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool r = __shfl_sync(0xffffffffu, mbar_wait(bar, parity), 0);
      __syncwarp();
      return r;
    };
    // QK^T of the tile whose K is in the slot; `last`: the unit's last, after which Q is free
    auto issue_qk = [&](bool last) {
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4;
          umma_ss(tm + kColS, q_desc + off, k_desc + off, idesc_s, kk > 0);
        }
        umma_commit(&sh->s_full[0]);
        umma_commit(&sh->k_empty[0]);
        if (last) umma_commit(&sh->q_empty);
      }
      __syncwarp();
    };
    bool ok = true;
    for (int i = 0; ok && i < n_units; ++i) {
      ok = wait_all(&sh->q_full, i & 1);
      if (ok && i == 0) ok = wait_all(&sh->k_full[0], 0);
      if (!ok) break;
      issue_qk(nt == 1);
      for (int t = 0; ok && t < nt; ++t) {
        const int T = i * nt + t;
        if (t == 0 && i > 0 && !wait_all(&sh->o_free, (i - 1) & 1)) { ok = false; break; }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          // half 0 also brings V_T, half 1 also the K of the next tile
          if (!wait_all(&sh->p_full[0][q], T & 1)) { ok = false; break; }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = q * 4; kk < q * 4 + 4; ++kk)
              umma_ts(tm + kColO, tm + kColS + kk * 8, v_desc + (uint64_t)(kk * 2048 >> 4), idesc_o, (t > 0 || kk > 0));
            if (q == 1) umma_commit(&sh->v_empty[0]);
          }
          __syncwarp();
        }
        if (ok && t + 1 < nt) issue_qk(t + 2 == nt);   // overwrites S (P_T) after PV_T in issue order
      }
      if (leader) umma_commit(&sh->o_done);   // every MMA of the unit
      __syncwarp();
    }
  } else if (warp == 1) {
    // MMA issuer: the whole warp runs the loop, waits and builds the descriptors (warp-uniform
    // values); one elected lane issues each tcgen05.mma and commit
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
    const bool leader = elect_one();
    // descriptor of a shared-memory address a: desc(base) + (a - base) / 16 (the start-address
    // field is the low 14 bits of a / 16 and never carries: shared memory is below 256 KB)
    const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t k_desc = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t v_desc = sdesc_sw128(smem_u32(sV), kTileBytes / 2, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool r = __shfl_sync(0xffffffffu, mbar_wait(bar, parity), 0);
      __syncwarp();
      return r;
    };
    // QK^T of tile t; the first tile of each parity waits for its K here, later ones through p_full
    auto issue_qk = [&](int t) -> bool {
      const int sk = t % KS, b = t % kPar;
      if (t < kPar && !wait_all(&sh->k_full[t], 0)) return false;
      tc_fence_after();
      const uint64_t kd = k_desc + (uint64_t)((sk * kTileBytes) >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4;
          umma_ss(tm + kColS + b * 128, q_desc + off, kd + off, idesc_s, kk > 0);
        }
        umma_commit(&sh->s_full[b]);
        umma_commit(&sh->k_empty[sk]);   // K_t is free once S_t is computed
      }
      __syncwarp();
      return true;
    };
    bool ok = wait_all(&sh->q_full, 0);
    if (ok) ok = issue_qk(0);
    if (kPar == 2 && ok && nt > 1) ok = issue_qk(1);
    for (int t = 0; ok && t < nt; ++t) {
      const int b = t % kPar, sv = t % VS;
      const uint64_t vd = v_desc + (uint64_t)((sv * kTileBytes) >> 4);

      // PV half by half of the keys: the first starts while the softmax warps are still
      // computing the exponentials of the second
      bool got = true;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        // half 0 also brings V_t, half 1 also the K of QK^T(t + kPar)
        if (!wait_all(&sh->p_full[b][q], (t / kPar) & 1)) { got = false; break; }
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = q * 4; kk < q * 4 + 4; ++kk) {
            // V tile: key rows of 128 B (64 channels) per box; 16 keys = two 1024-byte atoms
            umma_ts(tm + kColO + b * 128, tm + kColS + b * 128 + kk * 8, vd + (uint64_t)(kk * 2048 >> 4), idesc_o,
                    (t >= kPar || kk > 0));
          }
          if (q == 1) umma_commit(&sh->v_empty[sv]);   // V_t is free once PV_t is done
        }
        __syncwarp();
      }
      if (!got) break;
      if (t + kPar < nt) ok = issue_qk(t + kPar);   // overwrites S_b (P_t) after PV_t in issue order
    }
    if (leader) umma_commit(&sh->o_done);   // every MMA of this CTA
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int par = (warp - 2) >> 2;                // tile parity this warp handles
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tm + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_col = lane_base + kColS + par * 128, o_col = lane_base + kColO + par * 128;
    const float sc = 0.12751743074680484f;          // log2(e) / sqrt(128)
    for (int iu = 0; iu < n_units; ++iu) {   // one unit unless kPar == 1
    float m = -INFINITY, l = 0.f;
    for (int t = par; t < nt; t += kPar) {
      mbar_wait(&sh->s_full[par], ((iu * nt + t) / kPar) & 1);
      __syncwarp();
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        tmem_ld32(s_col + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + q4 * 32));
      tmem_ld_wait();

      if ((j0 + t + 1) * kAttnBN > L) {  // ragged last tile only: keys beyond L get -inf
        const int valid = L - (j0 + t) * kAttnBN;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 8; c < 128; c += 2)
        mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
      const float m_tile = sc * fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                      fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // lazy rescale: the max moves only when it grew by more than 2^8; O_par is then scaled
      // after P is stored, when the S registers are free
      bool need = false;
      float corr = 1.0f;
      if (t == par) {
        m = m_tile;
      } else if (m_tile > m + 8.0f) {
        need = true;
        corr = ex2_approx(m - m_tile);
        l *= corr;
        m = m_tile;
      }
      // a warp that rescales O_par releases both halves of P after the rescale; the others
      // release the first half as soon as its stores have landed
      const bool any_need = __any_sync(0xffffffffu, need);
      const float neg_m = -m;
      const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(neg_m, neg_m);
      float2 rs4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[32];
#pragma unroll
        for (int c = hh * 64; c < hh * 64 + 64; c += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2);
          const bool poly = (c & 7) >= 8 - kPolyPer8;  // compile-time per unrolled column pair
          const float p0 = poly ? ex2_poly(x.x) : ex2_approx(x.x);
          const float p1 = poly ? ex2_poly(x.y) : ex2_approx(x.y);
          rs4[(c >> 1) & 3] = fadd2(rs4[(c >> 1) & 3], make_float2(p0, p1));
          pk[(c >> 1) & 31] = pack_bf16x2(p0, p1);
          // P column i holds keys 2i, 2i+1 of the tile, over S_par's first 64 columns; stored
          // every 32 keys (16 columns)
          if ((c & 31) == 30) tmem_st16(s_col + (c >> 5) * 16, pk + ((c >> 1) & 31) - 15);
          if (hh == 1 && c == 66 && !any_need) {
            // the first half's stores were issued two column pairs ago
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sh->p_full[par][0]);
          }
        }
      }
      l += ((rs4[0].x + rs4[0].y) + (rs4[1].x + rs4[1].y)) + ((rs4[2].x + rs4[2].y) + (rs4[3].x + rs4[3].y));
      if (any_need) {
        // O_par holds PV of this parity's previous tile, complete: S_par was written by an MMA
        // issued after that PV, and the s_full wait above covered it.  PV of this tile starts
        // only after this warp's p_full arrivals below.
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(o_col + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
          tmem_st32(o_col + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      if (any_need) mbar_arrive(&sh->p_full[par][0]);
      mbar_arrive(&sh->p_full[par][1]);
    }
    // ---------------------------------------------------------------- epilogue
    if constexpr (kPar == 1) {
      // one parity, whole key range (the host never splits these units): O / l of unit iu
      mbar_wait(&sh->o_done, iu & 1);
      __syncwarp();
      tc_fence_after();
      const int ui = (int)blockIdx.x + iu * (int)gridDim.x;
      const int m0u = ui % grid.QT * kAttnBM, hu = ui / grid.QT;
      const float inv_l = 1.0f / l;
      // The unit's last PV is done, so the V slot is free until this warp's stage_free arrival:
      // the warp stages its 32 rows there (256 B each, the 16-byte chunks of row r XOR-rotated by
      // r % 16), then writes them out with 16 lanes per row, two whole rows per store instead of
      // 32 rows' fragments.  O is released to the next unit's first PV once it is in registers.
      uint8_t* stage = sV + quarter * (32 * 256);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        __syncwarp();
        tmem_ld32(o_col + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 pk4;
          pk4.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
          pk4.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
          pk4.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
          pk4.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
          const int chunk = c * 4 + (e >> 3);
          *reinterpret_cast<uint4*>(stage + lane * 256 + ((chunk ^ (lane & 15)) << 4)) = pk4;
        }
      }
      tc_fence_before();
      mbar_arrive(&sh->o_free);
      __syncwarp();
      const int cl = lane & 15;
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int r = 2 * i + (lane >> 4);
        const uint4 val = *reinterpret_cast<const uint4*>(stage + r * 256 + ((cl ^ (r & 15)) << 4));
        const int grow = m0u + quarter * 32 + r;
        if (grow < M) *reinterpret_cast<uint4*>(O + (size_t)grow * (H * 128) + hu * 128 + cl * 8) = val;
      }
      // the next unit's first V may overwrite the staging area once every row is read back
      fence_proxy_async_smem();
      mbar_arrive(&sh->stage_free);
    } else {
    // merge the two parities; parity 1 has tiles only when nt >= 2
    sh->xm[par][row] = m;
    sh->xl[par][row] = l;
    named_bar_sync(1 + quarter, 64);                // the even and the odd warp of this lane quarter
    const bool two = nt >= 2;
    const float m0v = sh->xm[0][row], m1v = sh->xm[1][row];
    const float mm = two ? fmaxf(m0v, m1v) : m0v;
    const float a0 = ex2_approx(m0v - mm);
    const float a1 = two ? ex2_approx(m1v - mm) : 0.f;
    const float inv_l = 1.0f / (a0 * sh->xl[0][row] + a1 * sh->xl[1][row]);
    const float w0 = a0 * inv_l, w1 = a1 * inv_l;
    mbar_wait(&sh->o_done, 0);
    __syncwarp();
    tc_fence_after();
    const int grow = m0 + row;
    if (slot >= 0) {
      // split CTA: unnormalised O relative to mm, and (mm, a0 l_0 + a1 l_1), for k_attn_combine
      float* dst_o = grid.part_o + ((size_t)slot * kAttnBM + row) * 128;
      if (par == 0) grid.part_ml[(size_t)slot * kAttnBM + row] = make_float2(mm, a0 * sh->xl[0][row] + a1 * sh->xl[1][row]);
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const uint32_t col = (uint32_t)(par * 64 + c * 32);
        uint32_t o0[32], o1[32];
        __syncwarp();
        tmem_ld32(lane_base + kColO + col, o0);
        if (two) tmem_ld32(lane_base + kColO + 128 + col, o1);
        tmem_ld_wait();
        if (!two) {
#pragma unroll
          for (int e = 0; e < 32; ++e) o1[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst_o + col + e) =
              make_float4(fmaf(__uint_as_float(o0[e + 0]), a0, __uint_as_float(o1[e + 0]) * a1),
                          fmaf(__uint_as_float(o0[e + 1]), a0, __uint_as_float(o1[e + 1]) * a1),
                          fmaf(__uint_as_float(o0[e + 2]), a0, __uint_as_float(o1[e + 2]) * a1),
                          fmaf(__uint_as_float(o0[e + 3]), a0, __uint_as_float(o1[e + 3]) * a1));
      }
    } else {
    // this warp writes output columns [par * 64, par * 64 + 64) of the head
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      const uint32_t col = (uint32_t)(par * 64 + c * 32);
      uint32_t o0[32], o1[32];
      __syncwarp();  // reconverge after the guarded stores before the warp-collective loads
      tmem_ld32(lane_base + kColO + col, o0);
      if (two) tmem_ld32(lane_base + kColO + 128 + col, o1);
      tmem_ld_wait();
      if (!two) {
#pragma unroll
        for (int e = 0; e < 32; ++e) o1[e] = 0u;
      }
      if (grow < M) {
        __nv_bfloat16* dst = O + (size_t)grow * (H * 128) + h * 128 + col;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          float f[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) f[t] = fmaf(__uint_as_float(o0[e + t]), w0, __uint_as_float(o1[e + t]) * w1);
          uint4 pk4;
          pk4.x = pack_bf16x2(f[0], f[1]);
          pk4.y = pack_bf16x2(f[2], f[3]);
          pk4.z = pack_bf16x2(f[4], f[5]);
          pk4.w = pack_bf16x2(f[6], f[7]);
          *reinterpret_cast<uint4*>(dst + e) = pk4;
        }
      }
    }
    }
    }  // two-parity merge
    }  // units
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tm, AttnCfg<kPar>::kCols);
  }
}

// Merge the key-range splits of the tail units: one warp per (tail unit, row), lane = 4 channels.
//   O = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s,  m = max_s m_s.
__global__ void __launch_bounds__(256) k_attn_combine(const float* __restrict__ part_o,
                                                      const float2* __restrict__ part_ml, int n_tail, int s_tail,
                                                      int u_full, int QT, int M, int H,
                                                      __nv_bfloat16* __restrict__ O) {
  pdl_prologue();
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int tu = w / kAttnBM, row = w % kAttnBM;
  if (tu >= n_tail) return;
  const int u = u_full + tu;
  const int grow = (u % QT) * kAttnBM + row, h = u / QT;
  if (grow >= M) return;
  float mx = -INFINITY;
  for (int sp = 0; sp < s_tail; ++sp) mx = fmaxf(mx, part_ml[(size_t)(tu * s_tail + sp) * kAttnBM + row].x);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  for (int sp = 0; sp < s_tail; ++sp) {
    const size_t r = (size_t)(tu * s_tail + sp) * kAttnBM + row;
    const float2 ml = part_ml[r];
    const float a = exp2f(ml.x - mx);
    den = fmaf(a, ml.y, den);
    const float4 o = *reinterpret_cast<const float4*>(part_o + r * 128 + lane * 4);
    acc = make_float4(fmaf(a, o.x, acc.x), fmaf(a, o.y, acc.y), fmaf(a, o.z, acc.z), fmaf(a, o.w, acc.w));
  }
  const float inv = 1.0f / den;
  uint2 pk;
  pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(O + (size_t)grow * (H * 128) + h * 128 + lane * 4) = pk;
}

namespace {
struct TailSplit {
  int u_full, s_tail, n_tail;   // s_tail == 1: no split
};
// Units of the complete waves run whole; the n_tail units of an incomplete last wave are split
// over S key ranges, S minimising the tail's time ceil(n_tail S / SMs) / S (in whole-unit times)
// plus a small per-split cost (each split CTA refills the pipeline).  Each split keeps at least
// two key tiles, and a split is taken only when it saves at least 15 % of the tail's time.
TailSplit plan_tail(int U, int nj_all, int sms) {
  TailSplit p{U, 1, 0};
  const int tail = U % sms;
  if (tail == 0) return p;
  int best_s = 1;
  double best = 0.85;
  for (int S = 2; S <= 16 && 2 * S <= nj_all; ++S) {
    const double t = (double)((tail * S + sms - 1) / sms) / S + 0.02 * S;
    if (t < best - 1e-9) {
      best = t;
      best_s = S;
    }
  }
  if (best_s == 1) return p;
  return TailSplit{U - tail, best_s, tail};
}
size_t tail_split_bytes(const TailSplit& p) {
  if (p.s_tail <= 1) return 0;
  const size_t slots = (size_t)p.n_tail * p.s_tail * kAttnBM;
  return align256(slots * 128 * sizeof(float)) + align256(slots * sizeof(float2));
}
}  // namespace

size_t attention_split_bytes(int M, int L, int H) {
  if (M <= 0 || L <= 0 || H <= 0) return 0;
  if ((L + kAttnBN - 1) / kAttnBN <= kShortMaxTiles) return 0;   // one-parity CTAs: no split
  const int QT = (M + kAttnBM - 1) / kAttnBM;
  return tail_split_bytes(plan_tail(QT * H, (L + kAttnBN - 1) / kAttnBN, num_sms()));
}

// bf16 attention; with a workspace of at least attention_split_bytes(M, L, H) the tail units
// are split over key ranges (otherwise, or with none, every unit runs whole).
int attention_bf16(const void* Q, int M, const void* K, const void* V, int L, int H, void* O, cudaStream_t st,
                   void* ws, size_t ws_bytes) {
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
  static PerContextOnce attr;
  rc = attr.ensure([](void**) {
    if (cudaFuncSetAttribute(k_attn_tc<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnCfg<2>::kSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(k_attn_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnCfg<1>::kSmem) !=
            cudaSuccess)
      return check_launch("attention: shared-memory attribute");
    return (int)HSA_OK;
  });
  if (rc) return rc;
  const int nj_all = (L + kAttnBN - 1) / kAttnBN;
  if (nj_all <= kShortMaxTiles) {
    // short key range: persistent one-parity CTAs, two per SM, each walking units blockIdx.x,
    // blockIdx.x + grid, ... (all whole)
    const int QT = (M + kAttnBM - 1) / kAttnBM, U = QT * H;
    const int ctas = U < 2 * num_sms() ? U : 2 * num_sms();
    AttnGrid g{QT, U, 1, nullptr, nullptr};
    ScopedTiming timing(HSA_KCLASS_ATTENTION, st);
    launch(k_attn_tc<1>, ctas, AttnCfg<1>::kThreads, AttnCfg<1>::kSmem, st, tq, tk, tv, M, L, H,
           reinterpret_cast<__nv_bfloat16*>(O), g);
    count_launch(1);
    return check_launch("attn_tc (one parity) launch");
  }
  const int QT = (M + kAttnBM - 1) / kAttnBM, U = QT * H;
  TailSplit ts = plan_tail(U, nj_all, num_sms());
  const size_t need = tail_split_bytes(ts);
  if (need == 0 || !ws || ws_bytes < need || !aligned16(ws)) ts = TailSplit{U, 1, 0};
  AttnGrid g{QT, ts.u_full, ts.s_tail, nullptr, nullptr};
  if (ts.s_tail > 1) {
    const size_t slots = (size_t)ts.n_tail * ts.s_tail * kAttnBM;
    g.part_o = static_cast<float*>(ws);
    g.part_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + align256(slots * 128 * sizeof(float)));
  }
  ScopedTiming timing(HSA_KCLASS_ATTENTION, st);
  const int ctas = ts.u_full + ts.n_tail * ts.s_tail;
  launch(k_attn_tc<2>, ctas, AttnCfg<2>::kThreads, AttnCfg<2>::kSmem, st, tq, tk, tv, M, L, H,
         reinterpret_cast<__nv_bfloat16*>(O), g);
  count_launch(1);
  if (ts.s_tail > 1) {
    rc = check_launch("attn_tc launch");
    if (rc) return rc;
    const int warps = ts.n_tail * kAttnBM;
    launch(k_attn_combine, (warps + 7) / 8, 256, 0, st, g.part_o, g.part_ml, ts.n_tail, ts.s_tail, ts.u_full, QT, M,
           H, reinterpret_cast<__nv_bfloat16*>(O));
    count_launch(1);
    return check_launch("attn_combine launch");
  }
  return check_launch("attn_tc launch");
}

}  // namespace hsa

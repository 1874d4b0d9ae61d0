// simt_f32.cu -- float32 linear layers and attention on the CUDA cores.
//
// The float32 workloads (the tiny single-layer loop) need true fp32
// arithmetic: tensor-core tf32 rounds operands to 10 mantissa bits, which is
// too coarse for a 1e-4 relative-L2 bar.  These kernels are register-tiled
// loops over shared-memory tiles; the bf16 path (gemm_tc.cu, attn_tc.cu) is the
// fast one.
#include "common.cuh"

namespace hsa {

// y = epilogue(x W^T + b): BM x 64 output tile per 256-thread block, BM/16 x 4 per thread.  The
// tile height is chosen per call so that small active sets still give the GPU two blocks per SM:
// the layer's time then follows the number of active rows instead of one block's latency.
template <int EPI, int BM>
__global__ void __launch_bounds__(256) k_gemm_f32(const float* __restrict__ A, const float* __restrict__ W, int M,
                                                  int Nout, int K, const float* __restrict__ bias,
                                                  const float* __restrict__ gate, float* __restrict__ out) {
  pdl_prologue();
  constexpr int RM = BM / 16;                       // rows per thread
  __shared__ float As[16][BM + 4];
  __shared__ float Ws[16][68];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * 64;
  const int lr = threadIdx.x >> 2, lk = (threadIdx.x & 3) * 4;
  float acc[RM][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), w = a;
    if (lr < BM && m0 + lr < M && k0 + lk < K)
      a = *reinterpret_cast<const float4*>(A + (size_t)(m0 + lr) * K + k0 + lk);
    if (n0 + lr < Nout && k0 + lk < K) w = *reinterpret_cast<const float4*>(W + (size_t)(n0 + lr) * K + k0 + lk);
    if (lr < BM) {
      As[lk + 0][lr] = a.x; As[lk + 1][lr] = a.y; As[lk + 2][lr] = a.z; As[lk + 3][lr] = a.w;
    }
    Ws[lk + 0][lr] = w.x; Ws[lk + 1][lr] = w.y; Ws[lk + 2][lr] = w.z; Ws[lk + 3][lr] = w.w;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float af[RM], wf[4];
#pragma unroll
      for (int i = 0; i < RM; ++i) af[i] = As[kk][ty * RM + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) wf[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(af[i], wf[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < RM; ++i) {
    const int m = m0 + ty * RM + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= Nout) continue;
      float v = acc[i][j] + (bias ? bias[n] : 0.f);
      float* y = out + (size_t)m * Nout + n;
      if (EPI == 1) {  // GELU(tanh)
        v = 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)));
        *y = v;
      } else if (EPI == 2) {  // residual += gate * v
        *y = fmaf(gate ? gate[n] : 1.f, v, *y);
      } else {
        *y = v;
      }
    }
  }
}

template <int EPI>
static void launch_gemm_f32(const float* A, int M, int K, const float* W, int Nout, const float* bias,
                            const float* gate, float* out, cudaStream_t st) {
  const long long nb = (Nout + 63) / 64, want = 2LL * num_sms();
  const auto blocks = [&](int bm) { return nb * ((M + bm - 1) / bm); };
  if (blocks(64) >= want) {
    launch(k_gemm_f32<EPI, 64>, dim3((unsigned)nb, (M + 63) / 64), 256, 0, st, A, W, M, Nout, K, bias, gate, out);
  } else if (blocks(32) >= want) {
    launch(k_gemm_f32<EPI, 32>, dim3((unsigned)nb, (M + 31) / 32), 256, 0, st, A, W, M, Nout, K, bias, gate, out);
  } else {
    launch(k_gemm_f32<EPI, 16>, dim3((unsigned)nb, (M + 15) / 16), 256, 0, st, A, W, M, Nout, K, bias, gate, out);
  }
}

int gemm_f32(const float* A, int M, int K, const float* W, int Nout, const float* bias, int epi, const float* gate,
             float* out, cudaStream_t st) {
  if (M <= 0) return HSA_OK;
  if (K <= 0 || K % 4 || Nout <= 0 || Nout % 4) return set_error(HSA_EINVAL, "f32 linear: need K, Nout % 4 == 0");
  if (!A || !W || !out || !aligned16(A) || !aligned16(W) || !aligned16(out))
    return set_error(HSA_EINVAL, "f32 linear: null or misaligned pointer");
  ScopedTiming timing(HSA_KCLASS_GEMM, st);
  switch (epi) {
    case 1: launch_gemm_f32<1>(A, M, K, W, Nout, bias, gate, out, st); break;
    case 2: launch_gemm_f32<2>(A, M, K, W, Nout, bias, gate, out, st); break;
    default: launch_gemm_f32<0>(A, M, K, W, Nout, bias, gate, out, st); break;
  }
  count_launch(1);
  return check_launch("gemm_f32 launch");
}

// o = softmax(q K^T / sqrt(128)) V per head in fp32 on the CUDA cores, tiled: a CTA takes 32 query
// rows of one head and one range of the keys, 64-key tiles of K and V staged in shared memory.
// Thread (ty, tx) of 256: rows 2ty, 2ty+1; logits of keys tx + 16 j (j < 4) of the tile, then
// output channels 8 tx .. 8 tx + 7.  Online softmax per row (max and sum shuffled across the 16
// threads of a row pair).  With several key ranges per (query block, head) each CTA writes its
// unnormalised O with the row max and sum, and k_attn_f32_combine merges them:
//   o = sum_s e^(m_s - m) O_s / sum_s e^(m_s - m) l_s,  m = max_s m_s.
constexpr int kF32BQ = 32, kF32BK = 64, kF32Ld = 132;
constexpr int kF32AttnSmem = (kF32BQ * kF32Ld + 2 * kF32BK * kF32Ld + kF32BQ * (kF32BK + 4)) * 4;

__global__ void __launch_bounds__(256, 2) k_attn_f32(const float* __restrict__ Q, int M, const float* __restrict__ K,
                                                     const float* __restrict__ V, int L, int H, int n_split,
                                                     float* __restrict__ O, float* __restrict__ part_o,
                                                     float2* __restrict__ part_ml) {
  pdl_prologue();
  extern __shared__ float4 sm4[];
  float* Qs = reinterpret_cast<float*>(sm4);        // [32][132]
  float* Ks = Qs + kF32BQ * kF32Ld;                  // [64][132]
  float* Vs = Ks + kF32BK * kF32Ld;                  // [64][132]
  float* Ps = Vs + kF32BK * kF32Ld;                  // [32][68]
  constexpr int kPsLd = kF32BK + 4;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int QB = (M + kF32BQ - 1) / kF32BQ;
  int b = blockIdx.x;
  const int split = b % n_split;
  b /= n_split;
  const int qb = b % QB, h = b / QB;
  const int D = H * 128, m0 = qb * kF32BQ;
  const int nk = (L + kF32BK - 1) / kF32BK;
  const int t0 = split * nk / n_split, t1 = (split + 1) * nk / n_split;
  for (int i = tid; i < kF32BQ * 32; i += 256) {
    const int r = i >> 5, c4 = i & 31;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m0 + r < M) v = *reinterpret_cast<const float4*>(Q + (size_t)(m0 + r) * D + h * 128 + 4 * c4);
    *reinterpret_cast<float4*>(Qs + r * kF32Ld + 4 * c4) = v;
  }
  const float scale = 0.08838834764831845f;          // 1 / sqrt(128)
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[2][8];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) o[i][c] = 0.f;
  const float* q0r = Qs + (2 * ty) * kF32Ld;
  const float* q1r = q0r + kF32Ld;
  for (int t = t0; t < t1; ++t) {
    const int k0 = t * kF32BK;
    __syncthreads();                                   // the previous tile's reads of Ks / Vs / Ps are done
    for (int i = tid; i < kF32BK * 32; i += 256) {
      const int key = i >> 5, c4 = i & 31;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (k0 + key < L) {
        kv = *reinterpret_cast<const float4*>(K + (size_t)(k0 + key) * D + h * 128 + 4 * c4);
        vv = *reinterpret_cast<const float4*>(V + (size_t)(k0 + key) * D + h * 128 + 4 * c4);
      }
      *reinterpret_cast<float4*>(Ks + key * kF32Ld + 4 * c4) = kv;
      *reinterpret_cast<float4*>(Vs + key * kF32Ld + 4 * c4) = vv;
    }
    __syncthreads();
    float s[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll 4
    for (int c = 0; c < 128; c += 4) {
      const float4 a0 = *reinterpret_cast<const float4*>(q0r + c);
      const float4 a1 = *reinterpret_cast<const float4*>(q1r + c);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 kk = *reinterpret_cast<const float4*>(Ks + (tx + 16 * j) * kF32Ld + c);
        s[0][j] = fmaf(a0.x, kk.x, fmaf(a0.y, kk.y, fmaf(a0.z, kk.z, fmaf(a0.w, kk.w, s[0][j]))));
        s[1][j] = fmaf(a1.x, kk.x, fmaf(a1.y, kk.y, fmaf(a1.z, kk.z, fmaf(a1.w, kk.w, s[1][j]))));
      }
    }
    float corr[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s[i][j] = (k0 + tx + 16 * j < L) ? s[i][j] * scale : -INFINITY;
        mx = fmaxf(mx, s[i][j]);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[i], mx);          // finite: every tile holds a key below L
      corr[i] = expf(m[i] - m_new);
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = expf(s[i][j] - m_new);
        sum += p;
        Ps[(2 * ty + i) * kPsLd + tx + 16 * j] = p;
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      l[i] = l[i] * corr[i] + sum;
      m[i] = m_new;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < 8; ++c) o[i][c] *= corr[i];
    const float* p0r = Ps + (2 * ty) * kPsLd;
    const float* p1r = p0r + kPsLd;
#pragma unroll 4
    for (int key = 0; key < kF32BK; ++key) {
      const float p0 = p0r[key], p1 = p1r[key];
      const float4 va = *reinterpret_cast<const float4*>(Vs + key * kF32Ld + 8 * tx);
      const float4 vb = *reinterpret_cast<const float4*>(Vs + key * kF32Ld + 8 * tx + 4);
      const float vv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        o[0][c] = fmaf(p0, vv[c], o[0][c]);
        o[1][c] = fmaf(p1, vv[c], o[1][c]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int row = 2 * ty + i, grow = m0 + row;
    if (grow >= M) continue;
    if (n_split == 1) {
      const float inv = 1.0f / l[i];
      float* dst = O + (size_t)grow * D + h * 128 + 8 * tx;
      *reinterpret_cast<float4*>(dst) = make_float4(o[i][0] * inv, o[i][1] * inv, o[i][2] * inv, o[i][3] * inv);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(o[i][4] * inv, o[i][5] * inv, o[i][6] * inv, o[i][7] * inv);
    } else {
      const size_t slot = (size_t)blockIdx.x * kF32BQ + row;
      float* dst = part_o + slot * 128 + 8 * tx;
      *reinterpret_cast<float4*>(dst) = make_float4(o[i][0], o[i][1], o[i][2], o[i][3]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(o[i][4], o[i][5], o[i][6], o[i][7]);
      if (tx == 0) part_ml[slot] = make_float2(m[i], l[i]);
    }
  }
}

// Merge of the key ranges: one warp per (query block, head, row), lane = 4 channels.
__global__ void __launch_bounds__(256) k_attn_f32_combine(const float* __restrict__ part_o,
                                                          const float2* __restrict__ part_ml, int M, int H,
                                                          int n_split, float* __restrict__ O) {
  pdl_prologue();
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int QB = (M + kF32BQ - 1) / kF32BQ;
  const int row = w % kF32BQ, unit = w / kF32BQ;       // unit = h * QB + qb
  if (unit >= QB * H) return;
  const int qb = unit % QB, h = unit / QB, grow = qb * kF32BQ + row;
  if (grow >= M) return;
  float mx = -INFINITY;
  for (int s = 0; s < n_split; ++s) mx = fmaxf(mx, part_ml[((size_t)unit * n_split + s) * kF32BQ + row].x);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const size_t slot = ((size_t)unit * n_split + s) * kF32BQ + row;
    const float2 ml = part_ml[slot];
    const float a = expf(ml.x - mx);
    den = fmaf(a, ml.y, den);
    const float4 v = *reinterpret_cast<const float4*>(part_o + slot * 128 + 4 * lane);
    acc = make_float4(fmaf(a, v.x, acc.x), fmaf(a, v.y, acc.y), fmaf(a, v.z, acc.z), fmaf(a, v.w, acc.w));
  }
  const float inv = 1.0f / den;
  *reinterpret_cast<float4*>(O + (size_t)grow * (H * 128) + h * 128 + 4 * lane) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

// Key ranges per (query block, head): enough CTAs for two per SM, at least 2 key tiles a range,
// and partials that fit the workspace.
static int f32_attn_splits(int M, int L, int H, size_t ws_bytes) {
  const int QB = (M + kF32BQ - 1) / kF32BQ, nk = (L + kF32BK - 1) / kF32BK;
  const long long units = (long long)QB * H;
  int S = (int)((2LL * num_sms() + units - 1) / units);
  if (S > nk / 2) S = nk / 2;
  const size_t per = (size_t)units * kF32BQ * (128 * sizeof(float) + sizeof(float2));
  if (per > 0 && (size_t)S * per > ws_bytes) S = (int)(ws_bytes / per);
  return S < 1 ? 1 : S;
}

size_t attention_f32_split_bytes(int M, int L, int H) {
  if (M <= 0 || L <= 0 || H <= 0) return 0;
  const int S = f32_attn_splits(M, L, H, ~size_t(0));
  if (S <= 1) return 0;
  const size_t slots = (size_t)((M + kF32BQ - 1) / kF32BQ) * H * S * kF32BQ;
  return align256(slots * 128 * sizeof(float)) + align256(slots * sizeof(float2));
}

int attention_f32(const float* Q, int M, const float* K, const float* V, int L, int H, float* O, cudaStream_t st,
                  void* ws, size_t ws_bytes) {
  if (M <= 0) return HSA_OK;
  if (L <= 0 || H <= 0) return set_error(HSA_EINVAL, "attention: need L > 0 and H > 0");
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return set_error(HSA_EINVAL, "attention: null or misaligned pointer");
  static PerContextOnce attr;
  int rc = attr.ensure([](void**) {
    if (cudaFuncSetAttribute(k_attn_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, kF32AttnSmem) != cudaSuccess)
      return check_launch("attention (fp32): shared-memory attribute");
    return (int)HSA_OK;
  });
  if (rc) return rc;
  const int QB = (M + kF32BQ - 1) / kF32BQ;
  int S = (ws && aligned16(ws)) ? f32_attn_splits(M, L, H, ws_bytes) : 1;
  const size_t slots = (size_t)QB * H * S * kF32BQ;
  float* part_o = S > 1 ? static_cast<float*>(ws) : nullptr;
  float2* part_ml =
      S > 1 ? reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + align256(slots * 128 * sizeof(float))) : nullptr;
  if (S > 1 && align256(slots * 128 * sizeof(float)) + slots * sizeof(float2) > ws_bytes) S = 1;
  ScopedTiming timing(HSA_KCLASS_ATTENTION, st);
  launch(k_attn_f32, (unsigned)(QB * H * S), 256, kF32AttnSmem, st, Q, M, K, V, L, H, S, O, part_o, part_ml);
  count_launch(1);
  rc = check_launch("attn_f32 launch");
  if (rc || S == 1) return rc;
  const long long warps = (long long)QB * H * kF32BQ;
  launch(k_attn_f32_combine, (unsigned)((warps + 7) / 8), 256, 0, st, part_o, part_ml, M, H, S, O);
  count_launch(1);
  return check_launch("attn_f32 combine launch");
}

}  // namespace hsa

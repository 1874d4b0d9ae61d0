// simt_f32.cu -- float32 linear layers and attention on the CUDA cores.
//
// The float32 workloads (the tiny single-layer loop) need true fp32
// arithmetic: tensor-core tf32 rounds operands to 10 mantissa bits, which is
// too coarse for a 1e-4 relative-L2 bar.  These kernels are plain register-
// tiled loops; the bf16 path (gemm_tc.cu, attn_tc.cu) is the fast one.
#include "common.cuh"

namespace hsa {

// y = epilogue(x W^T + b): 64 x 64 output tile per 256-thread block, 4 x 4 per thread.
template <int EPI>
__global__ void __launch_bounds__(256) k_gemm_f32(const float* __restrict__ A, const float* __restrict__ W, int M,
                                                  int Nout, int K, const float* __restrict__ bias,
                                                  const float* __restrict__ gate, float* __restrict__ out) {
  __shared__ float As[16][68];
  __shared__ float Ws[16][68];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int lr = threadIdx.x >> 2, lk = (threadIdx.x & 3) * 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), w = a;
    if (m0 + lr < M && k0 + lk < K) a = *reinterpret_cast<const float4*>(A + (size_t)(m0 + lr) * K + k0 + lk);
    if (n0 + lr < Nout && k0 + lk < K) w = *reinterpret_cast<const float4*>(W + (size_t)(n0 + lr) * K + k0 + lk);
    As[lk + 0][lr] = a.x; As[lk + 1][lr] = a.y; As[lk + 2][lr] = a.z; As[lk + 3][lr] = a.w;
    Ws[lk + 0][lr] = w.x; Ws[lk + 1][lr] = w.y; Ws[lk + 2][lr] = w.z; Ws[lk + 3][lr] = w.w;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float af[4], wf[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        af[i] = As[kk][ty * 4 + i];
        wf[i] = Ws[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(af[i], wf[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
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

int gemm_f32(const float* A, int M, int K, const float* W, int Nout, const float* bias, int epi, const float* gate,
             float* out, cudaStream_t st) {
  if (M <= 0) return HSA_OK;
  if (K <= 0 || K % 4 || Nout <= 0 || Nout % 4) return set_error(HSA_EINVAL, "f32 linear: need K, Nout % 4 == 0");
  if (!A || !W || !out || !aligned16(A) || !aligned16(W) || !aligned16(out))
    return set_error(HSA_EINVAL, "f32 linear: null or misaligned pointer");
  dim3 grid((Nout + 63) / 64, (M + 63) / 64);
  ScopedTiming timing(HSA_KCLASS_GEMM, st);
  switch (epi) {
    case 1: k_gemm_f32<1><<<grid, 256, 0, st>>>(A, W, M, Nout, K, bias, gate, out); break;
    case 2: k_gemm_f32<2><<<grid, 256, 0, st>>>(A, W, M, Nout, K, bias, gate, out); break;
    default: k_gemm_f32<0><<<grid, 256, 0, st>>>(A, W, M, Nout, K, bias, gate, out); break;
  }
  count_launch(1);
  return check_launch("gemm_f32 launch");
}

// o = softmax(q K^T / sqrt(128)) V per head; one warp per (query row, head),
// lanes split the 128 channels 4 each, online softmax over the L keys.
__global__ void __launch_bounds__(256) k_attn_f32(const float* __restrict__ Q, int M, const float* __restrict__ K,
                                                  const float* __restrict__ V, int L, int H,
                                                  float* __restrict__ O) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= M * H) return;
  const int r = gw / H, h = gw % H;
  const int D = H * 128;
  const float scale = 0.08838834764831845f;  // 1/sqrt(128)
  const float4 q = *reinterpret_cast<const float4*>(Q + (size_t)r * D + h * 128 + lane * 4);
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < L; ++j) {
    const float4 k = *reinterpret_cast<const float4*>(K + (size_t)j * D + h * 128 + lane * 4);
    float s = q.x * k.x + q.y * k.y + q.z * k.z + q.w * k.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    s *= scale;
    const float m_new = fmaxf(m, s);
    const float corr = expf(m - m_new), p = expf(s - m_new);
    const float4 v = *reinterpret_cast<const float4*>(V + (size_t)j * D + h * 128 + lane * 4);
    l = l * corr + p;
    acc.x = acc.x * corr + p * v.x;
    acc.y = acc.y * corr + p * v.y;
    acc.z = acc.z * corr + p * v.z;
    acc.w = acc.w * corr + p * v.w;
    m = m_new;
  }
  const float inv = 1.0f / l;
  *reinterpret_cast<float4*>(O + (size_t)r * D + h * 128 + lane * 4) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

int attention_f32(const float* Q, int M, const float* K, const float* V, int L, int H, float* O, cudaStream_t st) {
  if (M <= 0) return HSA_OK;
  if (L <= 0 || H <= 0) return set_error(HSA_EINVAL, "attention: need L > 0 and H > 0");
  const long long warps = (long long)M * H;
  ScopedTiming timing(HSA_KCLASS_ATTENTION, st);
  k_attn_f32<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(Q, M, K, V, L, H, O);
  count_launch(1);
  return check_launch("attn_f32 launch");
}

}  // namespace hsa

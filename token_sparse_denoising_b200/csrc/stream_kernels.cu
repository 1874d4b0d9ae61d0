// stream_kernels.cu -- the bandwidth-bound kernels of the HSA step.
//
//   k_euler            x += dsigma * v_hat over all N x C (HSA summary §2.3)
//   k_scatter_vhat     v_hat[idx[r]] = v_A[r]  (+ L1 score of the change, §2.1; + the Euler
//                      update of the row when every token is active)
//   k_l1_score         per-token L1 relative change (§2.1)
//   k_ln_rows          LayerNorm + modulation / affine, optional gather x[idx] (§2.2: active rows only)
//   k_qk_norm_rope     q/k RMSNorm over D, 3D RoPE, compact Q, K/V scattered into the cache (§2.2)
//   k_rms_rows         RMSNorm rows (cross-attention query / context keys), or plain copy
//   k_gather_rows      x[idx[r]] -> compacted rows (patch-embedding input)
//
// All rows are read and written with 16-byte vectors; one warp owns one row,
// so a row's reduction stays in registers and warp shuffles.
#include <type_traits>

#include "common.cuh"

namespace hsa {

constexpr float kScoreEps = 1e-8f;
constexpr float kNormEps = 1e-6f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float4 ld4_stream(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }

// 4 consecutive elements of a float or bf16 row, widened to float
__device__ __forceinline__ float4 load4(const float* p) { return ld4(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x), b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(float* p, float4 v) { st4(p, v); }
// raw register forms of 4 consecutive elements, widened to float
__device__ __forceinline__ float4 widen4(float4 v) { return v; }
__device__ __forceinline__ float4 widen4(uint2 u) {
  const float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
  const float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// ------------------------------------------------------------------ §2.3 cached Euler
// x[e] += dsigma * v_hat[e] for every element; n4 float4 groups.  Each thread takes up to U
// groups a grid-stride apart per pass, all loaded before any is used; the host sizes the grid
// as a whole number of blocks per SM, so one pass is one balanced wave.
__global__ void __launch_bounds__(256) k_euler(float* __restrict__ x, const float* __restrict__ vhat, size_t n4,
                                               float dsigma) {
  pdl_prologue();
  constexpr int U = 4;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t base = (size_t)blockIdx.x * blockDim.x + threadIdx.x; base < n4; base += U * stride) {
    float4 xv[U], v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const size_t i = base + u * stride;
      if (i < n4) {
        xv[u] = ld4_stream(x + 4 * i);
        v[u] = ld4_stream(vhat + 4 * i);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const size_t i = base + u * stride;
      if (i < n4) {
        xv[u].x = fmaf(dsigma, v[u].x, xv[u].x);
        xv[u].y = fmaf(dsigma, v[u].y, xv[u].y);
        xv[u].z = fmaf(dsigma, v[u].z, xv[u].z);
        xv[u].w = fmaf(dsigma, v[u].w, xv[u].w);
        __stcs(reinterpret_cast<float4*>(x + 4 * i), xv[u]);
      }
    }
  }
}

// v_hat[idx[r]] = v_A[r]; with score != nullptr also
// score[idx[r]] = sum|v_A[r] - v_hat_old| / (sum|v_hat_old| + eps).  One warp per row.
// When `x` is given the Euler update of that row is fused in (full steps).
__global__ void __launch_bounds__(256) k_scatter_vhat(float* __restrict__ vhat, const float* __restrict__ vA,
                                                      const int* __restrict__ idx, int M, int N, int C,
                                                      float* __restrict__ score, float* __restrict__ x,
                                                      float dsigma) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const int n = idx[r];
  if (n < 0 || n >= N) {
    if (lane == 0) flag_error(HSA_EINDEX);
    return;
  }
  float* vrow = vhat + (size_t)n * C;
  const float* arow = vA + (size_t)r * C;
  float* xrow = x ? x + (size_t)n * C : nullptr;
  float num = 0.f, den = 0.f;
  // U chunks of 128 floats per warp iteration: every load of the group is issued
  // before the first one is used, so a warp keeps 3U 16-byte loads in flight
  constexpr int U = 4;
  for (int c0 = 4 * lane; c0 < C; c0 += 128 * U) {
    float4 a[U], o[U], xv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 128 * u;
      if (c < C) {
        a[u] = ld4_stream(arow + c);
        if (score) o[u] = ld4_stream(vrow + c);
        if (xrow) xv[u] = ld4_stream(xrow + c);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 128 * u;
      if (c < C) {
        if (score) {
          num += fabsf(a[u].x - o[u].x) + fabsf(a[u].y - o[u].y) + fabsf(a[u].z - o[u].z) + fabsf(a[u].w - o[u].w);
          den += fabsf(o[u].x) + fabsf(o[u].y) + fabsf(o[u].z) + fabsf(o[u].w);
        }
        __stcs(reinterpret_cast<float4*>(vrow + c), a[u]);
        if (xrow) {
          float4 t = xv[u];
          t.x = fmaf(dsigma, a[u].x, t.x);
          t.y = fmaf(dsigma, a[u].y, t.y);
          t.z = fmaf(dsigma, a[u].z, t.z);
          t.w = fmaf(dsigma, a[u].w, t.w);
          __stcs(reinterpret_cast<float4*>(xrow + c), t);
        }
      }
    }
  }
  if (score) {
    num = warp_sum(num);
    den = warp_sum(den);
    if (lane == 0) score[n] = num / (den + kScoreEps);
  }
}

// §2.1 score on its own: score[n] = sum|v_new - v_prev| / (sum|v_prev| + eps).
__global__ void __launch_bounds__(256) k_l1_score(const float* __restrict__ vnew, const float* __restrict__ vprev,
                                                  int N, int C, float* __restrict__ score) {
  pdl_prologue();
  const int n = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  const float* a = vnew + (size_t)n * C;
  const float* b = vprev + (size_t)n * C;
  float num = 0.f, den = 0.f;
  for (int c = 4 * lane; c < C; c += 128) {
    const float4 u = ld4(a + c), v = ld4(b + c);
    num += fabsf(u.x - v.x) + fabsf(u.y - v.y) + fabsf(u.z - v.z) + fabsf(u.w - v.w);
    den += fabsf(v.x) + fabsf(v.y) + fabsf(v.z) + fabsf(v.w);
  }
  num = warp_sum(num);
  den = warp_sum(den);
  if (lane == 0) score[n] = num / (den + kScoreEps);
}


// ------------------------------------------------------------------ LayerNorm rows
// h[r] = LN(X[r]) * mul' + add over D channels (biased variance, eps 1e-6), with
// mul' = 1 + mul (modulation scale) when mul_plus_one, else mul (affine gain).
// When x_src is given the row is first gathered: X[r] = x_src[idx[r]] (and
// written to X).  VPT float4 per lane are kept in registers (D = 128 * VPT).
template <int VPT, typename TOut>
__global__ void __launch_bounds__(256) k_ln_rows(float* __restrict__ X, const float* __restrict__ x_src,
                                                 const int* __restrict__ idx, int M, int N,
                                                 const float* __restrict__ mul, const float* __restrict__ add,
                                                 int mul_plus_one, TOut* __restrict__ h) {
  pdl_prologue();
  constexpr int D = VPT * 128;
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const float* src = X + (size_t)r * D;
  if (x_src) {
    const int n = idx[r];
    if (n < 0 || n >= N) {
      if (lane == 0) flag_error(HSA_EINDEX);
      return;
    }
    src = x_src + (size_t)n * D;
  }
  float4 v[VPT];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    v[i] = ld4(src + (i * 32 + lane) * 4);
    s += v[i].x + v[i].y + v[i].z + v[i].w;
  }
  if (x_src) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) st4(X + (size_t)r * D + (i * 32 + lane) * 4, v[i]);
  }
  const float mean = warp_sum(s) * (1.0f / D);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
    q += a * a + b * b + c * c + d * d;
  }
  const float rstd = rsqrtf(warp_sum(q) * (1.0f / D) + kNormEps);
  const float one = mul_plus_one ? 1.f : 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = (i * 32 + lane) * 4;
    const float4 g = ld4(mul + c), b = ld4(add + c);
    float4 y;
    y.x = (v[i].x - mean) * rstd * (one + g.x) + b.x;
    y.y = (v[i].y - mean) * rstd * (one + g.y) + b.y;
    y.z = (v[i].z - mean) * rstd * (one + g.z) + b.z;
    y.w = (v[i].w - mean) * rstd * (one + g.w) + b.w;
    store4(h + (size_t)r * D + c, y);
  }
}

// Same for any D % 128 == 0, streaming the row from global memory three times.
template <typename TOut>
__global__ void __launch_bounds__(256) k_ln_rows_any(float* __restrict__ X, const float* __restrict__ x_src,
                                                     const int* __restrict__ idx, int M, int N, int D,
                                                     const float* __restrict__ mul, const float* __restrict__ add,
                                                     int mul_plus_one, TOut* __restrict__ h) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const float* src = X + (size_t)r * D;
  if (x_src) {
    const int n = idx[r];
    if (n < 0 || n >= N) {
      if (lane == 0) flag_error(HSA_EINDEX);
      return;
    }
    src = x_src + (size_t)n * D;
  }
  float s = 0.f;
  for (int c = 4 * lane; c < D; c += 128) {
    const float4 v = ld4(src + c);
    s += v.x + v.y + v.z + v.w;
    if (x_src) st4(X + (size_t)r * D + c, v);
  }
  const float mean = warp_sum(s) / D;
  float q = 0.f;
  for (int c = 4 * lane; c < D; c += 128) {
    const float4 v = ld4(src + c);
    const float a = v.x - mean, b = v.y - mean, cc = v.z - mean, d = v.w - mean;
    q += a * a + b * b + cc * cc + d * d;
  }
  const float rstd = rsqrtf(warp_sum(q) / D + kNormEps);
  const float one = mul_plus_one ? 1.f : 0.f;
  for (int c = 4 * lane; c < D; c += 128) {
    const float4 v = ld4(src + c), g = ld4(mul + c), b = ld4(add + c);
    float4 y;
    y.x = (v.x - mean) * rstd * (one + g.x) + b.x;
    y.y = (v.y - mean) * rstd * (one + g.y) + b.y;
    y.z = (v.z - mean) * rstd * (one + g.z) + b.z;
    y.w = (v.w - mean) * rstd * (one + g.w) + b.w;
    store4(h + (size_t)r * D + c, y);
  }
}

// ------------------------------------------------------------------ 3D RoPE
// Channel c (0..127) of a head belongs to axis 0 (frame) for c < 44, 1 (row) for
// c < 86, else 2 (column); pair j of an axis segment of width w turns by
// pos_axis * 10000^(-2j/w).  Returns (cos, sin) of pair (c, c+1), c even.
__device__ __forceinline__ float2 rope_cs(int c, int pf, int ph, int pw) {
  int axis, j, w;
  if (c < 44) { axis = 0; j = c >> 1; w = 44; }
  else if (c < 86) { axis = 1; j = (c - 44) >> 1; w = 42; }
  else { axis = 2; j = (c - 86) >> 1; w = 42; }
  const float p = (float)(axis == 0 ? pf : (axis == 1 ? ph : pw));
  // 10000^(-2j/w) = 2^(-(2j/w) * log2(10000))
  const float inv_freq = exp2f(-(float)(2 * j) / (float)w * 13.287712379549449f);
  // angle reduced to [-pi, pi] by k multiples of 2 pi, 2 pi split into a float head and its
  // remainder (Cody-Waite), then the fast intrinsic; angles here are position x frequency,
  // below ~100 rad, so the reduction error stays near 1e-6
  const float ang = p * inv_freq;
  const float k = rintf(ang * 0.15915494309189535f);
  const float r = fmaf(-k, -1.7484556025237907e-07f, fmaf(-k, 6.2831854820251465f, ang));
  float sn, cs;
  __sincosf(r, &sn, &cs);
  return make_float2(cs, sn);
}

// One warp per active row r: q, k <- RMSNorm over all D channels times g_q / g_k,
// then RoPE at the token's (frame, row, column); Q[r] = q (compacted),
// Kc[idx[r]] = k, Vc[idx[r]] = v.  Rows of skipped tokens are never touched.
template <int VPT, typename TIn, typename TOut>
__global__ void __launch_bounds__(256) k_qk_norm_rope(const TIn* __restrict__ qkv, const int* __restrict__ idx,
                                                      const int* __restrict__ pos, int M, int N,
                                                      const float* __restrict__ g_q, const float* __restrict__ g_k,
                                                      TOut* __restrict__ Q, TOut* __restrict__ Kc,
                                                      TOut* __restrict__ Vc) {
  pdl_prologue();
  constexpr int D = VPT * 128;
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const int n = idx[r];
  if (n < 0 || n >= N) {
    if (lane == 0) flag_error(HSA_EINDEX);
    return;
  }
  const int pf = pos[3 * n + 0], ph = pos[3 * n + 1], pw = pos[3 * n + 2];
  const TIn* row = qkv + (size_t)r * 3 * D;
  // q and k stay in registers in their input type (bf16: 8 bytes per 4 channels) and v is
  // copied to the cache in this first pass, so the second pass holds only q, k and the
  // gains: 128 registers instead of 189 for D = 1536, two CTAs per SM instead of one
  using Raw = typename std::conditional<sizeof(TIn) == 2, uint2, float4>::type;
  Raw q[VPT], k[VPT];
  float sq = 0.f, sk = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = (i * 32 + lane) * 4;
    q[i] = *reinterpret_cast<const Raw*>(row + c);
    k[i] = *reinterpret_cast<const Raw*>(row + D + c);
    store4(Vc + (size_t)n * D + c, load4(row + 2 * D + c));
    const float4 a = widen4(q[i]), b = widen4(k[i]);
    sq += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
    sk += b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
  }
  const float rq = rsqrtf(warp_sum(sq) * (1.0f / D) + kNormEps);
  const float rk = rsqrtf(warp_sum(sk) * (1.0f / D) + kNormEps);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = (i * 32 + lane) * 4;
    const int ch = c & 127;  // channel within the head; c..c+3 stay in one head
    const float4 gq = ld4(g_q + c), gk = ld4(g_k + c);
    const float4 qv = widen4(q[i]), kv = widen4(k[i]);
    const float4 a = make_float4(qv.x * rq * gq.x, qv.y * rq * gq.y, qv.z * rq * gq.z, qv.w * rq * gq.w);
    const float4 b = make_float4(kv.x * rk * gk.x, kv.y * rk * gk.y, kv.z * rk * gk.z, kv.w * rk * gk.w);
    const float2 t0 = rope_cs(ch, pf, ph, pw), t1 = rope_cs(ch + 2, pf, ph, pw);
    float4 qo, ko;
    qo.x = a.x * t0.x - a.y * t0.y;  qo.y = a.x * t0.y + a.y * t0.x;
    qo.z = a.z * t1.x - a.w * t1.y;  qo.w = a.z * t1.y + a.w * t1.x;
    ko.x = b.x * t0.x - b.y * t0.y;  ko.y = b.x * t0.y + b.y * t0.x;
    ko.z = b.z * t1.x - b.w * t1.y;  ko.w = b.z * t1.y + b.w * t1.x;
    store4(Q + (size_t)r * D + c, qo);
    store4(Kc + (size_t)n * D + c, ko);
  }
}

// out[r] = RMSNorm(in[r]) * g over D (g == nullptr: plain copy).  in rows are
// `in_stride` elements apart (a slice of a wider GEMM output).
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) k_rms_rows(const TIn* __restrict__ in, int in_stride, int M, int D,
                                                  const float* __restrict__ g, TOut* __restrict__ out) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const TIn* row = in + (size_t)r * in_stride;
  float scale = 1.f;
  if (g) {
    float s = 0.f;
    for (int c = 4 * lane; c < D; c += 128) {
      const float4 v = load4(row + c);
      s += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    scale = rsqrtf(warp_sum(s) / D + kNormEps);
  }
  for (int c = 4 * lane; c < D; c += 128) {
    float4 v = load4(row + c);
    if (g) {
      const float4 w = ld4(g + c);
      v = make_float4(v.x * scale * w.x, v.y * scale * w.y, v.z * scale * w.z, v.w * scale * w.w);
    }
    store4(out + (size_t)r * D + c, v);
  }
}


// k_qk_norm_rope for any D % 128 == 0: the row is read twice instead of held in registers.
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) k_qk_norm_rope_any(const TIn* __restrict__ qkv, const int* __restrict__ idx,
                                                          const int* __restrict__ pos, int M, int N, int D,
                                                          const float* __restrict__ g_q,
                                                          const float* __restrict__ g_k, TOut* __restrict__ Q,
                                                          TOut* __restrict__ Kc, TOut* __restrict__ Vc) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const int n = idx[r];
  if (n < 0 || n >= N) {
    if (lane == 0) flag_error(HSA_EINDEX);
    return;
  }
  const int pf = pos[3 * n + 0], ph = pos[3 * n + 1], pw = pos[3 * n + 2];
  const TIn* row = qkv + (size_t)r * 3 * D;
  float sq = 0.f, sk = 0.f;
  for (int c = 4 * lane; c < D; c += 128) {
    const float4 q = load4(row + c), k = load4(row + D + c);
    sq += q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
    sk += k.x * k.x + k.y * k.y + k.z * k.z + k.w * k.w;
  }
  const float rq = rsqrtf(warp_sum(sq) / D + kNormEps);
  const float rk = rsqrtf(warp_sum(sk) / D + kNormEps);
  for (int c = 4 * lane; c < D; c += 128) {
    const int ch = c & 127;
    const float4 q = load4(row + c), k = load4(row + D + c);
    const float4 gq = ld4(g_q + c), gk = ld4(g_k + c);
    const float4 a = make_float4(q.x * rq * gq.x, q.y * rq * gq.y, q.z * rq * gq.z, q.w * rq * gq.w);
    const float4 b = make_float4(k.x * rk * gk.x, k.y * rk * gk.y, k.z * rk * gk.z, k.w * rk * gk.w);
    const float2 t0 = rope_cs(ch, pf, ph, pw), t1 = rope_cs(ch + 2, pf, ph, pw);
    float4 qo, ko;
    qo.x = a.x * t0.x - a.y * t0.y;  qo.y = a.x * t0.y + a.y * t0.x;
    qo.z = a.z * t1.x - a.w * t1.y;  qo.w = a.z * t1.y + a.w * t1.x;
    ko.x = b.x * t0.x - b.y * t0.y;  ko.y = b.x * t0.y + b.y * t0.x;
    ko.z = b.z * t1.x - b.w * t1.y;  ko.w = b.z * t1.y + b.w * t1.x;
    store4(Q + (size_t)r * D + c, qo);
    store4(Kc + (size_t)n * D + c, ko);
    store4(Vc + (size_t)n * D + c, load4(row + 2 * D + c));
  }
}

// out[r] = x[idx[r]] converted to TOut (C % 4 == 0); one warp per row.
template <typename TOut>
__global__ void __launch_bounds__(256) k_gather_rows(const float* __restrict__ x, const int* __restrict__ idx, int M,
                                                     int N, int C, TOut* __restrict__ out) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const int n = idx[r];
  if (n < 0 || n >= N) {
    if (lane == 0) flag_error(HSA_EINDEX);
    return;
  }
  for (int c = 4 * lane; c < C; c += 128) store4(out + (size_t)r * C + c, ld4(x + (size_t)n * C + c));
}

}  // namespace hsa

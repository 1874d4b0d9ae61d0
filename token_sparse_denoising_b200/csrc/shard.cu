// shard.cu -- building blocks of a DiT block whose heads are split over G GPUs (head parallelism).
//
// With the heads split, a rank holds only its heads' channels of q and k, while the q/k RMSNorm
// of the block runs over all D channels of a row (HSA summary §2.2 with the Wan-style block: the
// norm precedes the head split).  The norm therefore takes the row sums of squares from outside:
// each rank computes its channels' partial sums (k_row_sumsq), the ranks add them (a collective
// of M floats), and the normalisation, RoPE and cache scatter run on the local channels with the
// global sums (k_qk_norm_rope_ext, k_rms_rows_ext).  The output projection and FFN2 of a rank
// produce partial sums of the full-width result; after the ranks reduce them, k_gated_residual
// adds bias and gate into the rank's rows of the residual stream.
//
//   k_row_sumsq         ss[r] = sum_c in[r, c]^2 over D channels
//   k_qk_norm_rope_ext  q, k <- x * rsqrt(ss / D_total + eps) * g, RoPE, Q compact, K/V scattered
//   k_rms_rows_ext      out = in * rsqrt(ss / D_total + eps) * g (or a plain copy)
//   k_gated_residual    X += gate * (y + b)
#include "common.cuh"

namespace hsa {

template <typename T>
__global__ void __launch_bounds__(256) k_row_sumsq(const T* __restrict__ in, int in_stride, int M, int D,
                                                   float* __restrict__ ss, int ss_stride) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const T* row = in + (size_t)r * in_stride;
  float s = 0.f;
  for (int c = 4 * lane; c < D; c += 128) {
    const float4 v = load4(row + c);
    s += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  s = warp_sum(s);
  if (lane == 0) ss[(size_t)r * ss_stride] = s;
}

// One warp per row r of qkv = [q | k | v], each Dl channels (whole heads of 128): q and k are
// normalised with the row sums of squares over all D_total channels, ss[2r] (q) and ss[2r+1]
// (k), times their gains, then turned by 3D RoPE at the token's position; Q[r] = q,
// Kc[idx[r]] = k, Vc[idx[r]] = v (rows Dl wide).
template <typename T>
__global__ void __launch_bounds__(256) k_qk_norm_rope_ext(const T* __restrict__ qkv, const int* __restrict__ idx,
                                                          const int* __restrict__ pos, int M, int N, int Dl,
                                                          float inv_d, const float* __restrict__ ss,
                                                          const float* __restrict__ g_q,
                                                          const float* __restrict__ g_k, T* __restrict__ Q,
                                                          T* __restrict__ Kc, T* __restrict__ Vc) {
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
  const T* row = qkv + (size_t)r * 3 * Dl;
  const float rq = rsqrtf(ss[2 * (size_t)r] * inv_d + kNormEps);
  const float rk = rsqrtf(ss[2 * (size_t)r + 1] * inv_d + kNormEps);
  for (int c = 4 * lane; c < Dl; c += 128) {
    const int ch = c & 127;
    const float4 q = load4(row + c), k = load4(row + Dl + c);
    const float4 gq = ld4(g_q + c), gk = ld4(g_k + c);
    const float4 a = make_float4(q.x * rq * gq.x, q.y * rq * gq.y, q.z * rq * gq.z, q.w * rq * gq.w);
    const float4 b = make_float4(k.x * rk * gk.x, k.y * rk * gk.y, k.z * rk * gk.z, k.w * rk * gk.w);
    const float2 t0 = rope_cs(ch, pf, ph, pw), t1 = rope_cs(ch + 2, pf, ph, pw);
    float4 qo, ko;
    qo.x = a.x * t0.x - a.y * t0.y;  qo.y = a.x * t0.y + a.y * t0.x;
    qo.z = a.z * t1.x - a.w * t1.y;  qo.w = a.z * t1.y + a.w * t1.x;
    ko.x = b.x * t0.x - b.y * t0.y;  ko.y = b.x * t0.y + b.y * t0.x;
    ko.z = b.z * t1.x - b.w * t1.y;  ko.w = b.z * t1.y + b.w * t1.x;
    store4(Q + (size_t)r * Dl + c, qo);
    store4(Kc + (size_t)n * Dl + c, ko);
    store4(Vc + (size_t)n * Dl + c, load4(row + 2 * Dl + c));
  }
}

// out[r] = in[r] * rsqrt(ss[r * ss_stride] / D_total + eps) * g; with ss == nullptr a plain copy.
template <typename T>
__global__ void __launch_bounds__(256) k_rms_rows_ext(const T* __restrict__ in, int in_stride, int M, int D,
                                                      float inv_d, const float* __restrict__ ss, int ss_stride,
                                                      const float* __restrict__ g, T* __restrict__ out) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  const T* row = in + (size_t)r * in_stride;
  const float scale = ss ? rsqrtf(ss[(size_t)r * ss_stride] * inv_d + kNormEps) : 1.f;
  for (int c = 4 * lane; c < D; c += 128) {
    float4 v = load4(row + c);
    if (ss) {
      const float4 w = g ? ld4(g + c) : make_float4(1.f, 1.f, 1.f, 1.f);
      v = make_float4(v.x * scale * w.x, v.y * scale * w.y, v.z * scale * w.z, v.w * scale * w.w);
    }
    store4(out + (size_t)r * D + c, v);
  }
}

// X[r] += gate * (y[r] + b) over D channels (gate, b may be null: 1, 0).
__global__ void __launch_bounds__(256) k_gated_residual(float* __restrict__ X, const float* __restrict__ y, int M,
                                                        int D, const float* __restrict__ b,
                                                        const float* __restrict__ gate) {
  pdl_prologue();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= M) return;
  float* xr = X + (size_t)r * D;
  const float* yr = y + (size_t)r * D;
  for (int c = 4 * lane; c < D; c += 128) {
    float4 x = ld4(xr + c);
    const float4 v = ld4(yr + c);
    const float4 bb = b ? ld4(b + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 gg = gate ? ld4(gate + c) : make_float4(1.f, 1.f, 1.f, 1.f);
    x.x = fmaf(gg.x, v.x + bb.x, x.x);
    x.y = fmaf(gg.y, v.y + bb.y, x.y);
    x.z = fmaf(gg.z, v.z + bb.z, x.z);
    x.w = fmaf(gg.w, v.w + bb.w, x.w);
    st4(xr + c, x);
  }
}

static inline unsigned shard_warp_blocks(long long rows) { return (unsigned)((rows * 32 + 255) / 256); }
// 4-element vectors: 16 bytes for float32, 8 for bf16
static inline bool vec_aligned(const void* p, int dtype) {
  return (reinterpret_cast<uintptr_t>(p) & (dtype == HSA_BF16 ? 7u : 15u)) == 0;
}

}  // namespace hsa

using namespace hsa;

extern "C" int hsa_layernorm_rows(float* d_X, const float* d_x_src, const int32_t* d_idx, int M, int N, int D,
                                  const float* d_mul, const float* d_add, int modulate, int dtype, void* d_out,
                                  void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "layernorm_rows: unknown dtype");
  if (M < 0 || D <= 0 || D % 128) return set_error(HSA_EINVAL, "layernorm_rows: need M >= 0 and D % 128 == 0");
  if (M == 0) return HSA_OK;
  if (!d_X || !d_mul || !d_add || !d_out || !aligned16(d_X) || !aligned16(d_out) || !aligned16(d_mul) ||
      !aligned16(d_add))
    return set_error(HSA_EINVAL, "layernorm_rows: null or misaligned pointer");
  if (d_x_src && (!d_idx || !aligned16(d_x_src) || N < 1))
    return set_error(HSA_EINVAL, "layernorm_rows: a gather needs the index list and N >= 1");
  cudaStream_t st = as_stream(stream);
  if (dtype == HSA_BF16)
    return launch_ln(d_X, d_x_src, d_idx, M, N, D, d_mul, d_add, modulate ? 1 : 0,
                     static_cast<__nv_bfloat16*>(d_out), st);
  return launch_ln(d_X, d_x_src, d_idx, M, N, D, d_mul, d_add, modulate ? 1 : 0, static_cast<float*>(d_out), st);
}

extern "C" int hsa_row_sumsq(const void* d_in, int in_stride, int M, int D, int dtype, float* d_ss, int ss_stride,
                             void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "row_sumsq: unknown dtype");
  if (M < 0 || D <= 0 || D % 4 || in_stride < D || in_stride % 4 || ss_stride < 1)
    return set_error(HSA_EINVAL, "row_sumsq: need D % 4 == 0, in_stride >= D, in_stride % 4 == 0");
  if (M == 0) return HSA_OK;
  if (!d_in || !d_ss || !vec_aligned(d_in, dtype)) return set_error(HSA_EINVAL, "row_sumsq: null or misaligned pointer");
  cudaStream_t st = as_stream(stream);
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  if (dtype == HSA_BF16)
    launch(k_row_sumsq<__nv_bfloat16>, shard_warp_blocks(M), 256, 0, st,
           static_cast<const __nv_bfloat16*>(d_in), in_stride, M, D, d_ss, ss_stride);
  else
    launch(k_row_sumsq<float>, shard_warp_blocks(M), 256, 0, st, static_cast<const float*>(d_in), in_stride, M, D,
           d_ss, ss_stride);
  count_launch(1);
  return check_launch("row_sumsq launch");
}

extern "C" int hsa_qk_norm_rope_ext(const void* d_qkv, int M, int N, int Dl, int D_total, const float* d_ss,
                                    const float* d_g_q, const float* d_g_k, const int32_t* d_idx,
                                    const int32_t* d_pos, int dtype, void* d_Q, void* d_kcache, void* d_vcache,
                                    void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "qk_norm_rope_ext: unknown dtype");
  if (M < 0 || N < 1 || M > N || Dl <= 0 || Dl % 128 || D_total < Dl)
    return set_error(HSA_EINVAL, "qk_norm_rope_ext: need 0 <= M <= N, Dl % 128 == 0, D_total >= Dl");
  if (M == 0) return HSA_OK;
  if (!d_qkv || !d_ss || !d_g_q || !d_g_k || !d_idx || !d_pos || !d_Q || !d_kcache || !d_vcache ||
      !aligned16(d_qkv) || !aligned16(d_Q) || !aligned16(d_kcache) || !aligned16(d_vcache) || !aligned16(d_g_q) ||
      !aligned16(d_g_k))
    return set_error(HSA_EINVAL, "qk_norm_rope_ext: null or misaligned pointer");
  cudaStream_t st = as_stream(stream);
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  const float inv_d = 1.0f / (float)D_total;
  if (dtype == HSA_BF16) {
    using T = __nv_bfloat16;
    launch(k_qk_norm_rope_ext<T>, shard_warp_blocks(M), 256, 0, st, static_cast<const T*>(d_qkv), d_idx, d_pos, M, N,
           Dl, inv_d, d_ss, d_g_q, d_g_k, static_cast<T*>(d_Q), static_cast<T*>(d_kcache), static_cast<T*>(d_vcache));
  } else {
    launch(k_qk_norm_rope_ext<float>, shard_warp_blocks(M), 256, 0, st, static_cast<const float*>(d_qkv), d_idx, d_pos,
           M, N, Dl, inv_d, d_ss, d_g_q, d_g_k, static_cast<float*>(d_Q), static_cast<float*>(d_kcache),
           static_cast<float*>(d_vcache));
  }
  count_launch(1);
  return check_launch("qk_norm_rope_ext launch");
}

extern "C" int hsa_rms_rows_ext(const void* d_in, int in_stride, int M, int D, int D_total, const float* d_ss,
                                int ss_stride, const float* d_g, int dtype, void* d_out, void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "rms_rows_ext: unknown dtype");
  if (M < 0 || D <= 0 || D % 4 || in_stride < D || in_stride % 4 || D_total < D || (d_ss && ss_stride < 1))
    return set_error(HSA_EINVAL, "rms_rows_ext: need D % 4 == 0, in_stride >= D, D_total >= D");
  if (M == 0) return HSA_OK;
  if (!d_in || !d_out || !vec_aligned(d_in, dtype) || !vec_aligned(d_out, dtype) || (d_g && !aligned16(d_g)))
    return set_error(HSA_EINVAL, "rms_rows_ext: null or misaligned pointer");
  cudaStream_t st = as_stream(stream);
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  const float inv_d = 1.0f / (float)D_total;
  if (dtype == HSA_BF16) {
    using T = __nv_bfloat16;
    launch(k_rms_rows_ext<T>, shard_warp_blocks(M), 256, 0, st, static_cast<const T*>(d_in), in_stride, M, D, inv_d,
           d_ss, ss_stride, d_g, static_cast<T*>(d_out));
  } else {
    launch(k_rms_rows_ext<float>, shard_warp_blocks(M), 256, 0, st, static_cast<const float*>(d_in), in_stride, M, D,
           inv_d, d_ss, ss_stride, d_g, static_cast<float*>(d_out));
  }
  count_launch(1);
  return check_launch("rms_rows_ext launch");
}

extern "C" int hsa_gated_residual(float* d_X, const float* d_y, int M, int D, const float* d_b, const float* d_gate,
                                  void* stream) {
  if (M < 0 || D <= 0 || D % 4) return set_error(HSA_EINVAL, "gated_residual: need M >= 0 and D % 4 == 0");
  if (M == 0) return HSA_OK;
  if (!d_X || !d_y || !aligned16(d_X) || !aligned16(d_y) || (d_b && !aligned16(d_b)) ||
      (d_gate && !aligned16(d_gate)))
    return set_error(HSA_EINVAL, "gated_residual: null or misaligned pointer");
  cudaStream_t st = as_stream(stream);
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  launch(k_gated_residual, shard_warp_blocks(M), 256, 0, st, d_X, d_y, M, D, d_b, d_gate);
  count_launch(1);
  return check_launch("gated_residual launch");
}

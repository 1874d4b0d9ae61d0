// api.cu -- the C ABI entry points of libhsa (include/hsa.h): argument checks,
// workspace carving and the launch sequence of one HSA layer step.
#include <string>

#include "common.cuh"

namespace hsa {

int gemm_bf16(const void* A, int M, int K, const void* W, int Nout, const float* bias, int epi, const float* gate,
              void* out, cudaStream_t st);
int gemm_f32(const float* A, int M, int K, const float* W, int Nout, const float* bias, int epi, const float* gate,
             float* out, cudaStream_t st);
int attention_bf16(const void* Q, int M, const void* K, const void* V, int L, int H, void* O, cudaStream_t st,
                   void* ws, size_t ws_bytes);
size_t attention_split_bytes(int M, int L, int H);
int attention_f32(const float* Q, int M, const float* K, const float* V, int L, int H, float* O, cudaStream_t st,
                  void* ws, size_t ws_bytes);
size_t attention_f32_split_bytes(int M, int L, int H);

static inline unsigned warp_blocks(long long rows) { return (unsigned)((rows * 32 + 255) / 256); }
static inline size_t esize(int dtype) { return dtype == HSA_BF16 ? 2 : 4; }

#define HSA_TRY(x)            \
  do {                        \
    const int rc_ = (x);      \
    if (rc_ != HSA_OK) return rc_; \
  } while (0)

// LayerNorm rows, dispatched on D = 128 * VPT.
template <typename TOut>
static int launch_ln(float* X, const float* x_src, const int* idx, int M, int N, int D, const float* mul,
                     const float* add, int plus_one, TOut* h, cudaStream_t st) {
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  const unsigned g = warp_blocks(M);
  switch (D / 128 * (D % 128 == 0)) {
    case 1: launch(k_ln_rows<1, TOut>, g, 256, 0, st, X, x_src, idx, M, N, mul, add, plus_one, h); break;
    case 2: launch(k_ln_rows<2, TOut>, g, 256, 0, st, X, x_src, idx, M, N, mul, add, plus_one, h); break;
    case 4: launch(k_ln_rows<4, TOut>, g, 256, 0, st, X, x_src, idx, M, N, mul, add, plus_one, h); break;
    case 8: launch(k_ln_rows<8, TOut>, g, 256, 0, st, X, x_src, idx, M, N, mul, add, plus_one, h); break;
    case 12: launch(k_ln_rows<12, TOut>, g, 256, 0, st, X, x_src, idx, M, N, mul, add, plus_one, h); break;
    case 16: launch(k_ln_rows<16, TOut>, g, 256, 0, st, X, x_src, idx, M, N, mul, add, plus_one, h); break;
    default: launch(k_ln_rows_any<TOut>, g, 256, 0, st, X, x_src, idx, M, N, D, mul, add, plus_one, h); break;
  }
  count_launch(1);
  return check_launch("layernorm launch");
}

template <typename T>
static int launch_qk_rope(const T* qkv, const int* idx, const int* pos, int M, int N, int D, const float* g_q,
                          const float* g_k, T* Q, T* Kc, T* Vc, cudaStream_t st) {
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  const unsigned g = warp_blocks(M);
  switch (D / 128) {
    case 1: launch(k_qk_norm_rope<1, T, T>, g, 256, 0, st, qkv, idx, pos, M, N, g_q, g_k, Q, Kc, Vc); break;
    case 2: launch(k_qk_norm_rope<2, T, T>, g, 256, 0, st, qkv, idx, pos, M, N, g_q, g_k, Q, Kc, Vc); break;
    case 4: launch(k_qk_norm_rope<4, T, T>, g, 256, 0, st, qkv, idx, pos, M, N, g_q, g_k, Q, Kc, Vc); break;
    case 8: launch(k_qk_norm_rope<8, T, T>, g, 256, 0, st, qkv, idx, pos, M, N, g_q, g_k, Q, Kc, Vc); break;
    case 12: launch(k_qk_norm_rope<12, T, T>, g, 256, 0, st, qkv, idx, pos, M, N, g_q, g_k, Q, Kc, Vc); break;
    default: launch(k_qk_norm_rope_any<T, T>, g, 256, 0, st, qkv, idx, pos, M, N, D, g_q, g_k, Q, Kc, Vc); break;
  }
  count_launch(1);
  return check_launch("qk norm / rope launch");
}

template <typename T>
static int launch_rms(const T* in, int in_stride, int M, int D, const float* g, T* out, cudaStream_t st) {
  if (M <= 0) return HSA_OK;
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  launch(k_rms_rows<T, T>, warp_blocks(M), 256, 0, st, in, in_stride, M, D, g, out);
  count_launch(1);
  return check_launch("rms rows launch");
}

static int linear(const void* x, int M, int K, const void* W, int Nout, const float* b, int dtype, int epi,
                  const float* gate, void* y, cudaStream_t st) {
  if (dtype == HSA_BF16) return gemm_bf16(x, M, K, W, Nout, b, epi, gate, y, st);
  const int e = epi == HSA_EPI_GELU ? 1 : (epi == HSA_EPI_RESID ? 2 : 0);
  return gemm_f32(static_cast<const float*>(x), M, K, static_cast<const float*>(W), Nout, b, e, gate,
                  static_cast<float*>(y), st);
}

// ws (may be null): scratch for splitting the tail units of the bf16 kernel over key ranges
static int attention(const void* q, int M, const void* k, const void* v, int L, int H, int dtype, void* o,
                     cudaStream_t st, void* ws = nullptr, size_t ws_bytes = 0) {
  if (dtype == HSA_BF16) return attention_bf16(q, M, k, v, L, H, o, st, ws, ws_bytes);
  return attention_f32(static_cast<const float*>(q), M, static_cast<const float*>(k),
                       static_cast<const float*>(v), L, H, static_cast<float*>(o), st, ws, ws_bytes);
}

}  // namespace hsa

using namespace hsa;

// ------------------------------------------------------------------ §2.1 score, §2.3 Euler
extern "C" int hsa_l1_score(const float* d_v_new, const float* d_v_prev, int N, int C, float* d_score,
                            void* stream) {
  if (N < 0 || C <= 0 || C % 4) return set_error(HSA_EINVAL, "l1_score: need N >= 0 and C % 4 == 0");
  if (N == 0) return HSA_OK;
  if (!d_v_new || !d_v_prev || !d_score || !aligned16(d_v_new) || !aligned16(d_v_prev))
    return set_error(HSA_EINVAL, "l1_score: null or misaligned pointer");
  ScopedTiming timing(HSA_KCLASS_OTHER, as_stream(stream));
  launch(k_l1_score, warp_blocks(N), 256, 0, as_stream(stream), d_v_new, d_v_prev, N, C, d_score);
  count_launch(1);
  return check_launch("l1_score launch");
}

extern "C" int hsa_euler_update(float* d_x, float* d_vhat, const float* d_vA, const int32_t* d_idx, int M, int N,
                                int C, float dsigma, float* d_score, void* stream) {
  if (N <= 0 || C <= 0 || C % 4 || M < 0 || M > N)
    return set_error(HSA_EINVAL, "euler: need N > 0, C % 4 == 0 and 0 <= M <= N");
  if (!d_x || !d_vhat || !aligned16(d_x) || !aligned16(d_vhat))
    return set_error(HSA_EINVAL, "euler: null or misaligned x / v_hat");
  if (M > 0 && (!d_vA || !d_idx || !aligned16(d_vA))) return set_error(HSA_EINVAL, "euler: null v_A or idx");
  cudaStream_t st = as_stream(stream);
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  if (M == N) {
    // every token active: scatter, score and Euler in one pass over the rows
    launch(k_scatter_vhat, warp_blocks(M), 256, 0, st, d_vhat, d_vA, d_idx, M, N, C, d_score, d_x, dsigma);
    count_launch(1);
    return check_launch("euler (full step) launch");
  }
  if (M > 0) {
    launch(k_scatter_vhat, warp_blocks(M), 256, 0, st, d_vhat, d_vA, d_idx, M, N, C, d_score, nullptr, dsigma);
    count_launch(1);
    HSA_TRY(check_launch("v_hat scatter launch"));
  }
  const size_t n4 = (size_t)N * C / 4;
  // up to 4 float4 per thread per pass; the same number of 256-thread blocks on every SM (at most
  // 8, a full SM), so no SM holds one block more than another
  const size_t sms = (size_t)num_sms();
  const size_t per_sm = ((n4 + 1023) / 1024 + sms - 1) / sms;
  launch(k_euler, (unsigned)(sms * (per_sm < 8 ? per_sm : 8)), 256, 0, st, d_x, d_vhat, n4, dsigma);
  count_launch(1);
  return check_launch("euler launch");
}

// ------------------------------------------------------------------ building blocks
extern "C" int hsa_linear(const void* d_x, int M, int Kin, const void* d_w, int Nout, const float* d_b, int dtype,
                          int epilogue, const float* d_gate, void* d_y, void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "linear: unknown dtype");
  if (epilogue < HSA_EPI_STORE || epilogue > HSA_EPI_F32) return set_error(HSA_EINVAL, "linear: unknown epilogue");
  if (M < 0) return set_error(HSA_EINVAL, "linear: M < 0");
  return linear(d_x, M, Kin, d_w, Nout, d_b, dtype, epilogue, d_gate, d_y, as_stream(stream));
}

extern "C" int hsa_attention(const void* d_q, int M, const void* d_k, const void* d_v, int L, int H, int dtype,
                             void* d_o, void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "attention: unknown dtype");
  if (M < 0) return set_error(HSA_EINVAL, "attention: M < 0");
  return attention(d_q, M, d_k, d_v, L, H, dtype, d_o, as_stream(stream));
}

extern "C" size_t hsa_attention_workspace_size(int M, int L, int H, int dtype) {
  return dtype == HSA_BF16 ? attention_split_bytes(M, L, H) : attention_f32_split_bytes(M, L, H);
}

extern "C" int hsa_attention_ws(const void* d_q, int M, const void* d_k, const void* d_v, int L, int H, int dtype,
                                void* d_o, void* d_ws, size_t ws_bytes, void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "attention: unknown dtype");
  if (M < 0) return set_error(HSA_EINVAL, "attention: M < 0");
  if (d_ws && !aligned16(d_ws)) return set_error(HSA_EINVAL, "attention: misaligned workspace");
  return attention(d_q, M, d_k, d_v, L, H, dtype, d_o, as_stream(stream), d_ws, ws_bytes);
}

// ------------------------------------------------------------------ §2.2 context keys / values
extern "C" size_t hsa_context_kv_workspace_size(int L, int D) {
  if (L <= 0 || D <= 0) return 0;
  return align256((size_t)L * 2 * D * 4);
}

namespace hsa {
// Scratch the context projection really uses: the L x 2D projection in the path's own dtype.
// hsa_context_kv_workspace_size reports the fp32 size, which covers both dtypes.
size_t context_kv_scratch_bytes(int L, int D, int dtype) {
  if (L <= 0 || D <= 0) return 0;
  return align256((size_t)L * 2 * D * esize(dtype));
}
}  // namespace hsa

extern "C" int hsa_context_kv(const void* d_ctx, int L, int D, int dtype, const void* d_w_kv2, const float* d_b_kv2,
                              const float* d_g_k2, void* d_k2, void* d_v2, void* d_ws, size_t ws_bytes,
                              void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "context_kv: unknown dtype");
  if (L <= 0 || D <= 0 || D % 128) return set_error(HSA_EINVAL, "context_kv: need L > 0 and D % 128 == 0");
  if (!d_ctx || !d_w_kv2 || !d_g_k2 || !d_k2 || !d_v2 || !d_ws)
    return set_error(HSA_EINVAL, "context_kv: null pointer");
  if (ws_bytes < context_kv_scratch_bytes(L, D, dtype)) return set_error(HSA_EWORKSPACE, "context_kv: workspace");
  cudaStream_t st = as_stream(stream);
  HSA_TRY(linear(d_ctx, L, D, d_w_kv2, 2 * D, d_b_kv2, dtype, HSA_EPI_STORE, nullptr, d_ws, st));
  if (dtype == HSA_BF16) {
    auto* kv = static_cast<const __nv_bfloat16*>(d_ws);
    HSA_TRY(launch_rms(kv, 2 * D, L, D, d_g_k2, static_cast<__nv_bfloat16*>(d_k2), st));
    return launch_rms(kv + D, 2 * D, L, D, (const float*)nullptr, static_cast<__nv_bfloat16*>(d_v2), st);
  }
  auto* kv = static_cast<const float*>(d_ws);
  HSA_TRY(launch_rms(kv, 2 * D, L, D, d_g_k2, static_cast<float*>(d_k2), st));
  return launch_rms(kv + D, 2 * D, L, D, (const float*)nullptr, static_cast<float*>(d_v2), st);
}

// ------------------------------------------------------------------ §2.2 one block on the active rows
namespace {
struct StepWs {
  void *h, *qkv, *q, *att, *hid;
};
StepWs carve_step_ws(void* base, int M, int D, int F, int dtype) {
  const size_t e = esize(dtype);
  uint8_t* p = static_cast<uint8_t*>(base);
  StepWs w;
  w.h = p;   p += align256((size_t)M * D * e);
  w.qkv = p; p += align256((size_t)M * 3 * D * e);
  w.q = p;   p += align256((size_t)M * D * e);
  w.att = p; p += align256((size_t)M * D * e);
  w.hid = p;
  return w;
}
}  // namespace

extern "C" size_t hsa_layer_step_workspace_size(int M, int D, int F, int dtype) {
  if (M <= 0 || D <= 0 || F <= 0) return 0;
  const size_t e = esize(dtype);
  return align256((size_t)M * D * e) * 3 + align256((size_t)M * 3 * D * e) + align256((size_t)M * F * e);
}

extern "C" int hsa_layer_step(const hsa_layer_weights* w, void* d_kcache, void* d_vcache, int N, float* d_xA,
                              const float* d_x_src, const int32_t* d_idx, int M, const int32_t* d_pos,
                              const void* d_ctx_k, const void* d_ctx_v, int ctx_len, void* d_ws, size_t ws_bytes,
                              void* stream) {
  if (!w) return set_error(HSA_EINVAL, "layer_step: null weights");
  const int D = w->D, H = w->H, F = w->F, dt = w->dtype;
  if (dt != HSA_BF16 && dt != HSA_F32) return set_error(HSA_EINVAL, "layer_step: unknown dtype");
  if (H <= 0 || D != 128 * H) return set_error(HSA_EINVAL, "layer_step: need D = 128 H");
  if (F <= 0 || F % (dt == HSA_BF16 ? 64 : 4)) return set_error(HSA_EINVAL, "layer_step: FFN width not supported");
  if (N <= 0 || M < 1 || M > N) return set_error(HSA_EINVAL, "layer_step: need 1 <= M <= N");
  const void* mats[] = {w->w_qkv, w->w_o, w->w_1, w->w_2};
  const void* vecs[] = {w->b_qkv, w->g_q, w->g_k, w->b_o, w->b_1, w->b_2, w->mod};
  for (const void* p : mats)
    if (!p || !aligned16(p)) return set_error(HSA_EINVAL, "layer_step: null or misaligned weight matrix");
  for (const void* p : vecs)
    if (!p || !aligned16(p)) return set_error(HSA_EINVAL, "layer_step: null or misaligned weight vector");
  if (!d_kcache || !d_vcache || !d_xA || !d_idx || !d_pos || !d_ws || !aligned16(d_kcache) ||
      !aligned16(d_vcache) || !aligned16(d_xA) || (d_x_src && !aligned16(d_x_src)) || !aligned16(d_ws))
    return set_error(HSA_EINVAL, "layer_step: null or misaligned buffer");
  const bool cross = d_ctx_k != nullptr;
  if (cross) {
    if (!d_ctx_v || ctx_len <= 0 || !w->ln_c_g || !w->ln_c_b || !w->w_q2 || !w->b_q2 || !w->g_q2 || !w->w_o2 ||
        !w->b_o2)
      return set_error(HSA_EINVAL, "layer_step: incomplete cross-attention arguments");
  }
  if (ws_bytes < hsa_layer_step_workspace_size(M, D, F, dt))
    return set_error(HSA_EWORKSPACE, "layer_step: workspace smaller than hsa_layer_step_workspace_size");

  cudaStream_t st = as_stream(stream);
  StepWs ws = carve_step_ws(d_ws, M, D, F, dt);
  // the FFN hidden region and whatever the caller's workspace has beyond it are free until the
  // FFN: the attention calls may use them to split their tail over key ranges
  void* spare = ws.hid;
  const size_t spare_bytes = ws_bytes - (size_t)(static_cast<uint8_t*>(ws.hid) - static_cast<uint8_t*>(d_ws));
  const float* mod = w->mod;
  const bool bf = dt == HSA_BF16;
  using bf16 = __nv_bfloat16;

  // a1: gather + LN + (shift, scale) modulation
  if (bf) HSA_TRY(launch_ln(d_xA, d_x_src, d_idx, M, N, D, mod + D, mod, 1, static_cast<bf16*>(ws.h), st));
  else HSA_TRY(launch_ln(d_xA, d_x_src, d_idx, M, N, D, mod + D, mod, 1, static_cast<float*>(ws.h), st));
  // a2: QKV projection, q/k RMSNorm + RoPE, KV-cache scatter
  HSA_TRY(linear(ws.h, M, D, w->w_qkv, 3 * D, w->b_qkv, dt, HSA_EPI_STORE, nullptr, ws.qkv, st));
  if (bf)
    HSA_TRY(launch_qk_rope(static_cast<const bf16*>(ws.qkv), d_idx, d_pos, M, N, D, w->g_q, w->g_k,
                           static_cast<bf16*>(ws.q), static_cast<bf16*>(d_kcache), static_cast<bf16*>(d_vcache), st));
  else
    HSA_TRY(launch_qk_rope(static_cast<const float*>(ws.qkv), d_idx, d_pos, M, N, D, w->g_q, w->g_k,
                           static_cast<float*>(ws.q), static_cast<float*>(d_kcache), static_cast<float*>(d_vcache),
                           st));
  // a3: full-context attention over all N cache rows
  HSA_TRY(attention(ws.q, M, d_kcache, d_vcache, N, H, dt, ws.att, st, spare, spare_bytes));
  // a4: gated output projection into the residual stream
  HSA_TRY(linear(ws.att, M, D, w->w_o, D, w->b_o, dt, HSA_EPI_RESID, mod + 2 * D, d_xA, st));
  if (cross) {
    if (bf) HSA_TRY(launch_ln(d_xA, nullptr, d_idx, M, N, D, w->ln_c_g, w->ln_c_b, 0, static_cast<bf16*>(ws.h), st));
    else HSA_TRY(launch_ln(d_xA, nullptr, d_idx, M, N, D, w->ln_c_g, w->ln_c_b, 0, static_cast<float*>(ws.h), st));
    HSA_TRY(linear(ws.h, M, D, w->w_q2, D, w->b_q2, dt, HSA_EPI_STORE, nullptr, ws.qkv, st));
    if (bf) HSA_TRY(launch_rms(static_cast<const bf16*>(ws.qkv), D, M, D, w->g_q2, static_cast<bf16*>(ws.q), st));
    else HSA_TRY(launch_rms(static_cast<const float*>(ws.qkv), D, M, D, w->g_q2, static_cast<float*>(ws.q), st));
    HSA_TRY(attention(ws.q, M, d_ctx_k, d_ctx_v, ctx_len, H, dt, ws.att, st, spare, spare_bytes));
    HSA_TRY(linear(ws.att, M, D, w->w_o2, D, w->b_o2, dt, HSA_EPI_RESID, nullptr, d_xA, st));
  }
  // a4: gated GELU feed-forward
  if (bf) HSA_TRY(launch_ln(d_xA, nullptr, d_idx, M, N, D, mod + 4 * D, mod + 3 * D, 1, static_cast<bf16*>(ws.h), st));
  else HSA_TRY(launch_ln(d_xA, nullptr, d_idx, M, N, D, mod + 4 * D, mod + 3 * D, 1, static_cast<float*>(ws.h), st));
  HSA_TRY(linear(ws.h, M, D, w->w_1, F, w->b_1, dt, HSA_EPI_GELU, nullptr, ws.hid, st));
  return linear(ws.hid, M, F, w->w_2, D, w->b_2, dt, HSA_EPI_RESID, mod + 5 * D, d_xA, st);
}

// ------------------------------------------------------------------ patch model around the blocks
extern "C" size_t hsa_patch_workspace_size(int M, int D, int C, int dtype) {
  if (M <= 0 || D <= 0 || C <= 0) return 0;
  return align256((size_t)M * (C > D ? C : D) * esize(dtype));
}

extern "C" int hsa_patch_embed(const float* d_x, const int32_t* d_idx, int M, int N, int C, int D, int dtype,
                               const void* d_w_in, const float* d_b_in, float* d_X, void* d_ws, size_t ws_bytes,
                               void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "patch_embed: unknown dtype");
  if (M < 1 || M > N || C <= 0 || C % (dtype == HSA_BF16 ? 64 : 4) || D <= 0 || D % 64)
    return set_error(HSA_EINVAL, "patch_embed: unsupported sizes");
  if (!d_x || !d_idx || !d_w_in || !d_X || !d_ws || !aligned16(d_x) || !aligned16(d_ws))
    return set_error(HSA_EINVAL, "patch_embed: null or misaligned pointer");
  if (ws_bytes < hsa_patch_workspace_size(M, D, C, dtype)) return set_error(HSA_EWORKSPACE, "patch_embed: workspace");
  cudaStream_t st = as_stream(stream);
  ScopedTiming timing(HSA_KCLASS_OTHER, st);
  if (dtype == HSA_BF16)
    launch(k_gather_rows<__nv_bfloat16>, warp_blocks(M), 256, 0, st, d_x, d_idx, M, N, C,
           static_cast<__nv_bfloat16*>(d_ws));
  else
    launch(k_gather_rows<float>, warp_blocks(M), 256, 0, st, d_x, d_idx, M, N, C, static_cast<float*>(d_ws));
  count_launch(1);
  HSA_TRY(check_launch("gather launch"));
  return linear(d_ws, M, C, d_w_in, D, d_b_in, dtype, HSA_EPI_F32, nullptr, d_X, st);
}

extern "C" int hsa_velocity_head(const float* d_X, int M, int D, int C, int dtype, const float* d_head_mod,
                                 const void* d_w_out, const float* d_b_out, float* d_vA, void* d_ws, size_t ws_bytes,
                                 void* stream) {
  if (dtype != HSA_BF16 && dtype != HSA_F32) return set_error(HSA_EINVAL, "velocity_head: unknown dtype");
  if (M < 1 || D <= 0 || D % 128 || C <= 0 || C % (dtype == HSA_BF16 ? 64 : 4))
    return set_error(HSA_EINVAL, "velocity_head: unsupported sizes");
  if (!d_X || !d_head_mod || !d_w_out || !d_vA || !d_ws || !aligned16(d_X) || !aligned16(d_ws))
    return set_error(HSA_EINVAL, "velocity_head: null or misaligned pointer");
  if (ws_bytes < hsa_patch_workspace_size(M, D, C, dtype)) return set_error(HSA_EWORKSPACE, "velocity_head: workspace");
  cudaStream_t st = as_stream(stream);
  float* X = const_cast<float*>(d_X);  // read only: no gather source is given
  if (dtype == HSA_BF16)
    HSA_TRY(launch_ln(X, nullptr, nullptr, M, M, D, d_head_mod + D, d_head_mod, 1, static_cast<__nv_bfloat16*>(d_ws), st));
  else
    HSA_TRY(launch_ln(X, nullptr, nullptr, M, M, D, d_head_mod + D, d_head_mod, 1, static_cast<float*>(d_ws), st));
  return linear(d_ws, M, D, d_w_out, C, d_b_out, dtype, HSA_EPI_F32, nullptr, d_vA, st);
}

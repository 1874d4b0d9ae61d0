// host_io.cu -- one HSA iteration with the latent in host memory (hsa_iteration_host, include/hsa.h):
// the upload of x, the iteration's device work (HSA summary §2.2 layer step on A_i, §2.3 cached
// Euler update, §2.1 regrouping after a full step) and the download of x, each on its own stream
// and ordered by the caller's events, so that a caller alternating two slots overlaps the copies
// of neighbouring iterations with compute.
#include "common.cuh"

namespace hsa {
namespace {

int cuda_ok(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return HSA_OK;
  (void)cudaGetLastError();
  return set_error(HSA_ECUDA, std::string("iteration_host: ") + what + ": " + cudaGetErrorString(e));
}

// Every condition the iteration's calls check, tested before anything is enqueued.
int check_iteration(const hsa_iteration_args* a, const float* h_x_in, float* h_x_out, const hsa_host_slot* s) {
  if (!a || !a->w || !s || !h_x_in || !h_x_out) return set_error(HSA_EINVAL, "iteration_host: null argument");
  if (!s->d_x || !aligned16(s->d_x) || !s->ev_in || !s->ev_done || !s->ev_free)
    return set_error(HSA_EINVAL, "iteration_host: the slot needs an aligned d_x and its three events");
  const hsa_layer_weights* w = a->w;
  const int D = w->D, H = w->H, F = w->F, dt = w->dtype;
  if (dt != HSA_BF16 && dt != HSA_F32) return set_error(HSA_EINVAL, "iteration_host: unknown dtype");
  if (H <= 0 || D != 128 * H) return set_error(HSA_EINVAL, "iteration_host: need D = 128 H");
  if (F <= 0 || F % (dt == HSA_BF16 ? 64 : 4)) return set_error(HSA_EINVAL, "iteration_host: FFN width not supported");
  if (a->N <= 0 || a->M < 1 || a->M > a->N) return set_error(HSA_EINVAL, "iteration_host: need 1 <= M <= N");
  const void* need[] = {w->w_qkv, w->w_o, w->w_1, w->w_2, w->b_qkv, w->g_q, w->g_k, w->b_o, w->b_1, w->b_2, w->mod,
                        a->d_kcache, a->d_vcache, a->d_idx, a->d_pos, a->d_xA, a->d_vhat, a->d_ws};
  for (const void* p : need)
    if (!p || !aligned16(p)) return set_error(HSA_EINVAL, "iteration_host: null or misaligned device buffer");
  if (a->d_ctx_k && (!a->d_ctx_v || a->ctx_len <= 0 || !w->ln_c_g || !w->ln_c_b || !w->w_q2 || !w->b_q2 ||
                     !w->g_q2 || !w->w_o2 || !w->b_o2))
    return set_error(HSA_EINVAL, "iteration_host: incomplete cross-attention arguments");
  if (a->ws_bytes < hsa_layer_step_workspace_size(a->M, D, F, dt))
    return set_error(HSA_EWORKSPACE, "iteration_host: workspace smaller than hsa_layer_step_workspace_size");
  if (a->M == a->N && a->d_group) {
    if (!a->d_score || !a->d_order || !a->h_group_sizes || a->K < 1 || a->K > kMaxGroups)
      return set_error(HSA_EINVAL, "iteration_host: regrouping needs d_score, d_order and 1 <= K group sizes");
    long long sum = 0;
    for (int k = 0; k < a->K; ++k) {
      if (a->h_group_sizes[k] < 0) return set_error(HSA_EINVAL, "iteration_host: negative group size");
      sum += a->h_group_sizes[k];
    }
    if (sum != a->N) return set_error(HSA_EINVAL, "iteration_host: group sizes must sum to N");
    const size_t sel = hsa_select_tokens_workspace_size(a->N, a->K);
    if (sel > 0 && (!a->d_sel_ws || a->sel_ws_bytes < sel))
      return set_error(HSA_EWORKSPACE, "iteration_host: selection workspace smaller than its size");
  }
  return HSA_OK;
}

}  // namespace
}  // namespace hsa

extern "C" int hsa_iteration_host(const hsa_iteration_args* a, const float* h_x_in, float* h_x_out,
                                  const hsa_host_slot* slot, void* stream, void* stream_h2d, void* stream_d2h) {
  using namespace hsa;
  HSA_TRY(check_iteration(a, h_x_in, h_x_out, slot));
  cudaStream_t st = as_stream(stream), up = as_stream(stream_h2d), down = as_stream(stream_d2h);
  cudaEvent_t ev_in = static_cast<cudaEvent_t>(slot->ev_in), ev_done = static_cast<cudaEvent_t>(slot->ev_done),
              ev_free = static_cast<cudaEvent_t>(slot->ev_free);
  const int N = a->N, M = a->M, D = a->w->D;
  const size_t bytes = (size_t)N * D * sizeof(float);
  // 1. upload, once the slot's previous download has read d_x
  HSA_TRY(cuda_ok(cudaStreamWaitEvent(up, ev_free, 0), "wait for the slot"));
  HSA_TRY(cuda_ok(cudaMemcpyAsync(slot->d_x, h_x_in, bytes, cudaMemcpyHostToDevice, up), "upload"));
  HSA_TRY(cuda_ok(cudaEventRecord(ev_in, up), "record the upload"));
  // 2. the iteration on the compute stream
  HSA_TRY(cuda_ok(cudaStreamWaitEvent(st, ev_in, 0), "wait for the upload"));
  HSA_TRY(hsa_layer_step(a->w, a->d_kcache, a->d_vcache, N, a->d_xA, slot->d_x, a->d_idx, M, a->d_pos, a->d_ctx_k,
                         a->d_ctx_v, a->ctx_len, a->d_ws, a->ws_bytes, stream));
  const bool full = M == N;
  HSA_TRY(hsa_euler_update(slot->d_x, a->d_vhat, a->d_xA, a->d_idx, M, N, D, a->dsigma, full ? a->d_score : nullptr,
                           stream));
  if (full && a->d_group)
    HSA_TRY(hsa_select_tokens(a->d_score, N, a->K, a->h_group_sizes, a->d_group, a->d_order, a->d_sel_ws,
                              a->sel_ws_bytes, stream));
  HSA_TRY(cuda_ok(cudaEventRecord(ev_done, st), "record the iteration"));
  // 3. download
  HSA_TRY(cuda_ok(cudaStreamWaitEvent(down, ev_done, 0), "wait for the iteration"));
  HSA_TRY(cuda_ok(cudaMemcpyAsync(h_x_out, slot->d_x, bytes, cudaMemcpyDeviceToHost, down), "download"));
  return cuda_ok(cudaEventRecord(ev_free, down), "record the download");
}

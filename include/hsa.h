/*
 * hsa.h -- C ABI of libhsa: the hot path of Heterogeneous Step Allocation (HSA)
 * on one B200 (sm_100a).
 *
 * Source of the method: "Not All Tokens Need 40 Steps: Heterogeneous Step
 * Allocation in Diffusion Transformers for Efficient Video Generation"
 * (Chu & Patel, arXiv 2605.06892), as summarised on the gist.science pages
 * (section numbers below are those of the summary):
 *   §2.1 token partitioning and scheduling, dynamic token selection;
 *   §2.2 KV-cache synchronisation;
 *   §2.3 cached Euler update;
 *   §2.4 phase-aware caching window.
 *
 * Conventions shared by every entry point
 *   - Notation: N tokens, K groups G_1..G_K with step budgets s_k (s_k | T,
 *     s_1 = T), T iterations, m full steps at each end, sigma_0..sigma_T the
 *     noise schedule, A_i the active token list of iteration i (M = |A_i|),
 *     D hidden width, H heads of 128 channels (D = 128 H), F FFN width, C
 *     latent channels per token.
 *   - Ownership: the caller allocates and owns every buffer.  The library
 *     keeps no pointer after a call returns and allocates no device memory;
 *     scratch comes from the caller's workspace (`d_ws`, `ws_bytes`), sized
 *     by the matching *_workspace_size function.  Pointers prefixed d_ are
 *     device pointers, h_ host pointers; every device buffer must be 16-byte
 *     aligned and densely packed row-major with the stated shape.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *     default stream).  Device work is enqueued asynchronously on it.
 *   - Errors: every call returns an int status.  Argument errors are found on
 *     the host before anything is enqueued.  Faults found by a kernel (a token
 *     index outside [0, N), a bounded wait that ran out) never trap: the
 *     kernel skips the access, records the fault in a device status word and
 *     finishes; hsa_device_status() reports it after the stream drains.
 *     A wait that ran out also raises a per-device abort flag so that no other
 *     kernel can hang: until hsa_device_status() has been called (which reads
 *     and clears both), every later pipelined kernel on that device (attention,
 *     GEMM) returns early and leaves its outputs incomplete.  A caller that can
 *     meet a stall should therefore read the status after every step, not only
 *     at the end of a run, to know which step first went wrong.
 *   - Matrices in [out][in] layout (row o holds the weights of output o),
 *     dtype HSA_BF16 (tensor-core path) or HSA_F32 (CUDA-core path).  Biases,
 *     norm gains, modulation vectors, latents and velocities are float32.
 */
#ifndef HSA_H_
#define HSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
enum {
  HSA_OK = 0,
  HSA_EINVAL = 1,        /* an argument breaks a stated constraint                 */
  HSA_EINDEX = 2,        /* a kernel met a token index outside [0, N)              */
  HSA_ECUDA = 3,         /* a CUDA launch or API call failed                       */
  HSA_ETIMEOUT = 4,      /* a kernel's bounded wait ran out (pipeline stall)       */
  HSA_EWORKSPACE = 5     /* the workspace is smaller than *_workspace_size asks    */
};

enum { HSA_F32 = 0, HSA_BF16 = 1 };

/* Text of the last host-side error of this thread (never NULL). */
const char* hsa_last_error_string(void);

/* Waits for `stream`, then returns and clears the device status word of the
 * current device: HSA_OK, HSA_EINDEX or HSA_ETIMEOUT (the first fault seen). */
int hsa_device_status(void* stream);

/* Diagnostic, not part of the method: launches one warp that waits on an mbarrier no thread
 * ever completes.  The library's bounded wait gives up after its limit (1 s), records
 * HSA_ETIMEOUT in the device status word and raises the abort flag that makes every pending
 * wait of the library return at once; hsa_device_status() then returns HSA_ETIMEOUT and clears
 * both, after which the library runs normally.  Lets a test exercise the failure path of the
 * pipelined kernels without faulting or hanging the GPU.  Returns the launch status. */
int hsa_selftest_wait_timeout(void* stream);

/* Number of kernel launches the library has enqueued in this process. */
uint64_t hsa_launch_count(void);

/* Per-kernel timing (measurement support; off by default).  While enabled, every
 * launch libhsa makes is bracketed by two CUDA events recorded on its stream,
 * filed under a kernel class.  hsa_timing_read waits for the recorded events
 * and returns the summed device time (ms) and the launch count of one class;
 * hsa_timing_reset forgets every record.  Host state of this process. */
enum { HSA_KCLASS_ATTENTION = 0, HSA_KCLASS_GEMM = 1, HSA_KCLASS_OTHER = 2, HSA_KCLASS_COUNT = 3 };
int hsa_timing_enable(int on);
int hsa_timing_read(int kclass, double* total_ms, int* launches);
int hsa_timing_reset(void);

/* ------------------------------------------------------------------ §2.1 + §2.4 plan (host only)
 * Validates (T, K, s_k, n_k, N, m) and writes the schedule of the whole run.
 *   h_budgets[K]      s_k; s_1 = T, every s_k divides T, non-increasing.
 *   h_group_sizes[K]  n_k >= 0 with sum n_k = N.
 *   m                 full steps at each end, 0 <= 2m <= T.
 *   sigma_kind        0: sigma_i = 1 - i/T; 1: the shifted form
 *                     shift*sigma/(1 + (shift-1)*sigma) of that base.
 * Outputs (host buffers, may be NULL when not wanted):
 *   h_sigmas[T+1]        float32 schedule, computed in double then rounded.
 *   h_active_tab[T*K]    1 when group k runs at iteration i (0-based):
 *                        i < m, or i >= T-m, or i mod (T/s_k) == 0.
 *   h_n_active[T]        |A_i| = sum of n_k over the groups running at i.
 * Returns HSA_EINVAL when a constraint fails.  No device work. */
int hsa_plan_groups(int T, int K, const int* h_budgets, const int* h_group_sizes, int N, int m,
                    int sigma_kind, float shift, float* h_sigmas, uint8_t* h_active_tab,
                    int* h_n_active);

/* ------------------------------------------------------------------ §2.1 dynamic selection
 * Per-token L1 relative change of the velocity prediction:
 *   d_score[n] = sum_c |d_v_new[n,c] - d_v_prev[n,c]| / (sum_c |d_v_prev[n,c]| + 1e-8)
 * d_v_new, d_v_prev: N x C float32; d_score: N float32.  C % 4 == 0. */
int hsa_l1_score(const float* d_v_new, const float* d_v_prev, int N, int C, float* d_score,
                 void* stream);

/* Partition of the N tokens into K groups of the fixed sizes h_group_sizes[K]
 * by score: tokens ranked by (d_score descending, token index ascending) --
 * scores compared as float32, NaN ranking as +inf, values <= 0 as 0 -- fill
 * G_1 (the first n_1), then G_2, ... so the slowest-changing tokens get the
 * fewest steps (§2.1).  Outputs: d_group[N] (0-based group of each token) and
 * d_order[N] (the groups' token lists concatenated in group order, each
 * ascending by index; with nested budgets every A_i is a prefix of it).
 * Bit-exact: the result is unique under this total order.
 * Workspace: hsa_select_tokens_workspace_size(N, K) bytes.  1 <= K <= 16. */
size_t hsa_select_tokens_workspace_size(int N, int K);
int hsa_select_tokens(const float* d_score, int N, int K, const int* h_group_sizes,
                      int8_t* d_group, int32_t* d_order, void* d_ws, size_t ws_bytes,
                      void* stream);

/* The same partition with a set of pinned tokens (image-to-video, HSA summary §4: the
 * conditioning image must stay intact, read here as its latent frame's tokens keeping the
 * full step budget).  d_pinned[N] (uint8, device, may be NULL = none pinned): a token with
 * d_pinned[n] != 0 ranks ahead of every unpinned token whatever its score, NaN included;
 * pinned tokens rank among themselves by index.  So with at most n_1 pinned tokens all of
 * them land in G_1; more than n_1 continue into G_2, ... in index order (not an error).
 * Same outputs, workspace and errors as hsa_select_tokens, which equals this call with
 * d_pinned = NULL.  The pages give no mechanism for I2V; this is a reading. */
int hsa_select_tokens_pinned(const float* d_score, const uint8_t* d_pinned, int N, int K,
                             const int* h_group_sizes, int8_t* d_group, int32_t* d_order,
                             void* d_ws, size_t ws_bytes, void* stream);

/* A_i for iteration i (§2.1): the lists of the groups active at i, taken from d_order (the
 * groups' lists concatenated in group order, as hsa_select_tokens writes it), concatenated in
 * group order into d_idx[M], M = sum of the active groups' sizes (written to *h_M when h_M is
 * not NULL).  h_active[K]: 1 for a group running at i (a row of hsa_plan_groups' table).  With
 * nested budgets A_i is a prefix of d_order and needs no copy; this call covers every other
 * pattern with one launch.  HSA_EINVAL when the sizes do not sum to N or K is out of range. */
int hsa_active_rows(const int32_t* d_order, int N, int K, const int* h_group_sizes,
                    const uint8_t* h_active, int32_t* d_idx, int* h_M, void* stream);

/* ------------------------------------------------------------------ §2.3 cached Euler update
 * One iteration's solver update over all N tokens:
 *   1. v_hat[idx[r]] = v_A[r] for r < M (fresh velocities of A_i);
 *   2. x[n] += dsigma * v_hat[n] for every n (dsigma = sigma_{i+1} - sigma_i),
 *      one branch-free pass over N x C.
 * When d_score is not NULL (a step where every token is active, M == N), the
 * L1 relative change of v_A against the old v_hat is written to d_score[idx[r]]
 * before v_hat is overwritten, fused into the same pass.
 *   d_x, d_vhat: N x C float32 (updated in place); d_vA: M x C float32;
 *   d_idx: M token indices (distinct, in [0, N)).  C % 4 == 0. */
int hsa_euler_update(float* d_x, float* d_vhat, const float* d_vA, const int32_t* d_idx, int M,
                     int N, int C, float dsigma, float* d_score, void* stream);

/* ------------------------------------------------------------------ §2.2 one DiT block on A_i
 * Weights of one block (all device pointers).  Matrices [out][in] of dtype. */
typedef struct hsa_layer_weights {
  int D, H, F;          /* D = 128 H; D % 64 == 0; F % 64 == 0                      */
  int dtype;            /* HSA_BF16 or HSA_F32: matrices, KV cache, context K/V     */
  const void* w_qkv;    /* [3D][D]: rows [0,D) q, [D,2D) k, [2D,3D) v               */
  const float* b_qkv;   /* [3D]                                                     */
  const float* g_q;     /* [D] RMSNorm gain of q (RMS over all D channels)          */
  const float* g_k;     /* [D] RMSNorm gain of k                                    */
  const void* w_o;      /* [D][D]  */ const float* b_o;   /* [D] */
  const void* w_1;      /* [F][D]  */ const float* b_1;   /* [F] */
  const void* w_2;      /* [D][F]  */ const float* b_2;   /* [D] */
  const float* mod;     /* [6][D]: shift, scale, gate of attention; shift, scale, gate of FFN */
  /* cross-attention against a context; all NULL when the block has none */
  const float* ln_c_g;  /* [D] affine LayerNorm before the cross-attention          */
  const float* ln_c_b;  /* [D] */
  const void* w_q2;     /* [D][D]  */ const float* b_q2;  /* [D] */
  const float* g_q2;    /* [D] RMSNorm gain of the cross-attention query            */
  const void* w_o2;     /* [D][D]  */ const float* b_o2;  /* [D] */
} hsa_layer_weights;

/* Context keys/values of the cross-attention, once per run:
 *   K2 = RMSNorm(ctx W_k2^T + b_k2) * g_k2,  V2 = ctx W_v2^T + b_v2
 *   d_ctx: L x D in dtype; d_w_kv2: [2D][D] (k rows then v rows); d_b_kv2 [2D]; d_g_k2 [D];
 *   outputs d_k2, d_v2: L x D in dtype.  Workspace: hsa_context_kv_workspace_size(L, D) bytes,
 *   the fp32 size (L x 2D x 4), which covers both dtypes; the bf16 path needs only half of it. */
size_t hsa_context_kv_workspace_size(int L, int D);
int hsa_context_kv(const void* d_ctx, int L, int D, int dtype, const void* d_w_kv2,
                   const float* d_b_kv2, const float* d_g_k2, void* d_k2, void* d_v2, void* d_ws,
                   size_t ws_bytes, void* stream);

/* The same projection for callers that cannot allocate device memory.  The paper
 * has no counterpart: this entry exists for embedders that may not call cudaMalloc
 * (or any allocating library routine) where they need the context keys/values, for
 * instance a runtime whose device memory budget is fixed at start-up, or code on a
 * path where an allocation would synchronise the device.  Instead of a caller
 * workspace it uses a scratch array built into the library: 8 MiB
 * (hsa_context_kv_noalloc_max_bytes()), held by every GPU that loads libhsa until
 * the process exits.  It allocates nothing.
 *   - Arguments as hsa_context_kv, without the workspace.  The L x 2D projection in
 *     the call's dtype (4 bytes an element for HSA_F32, 2 for HSA_BF16) must fit the
 *     scratch, else HSA_EINVAL: L = 512 fits up to D = 2048 in fp32, D = 4096 in bf16.
 *   - The first call on a device looks up the scratch's device address (once per
 *     device, with that device current, and again after the device's context has been
 *     replaced, e.g. by cudaDeviceReset); make that first call before any stream
 *     capture.
 *   - Every call shares the one scratch array and leaves its contents behind; the
 *     projection writes each scratch element before reading it, so no clearing is
 *     needed.  Calls whose GPU work overlaps (other streams, other host threads on
 *     the same device) race on the scratch: order them on one stream. */
size_t hsa_context_kv_noalloc_max_bytes(void);
int hsa_context_kv_noalloc(const void* d_ctx, int L, int D, int dtype, const void* d_w_kv2,
                           const float* d_b_kv2, const float* d_g_k2, void* d_k2, void* d_v2,
                           void* stream);

/* One block on the active rows of iteration i (§2.2):
 *   X = x_A (M x D float32, the residual stream of the active tokens, in/out);
 *   h = LN(X)(1 + mod1) + mod0;  [q k v] = h W_qkv^T + b_qkv;
 *   q, k <- RMSNorm over D times g_q, g_k;  3D RoPE of each head at d_pos[idx[r]]
 *     (channels [0,44) frame, [44,86) row, [86,128) column; pair j of a segment of
 *     width w turns by pos * 10000^(-2j/w));
 *   Kc[idx[r]] = k, Vc[idx[r]] = v  (rows of skipped tokens are not touched);
 *   o = softmax(q Kc^T / sqrt(128)) Vc per head, over all N cache rows;
 *   X += mod2 * (o W_o^T + b_o);
 *   if d_ctx_k: X += CrossAttn(LN_affine(X)) against the L_ctx context rows;
 *   X += mod5 * (GELU_tanh((LN(X)(1 + mod4) + mod3) W_1^T + b_1) W_2^T + b_2).
 * d_kcache, d_vcache: N x D in dtype (the layer's cache, updated in place).
 * d_x_src: when not NULL, X is first gathered as d_x_src[idx[r]] (N x D float32)
 *   and written to d_xA; when NULL, d_xA already holds X.
 * d_idx: M distinct token indices in [0, N); d_pos: N x 3 int32 (frame, row, column).
 * 1 <= M <= N.  Workspace: hsa_layer_step_workspace_size(M, D, F, dtype).  A workspace sized
 * for a larger M (say N, reused for every step) leaves room the attention uses to split the
 * key range of its last, incomplete wave of work units (see hsa_attention_ws); results agree
 * with the unsplit path to rounding. */
size_t hsa_layer_step_workspace_size(int M, int D, int F, int dtype);
int hsa_layer_step(const hsa_layer_weights* w, void* d_kcache, void* d_vcache, int N, float* d_xA,
                   const float* d_x_src, const int32_t* d_idx, int M, const int32_t* d_pos,
                   const void* d_ctx_k, const void* d_ctx_v, int ctx_len, void* d_ws,
                   size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ one iteration, latent in host memory
 * One HSA iteration (§2.1-§2.3) of a model made of one block, whose output rows are the velocity
 * (C = D), for a caller that keeps the latent x in host memory between iterations.  The library
 * moves it:
 *   1. on stream_h2d: wait for slot->ev_free, copy h_x_in -> slot->d_x, record slot->ev_in;
 *   2. on stream: wait for slot->ev_in; v_A = hsa_layer_step of the M active rows d_idx,
 *      gathered from slot->d_x; hsa_euler_update (v_hat[A] = v_A, x += dsigma v_hat, and the L1
 *      relative-change score into d_score when M == N and d_score is not NULL); when M == N and
 *      d_group is not NULL, hsa_select_tokens regroups the tokens from that score into d_group
 *      and d_order; record slot->ev_done;
 *   3. on stream_d2h: wait for slot->ev_done, copy slot->d_x -> h_x_out, record slot->ev_free.
 * h_x_in, h_x_out: host buffers of N x D float32 (page-locked, or the copies do not overlap
 * compute); they may be the same buffer.  The device-side state (weights, caches, v_hat, the
 * velocity rows d_xA, M x D, the scores and groups, the workspaces) is the caller's, as in
 * hsa_layer_step, hsa_euler_update and hsa_select_tokens; d_order may be d_idx (a full step
 * reads A_i before it regroups).  The events are cudaEvent_t handles (passed as void*) created by
 * the caller, timing may be disabled; an event never recorded counts as complete.  A caller that
 * alternates two slots overlaps the upload of iteration k + 1 and the download of iteration k
 * with compute.  The three streams may be one stream (no overlap).  Copies are cudaMemcpyAsync,
 * and the call does not wait on the host: a caller that passes one call's h_x_out as a later
 * call's h_x_in waits for the first call's ev_free first (cudaEventSynchronize).  Every argument
 * is checked before anything is enqueued; a CUDA error after that returns HSA_ECUDA with the steps
 * before it enqueued. */
typedef struct hsa_iteration_args {
  const hsa_layer_weights* w;
  void* d_kcache;               /* N x D, dtype of w                                         */
  void* d_vcache;               /* N x D                                                     */
  int N;
  const int32_t* d_idx;         /* M active token indices (A_i)                              */
  int M;
  const int32_t* d_pos;         /* N x 3 (frame, row, column)                                */
  const void* d_ctx_k;          /* ctx_len x D or NULL (no cross-attention)                   */
  const void* d_ctx_v;
  int ctx_len;
  float* d_xA;                  /* M x D float32: the block's rows, v_A                      */
  float* d_vhat;                /* N x D float32, updated                                    */
  float dsigma;                 /* sigma_{i+1} - sigma_i                                     */
  float* d_score;               /* N float32 or NULL                                         */
  int K;                        /* groups of the regrouping                                  */
  const int* h_group_sizes;     /* K sizes (host), sum N                                     */
  int8_t* d_group;              /* N, or NULL: no regrouping                                 */
  int32_t* d_order;             /* N                                                         */
  void* d_ws;                   /* hsa_layer_step_workspace_size(M, D, F, dtype) bytes       */
  size_t ws_bytes;
  void* d_sel_ws;               /* hsa_select_tokens_workspace_size(N, K) bytes              */
  size_t sel_ws_bytes;
} hsa_iteration_args;

typedef struct hsa_host_slot {
  float* d_x;                   /* N x D float32 device copy of the latent                   */
  void* ev_in;                  /* cudaEvent_t: upload done                                  */
  void* ev_done;                /* cudaEvent_t: iteration done                               */
  void* ev_free;                /* cudaEvent_t: download done, the slot may be refilled      */
} hsa_host_slot;

int hsa_iteration_host(const hsa_iteration_args* a, const float* h_x_in, float* h_x_out,
                       const hsa_host_slot* slot, void* stream, void* stream_h2d, void* stream_d2h);

/* ------------------------------------------------------------------ building blocks of the step
 * Full-context attention of §2.2 on its own: M compacted queries against L
 * cached keys/values, H heads of 128: o = softmax(q K^T / sqrt(128)) V.
 *   d_q: M x 128H, d_k, d_v: L x 128H, d_o: M x 128H, all in dtype. */
int hsa_attention(const void* d_q, int M, const void* d_k, const void* d_v, int L, int H, int dtype,
                  void* d_o, void* stream);

/* The same attention with a workspace.  The work units are (128-query tile, head) pairs, one
 * per SM at a time.  The units that fill complete waves of the GPU's SMs run whole.  With
 * ws_bytes >= hsa_attention_workspace_size(M, L, H, dtype), each unit of the last, incomplete
 * wave is split over S ranges of key tiles, so the split CTAs fill that wave.  Each split
 * writes an unnormalised fp32 output and its row max and sum to d_ws, and a second kernel
 * merges them:
 *   o = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s,  m = max_s m_s.
 * A smaller or NULL workspace runs every unit whole, like hsa_attention.  Only the bf16 path
 * splits; the size is 0 when no split pays off (every wave complete, or fewer than 4 key tiles).
 * d_ws must be 16-byte aligned.  Not in the pages: a scheduling choice of this implementation. */
size_t hsa_attention_workspace_size(int M, int L, int H, int dtype);
int hsa_attention_ws(const void* d_q, int M, const void* d_k, const void* d_v, int L, int H, int dtype,
                     void* d_o, void* d_ws, size_t ws_bytes, void* stream);

/* Linear layer on compacted rows: y = epilogue(x W^T + b) for x: M x Kin (dtype),
 * W: [Nout][Kin] (dtype), b: [Nout] float32 (NULL = 0).
 *   epilogue HSA_EPI_STORE:  d_y (M x Nout, dtype) = acc + b
 *   epilogue HSA_EPI_GELU:   d_y (M x Nout, dtype) = GELU_tanh(acc + b)
 *   epilogue HSA_EPI_RESID:  d_y (M x Nout, float32) += gate * (acc + b), gate [Nout] float32
 *                            (NULL = 1)
 *   epilogue HSA_EPI_F32:    d_y (M x Nout, float32) = acc + b
 * Kin % 64 == 0 and Nout % 64 == 0 (bf16); Kin % 4 == 0, Nout % 4 == 0 (f32). */
enum { HSA_EPI_STORE = 0, HSA_EPI_GELU = 1, HSA_EPI_RESID = 2, HSA_EPI_F32 = 3 };
int hsa_linear(const void* d_x, int M, int Kin, const void* d_w, int Nout, const float* d_b,
               int dtype, int epilogue, const float* d_gate, void* d_y, void* stream);

/* Patch model around the blocks (latents with C channels per token):
 * hsa_patch_embed:  X (M x D float32) = x[idx[r]] W_in^T + b_in, W_in [D][C] dtype,
 *                   d_x: N x C float32.
 * hsa_velocity_head: v_A (M x C float32) = (LN(X)(1 + head_mod1) + head_mod0) W_out^T + b_out,
 *                   W_out [C][D] dtype, head_mod [2][D] float32.
 * Workspace: hsa_patch_workspace_size(M, D, C, dtype) bytes, shared by both. */
size_t hsa_patch_workspace_size(int M, int D, int C, int dtype);
int hsa_patch_embed(const float* d_x, const int32_t* d_idx, int M, int N, int C, int D, int dtype,
                    const void* d_w_in, const float* d_b_in, float* d_X, void* d_ws, size_t ws_bytes,
                    void* stream);
int hsa_velocity_head(const float* d_X, int M, int D, int C, int dtype, const float* d_head_mod,
                      const void* d_w_out, const float* d_b_out, float* d_vA, void* d_ws,
                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ head parallelism (one block over G GPUs)
 * The pages run each denoising model on one device; these calls let one block's heads be split
 * over G GPUs (each rank holding H/G heads of W_q, W_k, W_v, the KV cache of those heads for all
 * N tokens, the matching columns of W_o and 1/G of the FFN) with the collectives between them
 * issued by the caller (all-gather of the LayerNorm output, reduce of the partial projections,
 * sum of the q/k squares).  Not in the pages: a way to run the §2.2 step when one block does not
 * fit a GPU's time budget.  Every call is a plain kernel on local memory.
 *
 * LayerNorm rows: d_out[r] = LN(X[r]) * (1 + d_mul) + d_add (modulate != 0) or
 * LN(X[r]) * d_mul + d_add (affine), eps 1e-6, over D channels (D % 128 == 0), output in dtype.
 * With d_x_src (N x D float32) the rows are first gathered, X[r] = d_x_src[d_idx[r]], and
 * written to d_X (M x D float32). */
int hsa_layernorm_rows(float* d_X, const float* d_x_src, const int32_t* d_idx, int M, int N, int D,
                       const float* d_mul, const float* d_add, int modulate, int dtype, void* d_out,
                       void* stream);

/* Partial RMS statistics: d_ss[r * ss_stride] = sum_c d_in[r * in_stride + c]^2 for c < D
 * (float32 sums of dtype inputs; D % 4 == 0, in_stride % 4 == 0). */
int hsa_row_sumsq(const void* d_in, int in_stride, int M, int D, int dtype, float* d_ss, int ss_stride,
                  void* stream);

/* q/k RMSNorm with sums of squares taken over all D_total channels of the row (d_ss[2r] for q,
 * d_ss[2r+1] for k: the ranks' partial sums added), times the local gains d_g_q, d_g_k [Dl];
 * then 3D RoPE of each local 128-channel head at d_pos[d_idx[r]]; d_Q[r] = q (M x Dl),
 * d_kcache[d_idx[r]] = k, d_vcache[d_idx[r]] = v (N x Dl).  d_qkv rows are [q | k | v], Dl each
 * (Dl % 128 == 0).  Rows of skipped tokens are not touched; indices outside [0, N) are flagged
 * (HSA_EINDEX) and skipped. */
int hsa_qk_norm_rope_ext(const void* d_qkv, int M, int N, int Dl, int D_total, const float* d_ss,
                         const float* d_g_q, const float* d_g_k, const int32_t* d_idx,
                         const int32_t* d_pos, int dtype, void* d_Q, void* d_kcache, void* d_vcache,
                         void* stream);

/* d_out[r] (M x D, dense) = d_in[r] * rsqrt(d_ss[r * ss_stride] / D_total + 1e-6) * d_g
 * (d_g NULL = 1); with d_ss NULL a plain copy of the D first elements of each input row. */
int hsa_rms_rows_ext(const void* d_in, int in_stride, int M, int D, int D_total, const float* d_ss,
                     int ss_stride, const float* d_g, int dtype, void* d_out, void* stream);

/* Residual update of reduced partial projections: d_X[r] += d_gate * (d_y[r] + d_b) over D
 * channels (M x D float32 both; d_b, d_gate NULL = 0, 1). */
int hsa_gated_residual(float* d_X, const float* d_y, int M, int D, const float* d_b,
                       const float* d_gate, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* HSA_H_ */

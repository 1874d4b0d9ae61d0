"""Plain fp64 CPU oracle of one Heterogeneous Step Allocation (HSA) denoising iteration.

TEST INFRASTRUCTURE.  This package is the checker, not the product: only the
test-suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import it.  The CUDA library never calls it and shares no
code with it; both consume the same seeded arrays from
``token_sparse_denoising_b200.synthetic``.

Source: "Not All Tokens Need 40 Steps: Heterogeneous Step Allocation in
Diffusion Transformers for Efficient Video Generation" (Chu & Patel, arXiv
2605.06892), as summarised on the gist.science pages ("Technische
Samenvatting: Heterogene Staptoewijzing (HSA) ..." and its French, German and
Japanese translations).  Section numbers below are those of that summary:
  §2.1  token partitioning and scheduling (K groups, budgets s_k | T,
        s_1 = T, group k active iff i mod (T/s_k) = 0, dynamic selection by
        the per-token L1 relative change of velocity predictions);
  §2.2  KV-cache synchronisation (only A_i runs the QKV projections, their
        fresh K/V overwrite the per-layer cache, active queries attend to all
        N cached rows at O(|A_i| N) cost, skipped tokens do no query,
        cross-attention or feed-forward work);
  §2.3  cached Euler update (every token advances by (sigma_{i+1} - sigma_i)
        with its fresh or cached velocity v_hat_n, one branch-free op over N);
  §2.4  phase-aware caching window (the first and last m steps are full).

The pages name no network architecture.  The block is the Wan-style DiT block
of the Wan-1.3B / Wan-14B shapes this library targets: LayerNorm + modulation,
QKV with RMSNorm on q/k, 3D RoPE (44/42/42 channel split per 128-wide head),
softmax attention, gated output projection, optional cross-attention against
a text context, gated GELU(tanh) feed-forward.

Readings of what the pages leave open:
  * iteration index i is 0-based, i in [0, T); step i moves sigma_i -> sigma_{i+1};
  * groups are ranked by (score descending, token index ascending); group 1
    takes the highest scores; scores are compared as float32, NaN as +inf;
  * L1 relative change = sum_c |v_new - v_prev| / (sum_c |v_prev| + 1e-8);
  * selection re-runs after every step in which all N tokens were active;
  * the cache holds post-RMSNorm, post-RoPE K, and V;
  * compacted active rows are the groups' ascending index lists in group order;
  * image-to-video (§4 reports only the outcome): the conditioning frame's
    tokens are pinned ahead of every score, so they keep the full budget;
  * a static grouping (a fixed partition, never regrouped) is the plainest
    alternative to the dynamic selection.

Parity status: every function here is pinned by tests/test_oracle_pins.py
except the model-level quality of HSA itself (parity unpinned: the pages give
no worked numbers for it; their VBench scores need trained weights).
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
LN_EPS = 1e-6
RMS_EPS = 1e-6
SCORE_EPS = 1e-8
ROPE_THETA = 10000.0
HEAD_DIM = 128
ROPE_SPLIT = (44, 42, 42)          # temporal, height, width channels of each head


# ====================================================================== §2.1 scheduling

def validate_plan(T: int, budgets, sizes, N: int, m: int) -> None:
    """Constraints of §2.1 and §2.4: s_k divides T, s_1 = T, sizes partition N, 2m <= T.

    Budgets must also be non-increasing (group 1 is the baseline group).
    """
    K = len(budgets)
    if T <= 0 or K <= 0 or len(sizes) != K:
        raise ValueError("need T > 0 and one size per group")
    if budgets[0] != T:
        raise ValueError("the baseline group must have s_1 = T")
    for s in budgets:
        if s <= 0 or T % s:
            raise ValueError("every budget s_k must divide T")
    if any(budgets[k] < budgets[k + 1] for k in range(K - 1)):
        raise ValueError("budgets must be non-increasing")
    if any(n < 0 for n in sizes) or sum(sizes) != N:
        raise ValueError("group sizes must partition the N tokens")
    if m < 0 or 2 * m > T:
        raise ValueError("need 0 <= 2m <= T")


def group_periods(T: int, budgets) -> list[int]:
    """p_k = T / s_k: the gap, in global iterations, between two steps of group k (§2.1)."""
    return [T // s for s in budgets]


def active_table(T: int, budgets, m: int) -> np.ndarray:
    """(T, K) bool: group k is active at iteration i.

    §2.1: group k runs when i mod (T/s_k) = 0 (the baseline group, period 1,
    runs at every i).  §2.4: the first and last m iterations run every token.
    """
    p = group_periods(T, budgets)
    tab = np.zeros((T, len(budgets)), dtype=bool)
    for i in range(T):
        window_full = i < m or i >= T - m
        for k in range(len(budgets)):
            tab[i, k] = window_full or (i % p[k] == 0)
    return tab


def active_counts(tab: np.ndarray, sizes) -> np.ndarray:
    """|A_i| = sum of the sizes of the groups active at iteration i."""
    return np.array([sum(int(n) for n, a in zip(sizes, row) if a) for row in tab], dtype=np.int64)


def sigma_schedule(T: int, kind: int, shift: float = 1.0) -> np.ndarray:
    """sigma_0..sigma_T stored as float32.

    The pages use only the increment sigma_{i+1} - sigma_i (§2.3).  kind 0:
    sigma_i = 1 - i/T.  kind 1: the shifted flow-matching form
    s*sigma / (1 + (s - 1)*sigma) of the same base.
    """
    out = np.empty(T + 1, dtype=np.float32)
    for i in range(T + 1):
        sig = 1.0 - i / T
        if kind == 1:
            sig = shift * sig / (1.0 + (shift - 1.0) * sig)
        elif kind != 0:
            raise ValueError("sigma kind must be 0 or 1")
        out[i] = np.float32(sig)
    return out


# ====================================================================== §2.1 dynamic selection

def l1_relative_change(v_new: np.ndarray, v_prev: np.ndarray, eps: float = SCORE_EPS) -> np.ndarray:
    """Per-token L1 relative change of the velocity prediction (§2.1, dynamic token selection)."""
    v_new = np.asarray(v_new, F64)
    v_prev = np.asarray(v_prev, F64)
    return np.abs(v_new - v_prev).sum(axis=1) / (np.abs(v_prev).sum(axis=1) + eps)


def score_order_key(score_f32: np.ndarray) -> np.ndarray:
    """Order key of a float32 score: larger key = larger score; NaN counts as +inf, <= 0 as 0."""
    s = np.asarray(score_f32, dtype=np.float32)
    key = s.view(np.uint32).astype(np.int64)
    key[s <= 0] = 0
    key[np.isnan(s)] = 0x7F800000
    return key


def select_groups(score_f32: np.ndarray, sizes, pinned=None) -> tuple[np.ndarray, np.ndarray]:
    """Assign tokens to groups G_1..G_K by their score (§2.1).

    Tokens are ranked by (score descending, index ascending); the first n_1
    go to G_1 (full budget), the next n_2 to G_2, ..., so slowly-evolving
    tokens (low L1 change) land in the groups with the fewest steps.
    Returns group[N] (int8, 0-based) and order[N]: the groups' token lists
    concatenated in group order, each list ascending by token index.

    pinned (bool[N], optional): image-to-video reading of §4 (the conditioning
    image must survive): pinned tokens rank ahead of every other token, among
    themselves by index, so they fill G_1 first whatever their score.
    """
    key = score_order_key(score_f32)
    N = key.shape[0]
    if pinned is not None:
        key = key.copy()
        key[np.asarray(pinned, bool)] = 1 << 32       # above every 32-bit order key
    ranked = np.lexsort((np.arange(N), -key))
    group = np.empty(N, dtype=np.int8)
    start = 0
    for k, n_k in enumerate(sizes):
        group[ranked[start:start + n_k]] = k
        start += n_k
    order = np.concatenate([np.sort(np.nonzero(group == k)[0]) for k in range(len(sizes))])
    return group, order.astype(np.int32)


def active_rows(order: np.ndarray, sizes, active_groups) -> np.ndarray:
    """A_i: the token lists of the groups active at this iteration, in group order."""
    parts, start = [], 0
    for n_k, a in zip(sizes, active_groups):
        if a:
            parts.append(order[start:start + n_k])
        start += n_k
    return np.concatenate(parts).astype(np.int32) if parts else np.zeros(0, np.int32)


# ====================================================================== block arithmetic

def layer_norm(x, gamma=None, beta=None, eps: float = LN_EPS):
    """LayerNorm over the last axis (biased variance); affine when gamma/beta are given."""
    x = np.asarray(x, F64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, F64) + np.asarray(beta, F64)
    return y


def rms_norm(x, g, eps: float = RMS_EPS):
    """RMSNorm over the whole last axis (all heads together), times the gain g."""
    x = np.asarray(x, F64)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * np.asarray(g, F64)


def gelu_tanh(x):
    x = np.asarray(x, F64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def linear(x, w, b):
    """y = x W^T + b for W stored [out, in]."""
    return np.asarray(x, F64) @ np.asarray(w, F64).T + np.asarray(b, F64)


def rope_3d(x, pos):
    """3D rotary embedding of each 128-wide head at token positions (frame, row, column).

    Channels [0,44) rotate with the frame index, [44,86) with the row, [86,128)
    with the column.  In an axis segment of width w, channel pair j = (2j, 2j+1)
    rotates by the angle pos_axis * 10000^(-2j/w): (a, b) -> (a cos - b sin, a sin + b cos).
    """
    x = np.asarray(x, F64)
    M, width = x.shape
    H = width // HEAD_DIM
    xh = x.reshape(M, H, HEAD_DIM)
    out = xh.copy()
    pos = np.asarray(pos, F64)
    off = 0
    for axis, w in enumerate(ROPE_SPLIT):
        for j in range(w // 2):
            ang = pos[:, axis] * ROPE_THETA ** (-2.0 * j / w)
            c, s = np.cos(ang)[:, None], np.sin(ang)[:, None]
            a, b = xh[:, :, off + 2 * j], xh[:, :, off + 2 * j + 1]
            out[:, :, off + 2 * j] = a * c - b * s
            out[:, :, off + 2 * j + 1] = a * s + b * c
        off += w
    return out.reshape(M, width)


def attention(q, K, V):
    """Per head: softmax(q K^T / sqrt(128)) V.  q: (M, H*128); K, V: (L, H*128)."""
    q, K, V = (np.asarray(a, F64) for a in (q, K, V))
    M, width = q.shape
    H = width // HEAD_DIM
    out = np.empty((M, width), F64)
    for h in range(H):
        sl = slice(h * HEAD_DIM, (h + 1) * HEAD_DIM)
        logits = q[:, sl] @ K[:, sl].T / np.sqrt(HEAD_DIM)
        logits -= logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p /= p.sum(axis=1, keepdims=True)
        out[:, sl] = p @ V[:, sl]
    return out


def context_kv(bw, ctx):
    """Cross-attention keys/values of the text context, projected once per run (k RMSNorm'd)."""
    D = bw.w_o.shape[0]
    kv = linear(ctx, bw.w_kv2, bw.b_kv2)
    return rms_norm(kv[:, :D], bw.g_k2), kv[:, D:]


def qkv_projection(bw, X, pos):
    """Steps 1-4 of the block on rows X at positions pos: returns q, k (normed, rotated) and v."""
    D = X.shape[1]
    mod = np.asarray(bw.mod, F64)
    h = layer_norm(X) * (1.0 + mod[1]) + mod[0]
    qkv = linear(h, bw.w_qkv, bw.b_qkv)
    q = rope_3d(rms_norm(qkv[:, :D], bw.g_q), pos)
    k = rope_3d(rms_norm(qkv[:, D:2 * D], bw.g_k), pos)
    return q, k, qkv[:, 2 * D:]


def block_tail(bw, X, o, ctx_kv):
    """Steps 7-9 of the block: gated output projection, cross-attention, gated FFN."""
    mod = np.asarray(bw.mod, F64)
    X = np.asarray(X, F64) + mod[2] * linear(o, bw.w_o, bw.b_o)
    if ctx_kv is not None:
        y = layer_norm(X, bw.ln_c_g, bw.ln_c_b)
        q2 = rms_norm(linear(y, bw.w_q2, bw.b_q2), bw.g_q2)
        X = X + linear(attention(q2, ctx_kv[0], ctx_kv[1]), bw.w_o2, bw.b_o2)
    h = layer_norm(X) * (1.0 + mod[4]) + mod[3]
    return X + mod[5] * linear(gelu_tanh(linear(h, bw.w_1, bw.b_1)), bw.w_2, bw.b_2)


def dit_block_active(bw, X_A, idx, pos_all, Kc, Vc, ctx_kv=None):
    """One block on the active rows only (§2.2, gather form).

    X_A: (M, D) rows of the active tokens idx (in that order).  Kc, Vc: the
    layer's (N, D) cache.  Only the active rows are projected; their fresh K/V
    overwrite the cache rows idx and every other row stays as it was; each
    active query then attends to all N cache rows.  Returns (X_A out, Kc', Vc').
    """
    idx = np.asarray(idx, np.int64)
    q, k, v = qkv_projection(bw, X_A, np.asarray(pos_all)[idx])
    Kc = np.array(Kc, F64, copy=True)
    Vc = np.array(Vc, F64, copy=True)
    Kc[idx] = k
    Vc[idx] = v
    o = attention(q, Kc, Vc)
    return block_tail(bw, X_A, o, ctx_kv), Kc, Vc


def dit_block_masked(bw, X_all, active, pos_all, Kc, Vc, ctx_kv=None):
    """Brute-force twin of dit_block_active for tiny N (mask form, explicit loops).

    Runs the projections for every token, keeps the fresh K/V only where the
    token is active (the stale cache row elsewhere), attends with every active
    query over all N rows one (query, head, key) at a time, and returns the
    active tokens' outputs in ascending token order plus the caches.
    """
    X_all = np.asarray(X_all, F64)
    N, D = X_all.shape
    H = D // HEAD_DIM
    q, k, v = qkv_projection(bw, X_all, pos_all)
    K_used = np.where(np.asarray(active)[:, None], k, np.asarray(Kc, F64))
    V_used = np.where(np.asarray(active)[:, None], v, np.asarray(Vc, F64))
    rows = [n for n in range(N) if active[n]]
    o = np.zeros((len(rows), D), F64)
    scale = 1.0 / np.sqrt(HEAD_DIM)
    for r, n in enumerate(rows):
        for h in range(H):
            sl = slice(h * HEAD_DIM, (h + 1) * HEAD_DIM)
            logits = [float(np.dot(q[n, sl], K_used[j, sl])) * scale for j in range(N)]
            top = max(logits)
            w = [np.exp(l - top) for l in logits]
            tot = sum(w)
            acc = np.zeros(HEAD_DIM, F64)
            for j in range(N):
                acc += (w[j] / tot) * V_used[j, sl]
            o[r, sl] = acc
    out = block_tail(bw, X_all[rows], o, ctx_kv)
    return out, K_used, V_used


# ====================================================================== models

def head_projection(pm, X):
    """Output head of the patch model: LayerNorm + (shift, scale) modulation, then D -> C."""
    hm = np.asarray(pm.head_mod, F64)
    return linear(layer_norm(X) * (1.0 + hm[1]) + hm[0], pm.w_out, pm.b_out)


def patch_model_active(pm, x_A, idx, pos_all, caches, ctx_kvs=None):
    """Velocity of the active tokens through patch-embed, every block and the head."""
    X = linear(x_A, pm.w_in, pm.b_in)
    new_caches = []
    for b, bw in enumerate(pm.blocks):
        X, Kc, Vc = dit_block_active(bw, X, idx, pos_all, caches[b][0], caches[b][1],
                                     None if ctx_kvs is None else ctx_kvs[b])
        new_caches.append((Kc, Vc))
    return head_projection(pm, X), new_caches


# ====================================================================== §2.3 cached Euler

def cached_euler(x, v_hat, v_A, idx, dsigma):
    """§2.3: v_hat[A_i] <- fresh v_A, then every token x_n += (sigma_{i+1} - sigma_i) * v_hat_n."""
    v_hat = np.array(v_hat, F64, copy=True)
    v_hat[np.asarray(idx, np.int64)] = np.asarray(v_A, F64)
    return np.asarray(x, F64) + float(dsigma) * v_hat, v_hat


# ====================================================================== one iteration / the loop

def hsa_iteration(state: dict, i: int, plan: dict, velocity_fn) -> dict:
    """One HSA denoising iteration i, in the order the summary describes.

    state: x (N,C), v_hat (N,C), order (N,) group lists, caches (model state).
    plan:  T, budgets, sizes, m, sigmas (float32 T+1), table (T,K).
    velocity_fn(x_A, idx, caches) -> (v_A, caches').

    1. A_i from the schedule (§2.1, §2.4);
    2. v_A from the model on the active rows with the KV cache (§2.2);
    3. if every token is active, score = L1 relative change of v_A against
       the cached v_hat (before it is overwritten);
    4-5. cached Euler update of all N tokens (§2.3);
    6. after a full step, regroup the tokens by that score (§2.1).
    """
    sizes = plan["sizes"]
    act = plan["table"][i]
    idx = active_rows(state["order"], sizes, act)
    x_A = np.asarray(state["x"], F64)[idx]
    v_A, caches = velocity_fn(x_A, idx, state["caches"])
    full = len(idx) == state["x"].shape[0]
    score = None
    if full:
        prev = np.asarray(state["v_hat"], F64)[idx]
        score = np.zeros(len(idx), F64)          # token order
        score[idx] = l1_relative_change(v_A, prev)
    dsig = F64(plan["sigmas"][i + 1]) - F64(plan["sigmas"][i])
    x, v_hat = cached_euler(state["x"], state["v_hat"], v_A, idx, dsig)
    order = state["order"]
    group = state.get("group")
    if full and plan.get("static_groups") is None:
        group, order = select_groups(score.astype(np.float32), sizes, plan.get("pinned"))
    return {"x": x, "v_hat": v_hat, "order": order, "group": group, "caches": caches,
            "idx": idx, "score": score, "v_A": v_A}


def make_plan(T, budgets, sizes, m, sigma_kind, shift, N, pinned=None, static_groups=None) -> dict:
    """static_groups (int[N], optional): a fixed partition for the whole run (token n in group
    static_groups[n]; group k must hold sizes[k] tokens) instead of regrouping by score after full
    steps -- the plainest static alternative to the dynamic selection of §2.1."""
    validate_plan(T, budgets, sizes, N, m)
    if static_groups is not None:
        g = np.asarray(static_groups, np.int64)
        if g.shape != (N,) or [int(np.sum(g == k)) for k in range(len(sizes))] != list(sizes):
            raise ValueError("static groups must give group k exactly sizes[k] tokens")
    return {"T": T, "budgets": list(budgets), "sizes": list(sizes), "m": m,
            "sigmas": sigma_schedule(T, sigma_kind, shift), "table": active_table(T, budgets, m),
            "pinned": None if pinned is None else np.asarray(pinned, bool),
            "static_groups": None if static_groups is None else np.asarray(static_groups, np.int64)}


def static_order(static_groups, K: int) -> np.ndarray:
    """The groups' token lists of a fixed partition, concatenated in group order, each ascending."""
    g = np.asarray(static_groups, np.int64)
    return np.concatenate([np.nonzero(g == k)[0] for k in range(K)]).astype(np.int32)


def conditioning_frame_tokens(pos: np.ndarray, n_frames: int = 1) -> np.ndarray:
    """Image-to-video reading of §4: the tokens of the first n_frames latent frames carry the
    conditioning image; pos is the (N, 3) (frame, row, column) table of the tokens."""
    return np.asarray(pos)[:, 0] < n_frames


def hsa_denoise(x0, v_hat0, plan, velocity_fn, caches0, keep_states: bool = False):
    """The whole loop: T iterations of hsa_iteration from x0 with cached velocities v_hat0.

    The order before step 0 is the identity (step 0 is always a full step, so
    it never decides which tokens run); with static groups it is their fixed order.
    """
    N = x0.shape[0]
    order0 = np.arange(N, dtype=np.int32) if plan.get("static_groups") is None else \
        static_order(plan["static_groups"], len(plan["sizes"]))
    state = {"x": np.asarray(x0, F64), "v_hat": np.asarray(v_hat0, F64),
             "order": order0, "group": None, "caches": caches0}
    states = []
    for i in range(plan["T"]):
        state = hsa_iteration(state, i, plan, velocity_fn)
        if keep_states:
            states.append(state)
    return state, states

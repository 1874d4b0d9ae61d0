"""Step-by-step comparison of a whole HSA run on the GPU with the oracle's run.

The oracle runs the loop on its own from the seeded inputs (O.hsa_denoise); no
value of the CUDA run enters it.  The CUDA run then takes the same iterations one
at a time, and after each one its outputs are compared with the oracle's outputs
of that iteration: the velocity of the active rows, the latent, the cached
velocities v_hat (rows of skipped tokens bit-identical to before the step), the
KV caches (skipped rows byte-identical to before the step, fresh rows close to
the oracle's) and, at full steps, the L1 scores.

Two correct runs can part only at the regrouping: a token whose score sits
within rounding of a group boundary may land on either side.  At every full
step the CUDA run's own partition (its selection kernel on its own scores) is
therefore checked against the oracle's scores widened by a per-token bound
derived from the two runs' velocity differences (see score_bound), and the CUDA
run then continues on the oracle's partition, written into its order buffer (a
test input, oracle to CUDA), so that both runs keep the same active sets and
every later iteration stays comparable token by token.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import hsa_oracle as O
from tests._util import TOL_F32, host, rel_l2

# relative fp32 evaluation error allowed in the CUDA score on top of the derived bound: the
# kernel sums at most a few thousand terms per token in fp32 (error below 1e-5 relative)
SCORE_F32_SLACK = 1e-5


def score_bound(v_gpu, p_gpu, v_ref, p_ref, s_gpu):
    """Per-token bound on |s_gpu - s_ref| for the L1 relative change s = a / b,
    a = sum_c |v - p|, b = sum_c |p| + eps, computed from two runs' inputs.

    Triangle inequality: |a - a'| <= sum|v - v'| + sum|p - p'| = e_a and
    |b - b'| <= sum|p - p'| = e_b, so s - s' = (a - a')/b + s'(b' - b)/b gives
    |s - s'| <= (e_a + s' e_b) / b; plus the fp32 evaluation error of s'."""
    v_gpu, p_gpu, v_ref, p_ref = (np.asarray(a, np.float64) for a in (v_gpu, p_gpu, v_ref, p_ref))
    e_p = np.abs(p_gpu - p_ref).sum(axis=1)
    e_a = np.abs(v_gpu - v_ref).sum(axis=1) + e_p
    b = np.abs(p_ref).sum(axis=1) + O.SCORE_EPS
    s = np.asarray(s_gpu, np.float64)
    return (e_a + s * e_p) / b + SCORE_F32_SLACK * s + 1e-7


def check_partition(order_gpu, score_ref, delta, sizes, pinned=None, what=""):
    """The CUDA partition must be valid (each group's list ascending, all N tokens once) and
    consistent with the oracle's scores within +-delta: for every boundary, each token placed
    above it could outrank each token placed below it (pinned tokens rank above all others)."""
    N = len(order_gpu)
    starts = np.concatenate([[0], np.cumsum(sizes)])
    assert np.array_equal(np.sort(order_gpu), np.arange(N)), f"{what}: not a permutation"
    g = np.empty(N, np.int64)
    for k in range(len(sizes)):
        seg = order_gpu[starts[k]:starts[k + 1]]
        assert np.all(np.diff(seg) > 0), f"{what}: group {k} list not ascending"
        g[seg] = k
    hi_key = np.asarray(score_ref, np.float64) + delta
    lo_key = np.asarray(score_ref, np.float64) - delta
    if pinned is not None:
        hi_key[pinned] = np.inf
        lo_key[pinned] = np.inf
    for k in range(len(sizes) - 1):
        above, below = g <= k, g > k
        if above.any() and below.any():
            assert hi_key[above].min() >= lo_key[below].max(), \
                f"{what}: boundary {k}: a token placed below outranks one placed above beyond the score bound"
    return g


def _as_list(caches):
    return list(caches) if isinstance(caches, list) else [caches]


def run_stepwise(run, gpu_caches, gpu_velocity, x0, vh0, plan, velocity_fn, caches0, close, bf16: bool):
    """Runs `run` (an HSARun at step 0) iteration by iteration against the oracle's run of `plan`.

    gpu_caches() -> list of (K, V) device tensors of the model's layers; gpu_velocity(M) -> the
    device tensor holding the last step's velocity rows; velocity_fn / caches0 as for
    O.hsa_denoise; close(got, want, what) the tolerance check.  Returns (oracle final state,
    per-step statistics)."""
    final, states = O.hsa_denoise(x0, vh0, plan, velocity_fn, caches0, keep_states=True)
    N = x0.shape[0]
    sizes = plan["sizes"]
    pinned = plan.get("pinned")
    regroups = plan.get("static_groups") is None
    vh_ref_prev = np.asarray(vh0, np.float64)
    stats = []
    for i, st in enumerate(states):
        what = f"step {i}"
        vh_before = host(run.vhat).copy()
        caches_before = [(host(k).copy(), host(v).copy()) for k, v in gpu_caches()]
        rec = []
        run.step(rec)
        r = rec[0]
        idx = np.asarray(st["idx"], np.int64)
        assert r["M"] == len(idx) and np.array_equal(r["idx"], idx), f"{what}: active set"
        M = len(idx)
        skipped = np.setdiff1d(np.arange(N), idx)
        vA = host(gpu_velocity(M)).astype(np.float64)
        close(vA, st["v_A"], f"{what}: velocity of the active rows")
        x = host(run.x)
        close(x - x0, st["x"] - x0, f"{what}: latent displacement")
        vh = host(run.vhat)
        assert np.array_equal(vh[skipped], vh_before[skipped]), f"{what}: cached velocities of skipped tokens"
        close(vh[idx], st["v_hat"][idx], f"{what}: fresh cached velocities")
        for b, ((kb, vb), (ka, va), (ko, vo)) in enumerate(zip(
                caches_before, [(host(k), host(v)) for k, v in gpu_caches()], _as_list(st["caches"]))):
            assert np.array_equal(ka[skipped], kb[skipped]) and np.array_equal(va[skipped], vb[skipped]), \
                f"{what}: layer {b} cache rows of skipped tokens changed"
            close(ka[idx], ko[idx], f"{what}: layer {b} fresh K rows")
            close(va[idx], vo[idx], f"{what}: layer {b} fresh V rows")
        info = {"i": i, "M": M, "full": bool(r["full"]), "regrouped": False}
        if r["full"] and regroups:
            s_gpu = np.asarray(r["score"], np.float64)
            s_ref = np.asarray(st["score"], np.float64)
            # rows in token order (the oracle's scores and the CUDA score buffer are by token)
            v_gpu_tok = np.empty_like(vA)
            v_gpu_tok[idx] = vA
            v_ref_tok = np.empty_like(vA)
            v_ref_tok[idx] = st["v_A"]
            delta = score_bound(v_gpu_tok, vh_before, v_ref_tok, vh_ref_prev, s_gpu)
            err = np.abs(s_gpu - s_ref)
            assert np.all(err <= delta), f"{what}: score beyond its derived bound (worst {np.max(err - delta):.3e})"
            if not bf16 or np.array_equal(vh_before, vh_ref_prev.astype(np.float32)):
                tol = TOL_F32 if not bf16 else 2e-2
                assert rel_l2(s_gpu, s_ref) <= tol, f"{what}: score rel-L2 {rel_l2(s_gpu, s_ref):.3e}"
            g = check_partition(r["order"], s_ref, delta, sizes, pinned, what)
            g_ref = np.empty(N, np.int64)
            starts = np.concatenate([[0], np.cumsum(sizes)])
            for k in range(len(sizes)):
                g_ref[st["order"][starts[k]:starts[k + 1]]] = k
            info.update(regrouped=True, moved=int(np.sum(g != g_ref)), score_rel_l2=rel_l2(s_gpu, s_ref),
                        max_bound=float(np.max(delta)))
            # continue on the oracle's partition so that both runs keep the same active sets
            run.order.copy_(torch.from_numpy(np.ascontiguousarray(st["order"], np.int32)).to(run.order.device))
        stats.append(info)
        vh_ref_prev = np.asarray(st["v_hat"], np.float64)
    return final, stats

"""Pins of the CPU oracle against facts fixed outside it.

Each test ties one oracle function to something it does not compute itself:
hand-worked fixtures derived from the summary's rules (tests/golden/), closed
forms, invariants, brute force on tiny inputs, and torch float64 library
routines (layer_norm, rms_norm, gelu, scaled_dot_product_attention, a
complex-number rotary embedding) composed independently.  The planted-mistake
tests at the end break the oracle on purpose (on the CPU, by monkeypatching)
and check that a pin catches each mistake.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import hsa_oracle as O
from token_sparse_denoising_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _read_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ schedule (§2.1, §2.4)

def test_schedule_tiny_matches_hand_table():
    rows = _read_rows("schedule_T8_budgets8-4_m1.txt")
    want = np.array([[int(a) for a in r[1:]] for r in rows], dtype=bool)
    assert np.array_equal(O.active_table(8, [8, 4], 1), want)


def test_schedule_wan_loop_matches_hand_lists():
    rows = {r[0]: r[1:] for r in _read_rows("schedule_T40_budgets40-20-10_m4.txt")}
    tab = O.active_table(40, [40, 20, 10], 4)
    for k in range(3):
        assert list(np.nonzero(tab[:, k])[0]) == [int(v) for v in rows[f"G{k + 1}"]]
    sizes = S.group_sizes(32760, (0.25, 0.25, 0.5))
    assert sizes == [8190, 8190, 16380]
    frac = O.active_counts(tab, sizes).mean() / 32760
    assert frac == pytest.approx(float(rows["mean_active_fraction"][0]), abs=1e-15)


@pytest.mark.parametrize("T", [1, 2, 4, 8, 12, 30, 40, 60, 64])
def test_rule_alone_fires_exactly_s_k_times(T):
    divisors = [s for s in range(T, 0, -1) if T % s == 0]
    tab = O.active_table(T, divisors, 0)
    for k, s in enumerate(divisors):
        assert tab[:, k].sum() == s
    assert tab[:, 0].all()                   # baseline group s_1 = T runs every step


@pytest.mark.parametrize("T,budgets,m", [(8, [8, 4], 1), (40, [40, 20, 10], 4), (40, [40, 8, 5, 1], 3),
                                         (12, [12, 6, 4, 3], 0), (10, [10, 5, 2], 5)])
def test_count_closed_form(T, budgets, m):
    """count_k = 2m + #{multiples of p_k in [m, T-m)} = 2m + ceil((T-m)/p) - ceil(m/p)."""
    tab = O.active_table(T, budgets, m)
    for k, s in enumerate(budgets):
        p = T // s
        want = 2 * m + (-(-(T - m) // p)) - (-(-m // p))
        assert tab[:, k].sum() == want
    assert tab[:m].all() and tab[T - m:].all()


def test_validate_plan_rejects():
    ok = dict(T=8, budgets=[8, 4], sizes=[4, 4], N=8, m=1)
    O.validate_plan(**ok)
    for bad in (dict(budgets=[8, 3]), dict(budgets=[4, 4]), dict(budgets=[8, 8, 4], sizes=[4, 4]),
                dict(sizes=[4, 5]), dict(m=5), dict(budgets=[4, 8])):
        with pytest.raises(ValueError):
            O.validate_plan(**{**ok, **bad})


def test_sigma_schedules():
    lin = O.sigma_schedule(8, 0)
    assert lin[0] == 1.0 and lin[-1] == 0.0
    assert np.allclose(lin, 1 - np.arange(9) / 8, atol=0)   # all exactly representable
    sh = O.sigma_schedule(40, 1, 5.0)
    assert sh[0] == 1.0 and sh[-1] == 0.0 and np.all(np.diff(sh) < 0)
    # sigma = 0.5 (i = 20) shifted by 5: 2.5 / 3
    assert sh[20] == np.float32(2.5 / 3.0)


# ------------------------------------------------------------------ selection (§2.1)

def test_score_hand_example():
    rows = {r[0]: [float(v) for v in r[1:]] for r in _read_rows("score_example.txt")}
    got = O.l1_relative_change(np.array([rows["v_new"]]), np.array([rows["v_prev"]]))
    assert got[0] == pytest.approx(rows["score"][0], rel=1e-8)


def test_score_invariants():
    r = np.random.default_rng(0)
    v = r.standard_normal((50, 64))
    w = r.standard_normal((50, 64))
    assert np.all(O.l1_relative_change(v, v) == 0)
    a = O.l1_relative_change(w, v)
    assert np.allclose(O.l1_relative_change(3 * w, 3 * v), a, rtol=1e-6)   # eps-level difference
    assert np.allclose(O.l1_relative_change(w[:, ::-1], v[:, ::-1]), a, rtol=1e-12)


def test_selection_hand_example():
    rows = {r[0]: r[1:] for r in _read_rows("selection_example.txt")}
    scores = np.array([float(v) for v in rows["scores"]], np.float32)
    group, order = O.select_groups(scores, [int(v) for v in rows["sizes"]])
    assert list(group) == [int(v) for v in rows["group"]]
    assert list(order) == [int(v) for v in rows["order"]]


def _brute_rank(scores):
    """rank(n) = #{j : s_j > s_n or (s_j == s_n and j < n)}, NaN as +inf, <=0 as 0 (pure Python)."""
    def val(s):
        if math.isnan(s):
            return math.inf
        return max(float(s), 0.0)
    vals = [val(s) for s in scores]
    return [sum(1 for j in range(len(vals)) if vals[j] > vals[n] or (vals[j] == vals[n] and j < n))
            for n in range(len(vals))]


@pytest.mark.parametrize("seed", range(6))
def test_selection_vs_brute_force(seed):
    r = np.random.default_rng(seed)
    N = int(r.integers(1, 200))
    scores = r.choice([0.0, 0.25, 0.5, 1.0, np.nan], size=N).astype(np.float32) if seed % 2 else \
        r.random(N).astype(np.float32)
    K = int(r.integers(1, 5))
    cuts = np.sort(r.integers(0, N + 1, size=K - 1))
    sizes = list(np.diff(np.concatenate([[0], cuts, [N]])).astype(int))
    group, order = O.select_groups(scores, sizes)
    rank = _brute_rank(list(scores))
    bounds = np.cumsum(sizes)
    for n in range(N):
        assert group[n] == int(np.searchsorted(bounds, rank[n], side="right"))
    assert [int(np.sum(group == k)) for k in range(K)] == sizes
    start = 0
    for k, nk in enumerate(sizes):
        seg = list(order[start:start + nk])
        assert seg == sorted(seg) and all(group[t] == k for t in seg)
        start += nk


def test_selection_pinned_hand_example():
    rows = {r[0]: r[1:] for r in _read_rows("selection_pinned_example.txt")}
    scores = np.array([float(v) for v in rows["scores"]], np.float32)
    pinned = np.array([int(v) for v in rows["pinned"]], bool)
    for case in ("a", "b"):
        group, order = O.select_groups(scores, [int(v) for v in rows["sizes_" + case]], pinned)
        assert list(group) == [int(v) for v in rows["group_" + case]], case
        assert list(order) == [int(v) for v in rows["order_" + case]], case


def _brute_rank_pinned(scores, pinned):
    """rank(n) = #{j ranked before n}: pinned before unpinned; pinned by index; unpinned by
    (value descending, index ascending), NaN as +inf, <= 0 as 0 (pure Python)."""
    def val(s):
        return math.inf if math.isnan(s) else max(float(s), 0.0)
    vals = [val(s) for s in scores]

    def before(j, n):
        if pinned[j] != pinned[n]:
            return bool(pinned[j])
        if pinned[j]:
            return j < n
        return vals[j] > vals[n] or (vals[j] == vals[n] and j < n)
    return [sum(1 for j in range(len(vals)) if before(j, n)) for n in range(len(vals))]


@pytest.mark.parametrize("seed", range(6))
def test_selection_pinned_vs_brute_force(seed):
    r = np.random.default_rng(100 + seed)
    N = int(r.integers(1, 150))
    scores = r.choice([0.0, 0.25, 0.5, 1.0, np.nan], size=N).astype(np.float32) if seed % 2 else \
        r.random(N).astype(np.float32)
    pinned = r.random(N) < (0.05, 0.3, 0.9)[seed % 3]
    K = int(r.integers(1, 5))
    cuts = np.sort(r.integers(0, N + 1, size=K - 1))
    sizes = list(np.diff(np.concatenate([[0], cuts, [N]])).astype(int))
    group, order = O.select_groups(scores, sizes, pinned)
    rank = _brute_rank_pinned(list(scores), list(pinned))
    bounds = np.cumsum(sizes)
    for n in range(N):
        assert group[n] == int(np.searchsorted(bounds, rank[n], side="right"))
    n_pin = int(pinned.sum())
    if n_pin <= sizes[0]:
        assert np.all(group[pinned] == 0)          # every pinned token keeps the full budget


def test_selection_without_pins_is_unchanged():
    r = np.random.default_rng(7)
    scores = r.random(90).astype(np.float32)
    scores[::11] = np.nan
    sizes = [30, 30, 30]
    g0, o0 = O.select_groups(scores, sizes)
    g1, o1 = O.select_groups(scores, sizes, np.zeros(90, bool))
    assert np.array_equal(g0, g1) and np.array_equal(o0, o1)


def test_conditioning_frame_tokens_are_the_first_frame():
    grid = S.Grid(3, 2, 4)
    pos = S.token_positions(grid)
    mask = O.conditioning_frame_tokens(pos)
    assert mask.sum() == 8 and np.all(np.nonzero(mask)[0] == np.arange(8))   # raster order: frame 0 first
    assert O.conditioning_frame_tokens(pos, 2).sum() == 16


def test_static_groups_never_regroup():
    """With a fixed partition every full step keeps the order; the active rows of each step are the
    fixed groups' lists; a partition with the wrong sizes is rejected."""
    N, T = 12, 4
    groups = np.array([1, 0, 1, 0, 0, 1, 1, 0, 1, 0, 0, 1])
    plan = O.make_plan(T, [4, 2], [6, 6], 1, 0, 1.0, N, static_groups=groups)
    order = O.static_order(groups, 2)
    assert list(order) == [1, 3, 4, 7, 9, 10, 0, 2, 5, 6, 8, 11]
    model = lambda xA, idx, c: (xA * 0.5 + idx[:, None], c)
    x0, vh0 = np.ones((N, 4)), np.zeros((N, 4))
    _, states = O.hsa_denoise(x0, vh0, plan, model, None, keep_states=True)
    for i, st in enumerate(states):
        assert list(st["order"]) == list(order)
        assert list(st["idx"]) == (list(order) if i in (0, 2, 3) else list(order[:6]))
    with pytest.raises(ValueError):
        O.make_plan(T, [4, 2], [6, 6], 1, 0, 1.0, N, static_groups=np.zeros(N, int))


def test_active_rows_prefix_for_nested_budgets():
    order = np.array([3, 5, 0, 2, 1, 4], np.int32)
    assert list(O.active_rows(order, [2, 2, 2], [True, True, False])) == [3, 5, 0, 2]
    assert list(O.active_rows(order, [2, 2, 2], [True, False, True])) == [3, 5, 1, 4]


# ------------------------------------------------------------------ block arithmetic vs torch float64

def _t(a):
    return torch.tensor(np.asarray(a, np.float64))


def test_norms_and_gelu_vs_torch():
    r = np.random.default_rng(1)
    x = r.standard_normal((7, 256)) * 3 + 1
    g, b = r.standard_normal(256), r.standard_normal(256)
    assert np.allclose(O.layer_norm(x), F.layer_norm(_t(x), (256,), eps=1e-6).numpy(), atol=1e-12)
    assert np.allclose(O.layer_norm(x, g, b),
                       F.layer_norm(_t(x), (256,), _t(g), _t(b), eps=1e-6).numpy(), atol=1e-12)
    assert np.allclose(O.rms_norm(x, g), F.rms_norm(_t(x), (256,), _t(g), eps=1e-6).numpy(), atol=1e-12)
    assert np.allclose(O.gelu_tanh(x), F.gelu(_t(x), approximate="tanh").numpy(), atol=1e-12)


def test_attention_vs_torch_sdpa():
    r = np.random.default_rng(2)
    q, K, V = r.standard_normal((9, 256)), r.standard_normal((33, 256)), r.standard_normal((33, 256))
    ref = F.scaled_dot_product_attention(_t(q).view(9, 2, 128).transpose(0, 1),
                                         _t(K).view(33, 2, 128).transpose(0, 1),
                                         _t(V).view(33, 2, 128).transpose(0, 1))
    assert np.allclose(O.attention(q, K, V), ref.transpose(0, 1).reshape(9, 256).numpy(), atol=1e-12)


def test_attention_invariants():
    r = np.random.default_rng(3)
    q, V = r.standard_normal((4, 128)), r.standard_normal((20, 128))
    K = np.tile(r.standard_normal((1, 128)), (20, 1))        # identical keys -> mean of V
    assert np.allclose(O.attention(q, K, V), np.tile(V.mean(0), (4, 1)), atol=1e-12)
    K2 = np.zeros((20, 128)); K2[7, 0] = 1e4                 # one dominant key -> its value
    q2 = np.zeros((1, 128)); q2[0, 0] = 1.0
    assert np.allclose(O.attention(q2, K2, V)[0], V[7], atol=1e-12)


def _rope_complex(x, pos):
    """Rotary embedding written with torch complex multiplication by unit phasors."""
    xt = _t(x)
    M, W = xt.shape
    H = W // 128
    ang = []
    for axis, w in enumerate((44, 42, 42)):
        inv = 10000.0 ** (-torch.arange(0, w, 2, dtype=torch.float64) / w)
        ang.append(torch.outer(_t(pos[:, axis]), inv))
    ang = torch.cat(ang, 1)                                   # (M, 64)
    z = torch.view_as_complex(xt.view(M, H, 64, 2).contiguous())
    z = z * torch.polar(torch.ones_like(ang), ang)[:, None, :]
    return torch.view_as_real(z).reshape(M, W).numpy()


def test_rope_vs_complex_form_and_properties():
    r = np.random.default_rng(4)
    x = r.standard_normal((30, 256))
    pos = r.integers(0, 60, size=(30, 3))
    y = O.rope_3d(x, pos)
    assert np.allclose(y, _rope_complex(x, pos), atol=1e-12)
    assert np.allclose(np.linalg.norm(y.reshape(30, 2, 64, 2), axis=-1),
                       np.linalg.norm(x.reshape(30, 2, 64, 2), axis=-1), atol=1e-12)
    assert np.allclose(O.rope_3d(x, np.zeros_like(pos)), x, atol=0)
    # relative position: <R(q, p), R(k, p')> depends only on p - p'
    q, k = r.standard_normal((1, 128)), r.standard_normal((1, 128))
    p1, p2 = np.array([[3, 5, 7]]), np.array([[1, 9, 2]])
    d = p2 - p1
    a = float(O.rope_3d(q, p1) @ O.rope_3d(k, p2).T)
    b = float(O.rope_3d(q, p1 + 11) @ O.rope_3d(k, p2 + 11).T)
    c = float(q @ O.rope_3d(k, d).T)
    assert a == pytest.approx(b, abs=1e-9) and a == pytest.approx(c, abs=1e-9)
    # unit vector on channel 0 at frame 1 -> (cos 1, sin 1) on the first pair
    e = np.zeros((1, 128)); e[0, 0] = 1.0
    out = O.rope_3d(e, np.array([[1, 0, 0]]))
    assert out[0, 0] == pytest.approx(math.cos(1.0)) and out[0, 1] == pytest.approx(math.sin(1.0))


def _torch_block(bw, X, pos, ctx):
    """The all-active block composed from torch float64 library ops (independent of the oracle)."""
    D = X.shape[1]
    H = D // 128
    X = _t(X)
    mod = _t(bw.mod)
    def lin(x, w, b):
        return F.linear(x, _t(w), _t(b))
    def rope(x):
        return torch.tensor(_rope_complex(x.numpy(), pos))
    def sdpa(q, k, v):
        M, L = q.shape[0], k.shape[0]
        o = F.scaled_dot_product_attention(q.view(M, H, 128).transpose(0, 1), k.view(L, H, 128).transpose(0, 1),
                                           v.view(L, H, 128).transpose(0, 1))
        return o.transpose(0, 1).reshape(M, D)
    h = F.layer_norm(X, (D,), eps=1e-6) * (1 + mod[1]) + mod[0]
    qkv = lin(h, bw.w_qkv, bw.b_qkv)
    q = rope(F.rms_norm(qkv[:, :D], (D,), _t(bw.g_q), eps=1e-6))
    k = rope(F.rms_norm(qkv[:, D:2 * D], (D,), _t(bw.g_k), eps=1e-6))
    v = qkv[:, 2 * D:]
    X = X + mod[2] * lin(sdpa(q, k, v), bw.w_o, bw.b_o)
    if ctx is not None:
        kv = lin(_t(ctx), bw.w_kv2, bw.b_kv2)
        k2 = F.rms_norm(kv[:, :D], (D,), _t(bw.g_k2), eps=1e-6)
        y = F.layer_norm(X, (D,), _t(bw.ln_c_g), _t(bw.ln_c_b), eps=1e-6)
        q2 = F.rms_norm(lin(y, bw.w_q2, bw.b_q2), (D,), _t(bw.g_q2), eps=1e-6)
        X = X + lin(sdpa(q2, k2, kv[:, D:]), bw.w_o2, bw.b_o2)
    h = F.layer_norm(X, (D,), eps=1e-6) * (1 + mod[4]) + mod[3]
    f = F.gelu(lin(h, bw.w_1, bw.b_1), approximate="tanh")
    return (X + mod[5] * lin(f, bw.w_2, bw.b_2)).numpy(), k.numpy(), v.numpy()


def _small_block(cross, seed=7):
    shape = S.BlockShape(256, 2, 512, cross, 16)
    bw = S.perturb_vectors(S.block_weights(seed, shape, bf16=False, std=0.2), seed)
    return shape, bw


@pytest.mark.parametrize("cross", [False, True])
def test_all_active_block_equals_dense_torch_block(cross):
    """With every token active the cache holds only fresh rows: the HSA block is the dense block."""
    shape, bw = _small_block(cross)
    grid = S.Grid(2, 4, 5)
    pos = S.token_positions(grid)
    N = grid.N
    X = S.normal(11, (N, 256))
    ctx = S.normal(12, (16, 256)) if cross else None
    Kc, Vc = S.normal(13, (N, 256)), S.normal(14, (N, 256))
    idx = np.arange(N)
    out, K2, V2 = O.dit_block_active(bw, X, idx, pos, Kc, Vc, None if ctx is None else O.context_kv(bw, ctx))
    ref, kref, vref = _torch_block(bw, X, pos, ctx)
    assert np.allclose(out, ref, atol=1e-10)
    assert np.allclose(K2, kref, atol=1e-10) and np.allclose(V2, vref, atol=1e-10)


def _torch_patch_model(pm, x, pos, ctx):
    """The all-active patch model composed from torch float64 library ops: patch embedding,
    the blocks (each the dense torch block), LayerNorm + (shift, scale) head, D -> C."""
    X = F.linear(_t(x), _t(pm.w_in), _t(pm.b_in)).numpy()
    for bw in pm.blocks:
        X = _torch_block(bw, X, pos, ctx)[0]
    hm = _t(pm.head_mod)
    h = F.layer_norm(_t(X), (X.shape[1],), eps=1e-6) * (1.0 + hm[1]) + hm[0]
    return F.linear(h, _t(pm.w_out), _t(pm.b_out)).numpy()


def test_patch_model_all_active_equals_torch_composition():
    """The loop workload's velocity model: with every token active the oracle's patch model equals
    the torch composition (patch embedding, dense blocks, modulated LayerNorm head)."""
    shape = S.BlockShape(256, 2, 512, True, 16)
    pm = S.patch_model_weights(3, shape, 64, 2, bf16=False, std=0.2)
    pm.blocks = [S.perturb_vectors(bw, 30 + i) for i, bw in enumerate(pm.blocks)]
    pm.b_in = S.normal(41, pm.b_in.shape, 0.3)
    pm.b_out = S.normal(42, pm.b_out.shape, 0.3)
    pm.head_mod = S.normal(43, pm.head_mod.shape, 0.3)
    grid = S.Grid(2, 4, 5)
    pos = S.token_positions(grid)
    N = grid.N
    x = S.normal(44, (N, 64))
    ctx = S.normal(45, (16, 256))
    idx = np.arange(N)
    caches = [(S.normal(46 + b, (N, 256)), S.normal(50 + b, (N, 256))) for b in range(2)]
    ctx_kvs = [O.context_kv(bw, ctx) for bw in pm.blocks]
    v, _ = O.patch_model_active(pm, x, idx, pos, caches, ctx_kvs)
    ref = _torch_patch_model(pm, x, pos, ctx)
    assert np.allclose(v, ref, atol=1e-10)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gather_form_equals_mask_form(seed):
    """Brute force on N = 64 tokens (1x8x8): gather form == mask form to fp64 round-off."""
    shape, bw = _small_block(cross=(seed == 1), seed=20 + seed)
    grid = S.Grid(1, 8, 8)
    pos = S.token_positions(grid)
    N = grid.N
    r = np.random.default_rng(seed)
    active = r.random(N) < 0.4
    active[r.integers(0, N)] = True
    X = S.normal(30 + seed, (N, 256))
    Kc, Vc = S.normal(40 + seed, (N, 256)), S.normal(50 + seed, (N, 256))
    ctx_kv = O.context_kv(bw, S.normal(60, (16, 256))) if seed == 1 else None
    idx = np.nonzero(active)[0]
    got, Kg, Vg = O.dit_block_active(bw, X[idx], idx, pos, Kc, Vc, ctx_kv)
    want, Km, Vm = O.dit_block_masked(bw, X, active, pos, Kc, Vc, ctx_kv)
    assert np.allclose(got, want, atol=1e-12, rtol=0)
    assert np.allclose(Kg, Km, atol=1e-12) and np.allclose(Vg, Vm, atol=1e-12)


def test_skipped_cache_rows_byte_identical():
    shape, bw = _small_block(False)
    grid = S.Grid(2, 4, 8)
    pos = S.token_positions(grid)
    N = grid.N
    Kc, Vc = S.normal(70, (N, 256)).astype(np.float64), S.normal(71, (N, 256)).astype(np.float64)
    idx = np.array([1, 4, 9, 33, 60], np.int64)
    _, K2, V2 = O.dit_block_active(bw, S.normal(72, (len(idx), 256)), idx, pos, Kc, Vc)
    skipped = np.setdiff1d(np.arange(N), idx)
    assert K2[skipped].tobytes() == Kc[skipped].tobytes()
    assert V2[skipped].tobytes() == Vc[skipped].tobytes()
    assert not np.array_equal(K2[idx], Kc[idx])


# ------------------------------------------------------------------ cached Euler (§2.3) and the loop

@pytest.mark.parametrize("T,budgets,fracs,m,kind", [(8, (8, 4), (.5, .5), 1, 0),
                                                   (40, (40, 20, 10), (.25, .25, .5), 4, 1),
                                                   (12, (12, 3), (.3, .7), 0, 0)])
def test_cached_euler_telescopes_for_constant_velocity(T, budgets, fracs, m, kind):
    """A model that always returns the same v gives x_T = x_0 + (sigma_T - sigma_0) v under any schedule."""
    N, C = 40, 6
    r = np.random.default_rng(T)
    v_const = r.standard_normal((N, C))
    x0 = r.standard_normal((N, C))
    plan = O.make_plan(T, budgets, S.group_sizes(N, fracs), m, kind, 5.0, N)
    final, _ = O.hsa_denoise(x0, r.standard_normal((N, C)), plan,
                             lambda xA, idx, c: (v_const[idx], c), None)
    sig = plan["sigmas"].astype(np.float64)
    assert np.allclose(final["x"], x0 + (sig[-1] - sig[0]) * v_const, atol=1e-12)


def test_all_active_iteration_is_standard_euler():
    N, C = 16, 5
    r = np.random.default_rng(5)
    x0, vh0 = r.standard_normal((N, C)), r.standard_normal((N, C))
    Wm = r.standard_normal((C, C))
    plan = O.make_plan(4, (4,), [N], 0, 0, 1.0, N)
    st, _ = O.hsa_denoise(x0, vh0, plan, lambda xA, idx, c: (xA @ Wm, c), None)
    x = x0.copy()
    sig = plan["sigmas"].astype(np.float64)
    for i in range(4):
        x = x + (sig[i + 1] - sig[i]) * (x @ Wm)
    assert np.allclose(st["x"], x, atol=1e-12)


def test_iteration_scores_full_steps_and_keeps_stale_velocity():
    N, C = 12, 3
    r = np.random.default_rng(6)
    x0, vh0 = r.standard_normal((N, C)), r.standard_normal((N, C))
    plan = O.make_plan(4, (4, 2), [6, 6], 0, 0, 1.0, N)
    model = lambda xA, idx, c: (xA * 2.0 + idx[:, None], c)
    _, states = O.hsa_denoise(x0, vh0, plan, model, None, keep_states=True)
    s0 = states[0]
    assert s0["score"] is not None and len(s0["idx"]) == N
    assert np.allclose(s0["score"], O.l1_relative_change(x0 * 2 + np.arange(N)[:, None], vh0))
    s1 = states[1]                                             # step 1: only G_1 runs
    assert s1["score"] is None and len(s1["idx"]) == 6
    skipped = np.setdiff1d(np.arange(N), s1["idx"])
    assert np.array_equal(s1["v_hat"][skipped], s0["v_hat"][skipped])
    assert list(s1["idx"]) == list(s0["order"][:6])


# ------------------------------------------------------------------ planted mistakes are caught

def test_planted_mistakes_are_caught(monkeypatch):
    shape, bw = _small_block(False)
    grid = S.Grid(2, 4, 5)
    pos = S.token_positions(grid)
    X = S.normal(11, (grid.N, 256))
    idx = np.arange(grid.N)
    ref, _, _ = _torch_block(bw, X, pos, None)
    zeros = np.zeros((grid.N, 256))

    def run():
        return O.dit_block_active(bw, X, idx, pos, zeros, zeros)[0]

    original_rope = O.rope_3d
    mutants = {
        "rope_3d": lambda x, p: original_rope(x, -np.asarray(p)),                 # sign of the angle
        "rms_norm": lambda x, g, eps=1e-6: np.asarray(x) * np.asarray(g),          # dropped normalisation
        "gelu_tanh": lambda x: 0.5 * np.asarray(x) * (1 + np.tanh(np.asarray(x))),  # dropped term
        "linear": lambda x, w, b: np.asarray(x) @ np.asarray(w)[:, :np.asarray(x).shape[1]].T,  # no bias
    }
    for name, fn in mutants.items():
        monkeypatch.setattr(O, name, fn)
        try:
            bad = run()
        except Exception:
            bad = None
        monkeypatch.setattr(O, name, _ORIGINALS[name])
        assert bad is None or not np.allclose(bad, ref, atol=1e-8), name

    # schedule with 1-based iterations fails the hand table
    monkeypatch.setattr(O, "active_table", lambda T, b, m: np.roll(_ORIGINALS["active_table"](T, b, m), 1, 0))
    with pytest.raises(AssertionError):
        test_schedule_tiny_matches_hand_table()
    monkeypatch.setattr(O, "active_table", _ORIGINALS["active_table"])

    # score without the absolute value fails the worked example
    monkeypatch.setattr(O, "l1_relative_change",
                        lambda a, b, eps=1e-8: (np.asarray(a) - np.asarray(b)).sum(1) / (np.abs(b).sum(1) + eps))
    with pytest.raises(AssertionError):
        test_score_hand_example()
    monkeypatch.setattr(O, "l1_relative_change", _ORIGINALS["l1_relative_change"])

    # ties broken by descending index fail the worked selection
    def bad_select(score, sizes):
        key = O.score_order_key(score)
        ranked = np.lexsort((-np.arange(len(key)), -key))
        group = np.empty(len(key), np.int8)
        start = 0
        for k, n in enumerate(sizes):
            group[ranked[start:start + n]] = k
            start += n
        order = np.concatenate([np.sort(np.nonzero(group == k)[0]) for k in range(len(sizes))])
        return group, order
    monkeypatch.setattr(O, "select_groups", bad_select)
    with pytest.raises(AssertionError):
        test_selection_hand_example()
    monkeypatch.setattr(O, "select_groups", _ORIGINALS["select_groups"])

    # pinned tokens given the NaN key (+inf) instead of a key above it, or ranked by score among
    # themselves, fail the worked pinned selection
    original_key = O.score_order_key

    def pinned_as_inf(score, sizes, pinned=None):
        s = np.array(score, np.float32)
        if pinned is not None:
            s[np.asarray(pinned, bool)] = np.inf
        return _ORIGINALS["select_groups"](s, sizes)

    def pinned_by_score(score, sizes, pinned=None):
        key = original_key(score)
        if pinned is not None:
            key = key + np.where(np.asarray(pinned, bool), 1 << 32, 0)
        ranked = np.lexsort((np.arange(len(key)), -key))
        group = np.empty(len(key), np.int8)
        start = 0
        for k, n in enumerate(sizes):
            group[ranked[start:start + n]] = k
            start += n
        order = np.concatenate([np.sort(np.nonzero(group == k)[0]) for k in range(len(sizes))])
        return group, order
    for bad in (pinned_as_inf, pinned_by_score):
        monkeypatch.setattr(O, "select_groups", bad)
        with pytest.raises(AssertionError):
            test_selection_pinned_hand_example()
    monkeypatch.setattr(O, "select_groups", _ORIGINALS["select_groups"])

    # a velocity head without its (shift, scale) modulation fails the patch-model composition
    original_head = O.head_projection
    monkeypatch.setattr(O, "head_projection",
                        lambda pm, X: O.linear(O.layer_norm(X), pm.w_out, pm.b_out))
    with pytest.raises(AssertionError):
        test_patch_model_all_active_equals_torch_composition()
    monkeypatch.setattr(O, "head_projection", original_head)


_ORIGINALS = {n: getattr(O, n) for n in ("rope_3d", "rms_norm", "gelu_tanh", "linear", "active_table",
                                         "l1_relative_change", "select_groups")}

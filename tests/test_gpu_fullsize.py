"""Full-size parity at the workloads' own shapes, in the launch configuration bench.py times.

The oracle cannot run a whole Wan-shaped step in seconds, so these tests
compare sampled outputs it computes one by one: the fresh K/V rows of sampled
active tokens, and the block output of sampled query rows (attention over the
whole cache the oracle builds itself from the same inputs).  Properties that
hold at any size (skipped cache rows untouched) are checked on every row.
"""
import numpy as np
import pytest
import torch

from oracle import hsa_oracle as O
from token_sparse_denoising_b200 import hsa
from token_sparse_denoising_b200 import synthetic as S
from tests._util import assert_bf16_close, dev, host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLE_ROWS = 48


def _step(bw, grid, idx, x, kc0, vc0, ctx):
    N, D = x.shape
    w = hsa.LayerWeights(bw, "cuda", True)
    kc, vc = dev(kc0, torch.bfloat16), dev(vc0, torch.bfloat16)
    M = len(idx)
    xA = torch.empty((M, D), device="cuda")
    ws = torch.empty(hsa.layer_step_workspace_size(M, D, bw.w_1.shape[0], hsa.HSA_BF16), dtype=torch.uint8,
                     device="cuda")
    ck = cv = None
    if ctx is not None:
        ck = torch.empty((ctx.shape[0], D), dtype=torch.bfloat16, device="cuda")
        cv = torch.empty_like(ck)
        cws = torch.empty(hsa.context_kv_workspace_size(ctx.shape[0], D), dtype=torch.uint8, device="cuda")
        hsa.context_kv(dev(ctx, torch.bfloat16), w.t["w_kv2"], w.t["b_kv2"], w.t["g_k2"], ck, cv, cws)
    hsa.layer_step(w, kc, vc, xA, dev(idx), dev(S.token_positions(grid)), ws, x_src=dev(x), ctx_k=ck, ctx_v=cv)
    assert hsa.device_status() == 0
    return xA, kc, vc


def _oracle_cache(bw, x, idx, pos, kc0, vc0, chunk=4096):
    """The oracle's cache after the step: stale rows from the inputs, fresh rows projected from
    every active token (in chunks of rows, to bound the host memory of the fp64 projection)."""
    Kw, Vw = kc0.astype(np.float64), vc0.astype(np.float64)
    for s in range(0, len(idx), chunk):
        rows = idx[s:s + chunk]
        _, k, v = O.qkv_projection(bw, x[rows], pos[rows])
        Kw[rows], Vw[rows] = k, v
    return Kw, Vw


def _check(bw, grid, idx, x, kc0, vc0, ctx):
    N, D = x.shape
    pos = S.token_positions(grid)
    xA, kc, vc = _step(bw, grid, idx, x, kc0, vc0, ctx)
    M = len(idx)
    kc_h, vc_h = host(kc), host(vc)
    del kc, vc
    skipped = np.setdiff1d(np.arange(N), idx)
    assert np.array_equal(kc_h[skipped], kc0[skipped]) and np.array_equal(vc_h[skipped], vc0[skipped])
    r = np.random.default_rng(M)
    sample = np.sort(r.choice(M, size=min(SAMPLE_ROWS, M), replace=False))
    Kw, Vw = _oracle_cache(bw, x, idx, pos, kc0, vc0)
    assert_bf16_close(kc_h[idx[sample]], Kw[idx[sample]], "fresh K rows")
    assert_bf16_close(vc_h[idx[sample]], Vw[idx[sample]], "fresh V rows")
    q, _, _ = O.qkv_projection(bw, x[idx[sample]], pos[idx[sample]])
    ctx_kv = O.context_kv(bw, ctx) if ctx is not None else None
    want = O.block_tail(bw, x[idx[sample]], O.attention(q, Kw, Vw), ctx_kv)
    got = host(xA)[sample]
    assert_bf16_close(got - x[idx[sample]], want - x[idx[sample]], "sampled block output delta")
    assert_bf16_close(got, want, "sampled block output")


@pytest.mark.parametrize("frac", [1.0, 0.5, 0.25])
def test_wan13_block_fullsize(cuda_lib, frac):
    """Wan-1.3B block: N=32760 (21x30x52), D=1536, 12 heads, FFN 8960, 512-token context."""
    grid, shape = S.WAN13_GRID, S.WAN13_BLOCK
    N, D = grid.N, shape.D
    bw = S.block_weights(2, shape, True)
    x = S.normal(21, (N, D))
    kc0, vc0 = S.normal(24, (N, D), 1.0, True), S.normal(25, (N, D), 1.0, True)
    ctx = S.normal(23, (shape.ctx_len, D), 1.0, True)
    M = S.active_fraction_rows(N, frac)
    score = O.l1_relative_change(S.normal(26, (N, D)), S.normal(27, (N, D))).astype(np.float32)
    _, order = O.select_groups(score, [M, N - M])
    idx = order[:M]
    _check(bw, grid, idx, x, kc0, vc0, ctx)


@pytest.mark.parametrize("frac,pattern", [(0.125, "contiguous"), (0.125, "scattered"), (0.25, "contiguous"),
                                          (0.5, "scattered"), (1.0, "scattered")])
def test_wan14_block_fullsize(cuda_lib, frac, pattern):
    """Wan-14B block: N=32760, D=5120, 40 heads, FFN 13824, no context; contiguous and scattered masks.
    At every active fraction the sampled rows' block output is compared with the oracle's, whose
    attention runs over its own cache: every active token's fresh K/V projected by the oracle."""
    grid, shape = S.WAN13_GRID, S.WAN14_BLOCK
    N, D = grid.N, shape.D
    bw = S.block_weights(4, shape, True)
    x = S.normal(41, (N, D))
    kc0, vc0 = S.normal(44, (N, D), 1.0, True), S.normal(45, (N, D), 1.0, True)
    M = S.active_fraction_rows(N, frac)
    idx = (S.contiguous_mask if pattern == "contiguous" else S.scattered_mask)(46, N, M)
    _check(bw, grid, idx, x, kc0, vc0, None)


@pytest.mark.parametrize("N", [8190, 32760, 75600])
@pytest.mark.parametrize("frac", [1.0, 0.125])
def test_attention_sweep_sizes(cuda_lib, N, frac):
    """Attention kernel sweep: bf16 Q/K/V N(0,1), 12 heads, random active query rows."""
    H, D = 12, 1536
    M = S.active_fraction_rows(N, frac)
    q = S.normal(51, (M, D), 1.0, True)
    k, v = S.normal(52, (N, D), 1.0, True), S.normal(53, (N, D), 1.0, True)
    o = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    hsa.attention(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), H, o)
    assert hsa.device_status() == 0
    rows = np.sort(np.random.default_rng(N).choice(M, size=32, replace=False))
    assert_bf16_close(host(o)[rows], O.attention(q[rows], k, v), "sampled attention rows")


@pytest.mark.parametrize("N", [8190, 32760, 75600])
def test_euler_sweep_sizes(cuda_lib, N):
    """Euler update on N x 16 x (2x2) = N x 64 fp32 latents with fp32 sigma deltas."""
    C = 64
    x0, vh0 = S.normal(61, (N, C)), S.normal(62, (N, C))
    M = N // 4
    idx = S.scattered_mask(63, N, M)
    vA = S.normal(64, (M, C))
    sig = O.sigma_schedule(40, 1, 5.0)
    dsig = float(np.float32(sig[11]) - np.float32(sig[10]))
    x, vh = dev(x0), dev(vh0)
    hsa.euler_update(x, vh, dev(vA), dev(idx), dsig)
    want_x, want_vh = O.cached_euler(x0, vh0, vA, idx, dsig)
    assert np.array_equal(host(vh), want_vh.astype(np.float32))
    assert np.linalg.norm(host(x) - want_x) / np.linalg.norm(want_x) < 1e-6

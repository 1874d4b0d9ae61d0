"""Parity of the whole HSA layer step and of whole denoising loops with the oracle."""
import numpy as np
import pytest
import torch

from oracle import hsa_oracle as O
from token_sparse_denoising_b200 import hsa, pipeline
from token_sparse_denoising_b200 import synthetic as S
from tests._util import assert_bf16_close, assert_f32_close, dev, host, rel_l2

pytestmark = pytest.mark.gpu


def _block(seed, D, F, cross, bf16, std=0.05, ctx_len=16):
    shape = S.BlockShape(D, D // 128, F, cross, ctx_len)
    bw = S.perturb_vectors(S.block_weights(seed, shape, bf16, std), seed + 1000)
    return shape, bw


def _run_layer_step(bw, bf16, grid, idx, x, Kc0, Vc0, ctx):
    N, D = x.shape
    dt = torch.bfloat16 if bf16 else torch.float32
    w = hsa.LayerWeights(bw, "cuda", bf16)
    kc, vc = dev(Kc0, dt), dev(Vc0, dt)
    xA = torch.empty((len(idx), D), device="cuda")
    ws = torch.empty(hsa.layer_step_workspace_size(len(idx), D, bw.w_1.shape[0], w.dtype), dtype=torch.uint8,
                     device="cuda")
    ck = cv = None
    if ctx is not None:
        ck = torch.empty((ctx.shape[0], D), dtype=dt, device="cuda")
        cv = torch.empty_like(ck)
        cws = torch.empty(hsa.context_kv_workspace_size(ctx.shape[0], D), dtype=torch.uint8, device="cuda")
        hsa.context_kv(dev(ctx, dt), w.t["w_kv2"], w.t["b_kv2"], w.t["g_k2"], ck, cv, cws)
    hsa.layer_step(w, kc, vc, xA, dev(idx), dev(S.token_positions(grid)), ws, x_src=dev(x), ctx_k=ck, ctx_v=cv)
    assert hsa.device_status() == 0
    return host(xA), host(kc), host(vc), (None if ck is None else (host(ck), host(cv)))


@pytest.mark.parametrize("cross", [False, True])
@pytest.mark.parametrize("frac", [1.0, 0.5, 0.123])
def test_layer_step_bf16_small(cuda_lib, cross, frac):
    grid = S.Grid(3, 10, 10)                       # N = 300: two full 128-key tiles and a ragged one
    N = grid.N
    shape, bw = _block(7, 256, 512, cross, True)
    M = max(1, int(round(frac * N)))
    idx = S.scattered_mask(8, N, M)
    x = S.normal(9, (N, 256))
    Kc0, Vc0 = S.normal(10, (N, 256), 1.0, True), S.normal(11, (N, 256), 1.0, True)
    ctx = S.normal(12, (16, 256), 1.0, True) if cross else None
    xA, kc, vc, ckv = _run_layer_step(bw, True, grid, idx, x, Kc0, Vc0, ctx)
    ctx_kv = O.context_kv(bw, ctx) if cross else None
    if cross:
        assert_bf16_close(ckv[0], ctx_kv[0], "context K")
        assert_bf16_close(ckv[1], ctx_kv[1], "context V")
    want, Kw, Vw = O.dit_block_active(bw, x[idx], idx, S.token_positions(grid), Kc0, Vc0, ctx_kv)
    assert_bf16_close(xA - x[idx], want - x[idx], "block output delta")
    assert_bf16_close(xA, want, "block output")
    assert_bf16_close(kc[idx], Kw[idx], "fresh K rows")
    assert_bf16_close(vc[idx], Vw[idx], "fresh V rows")
    skipped = np.setdiff1d(np.arange(N), idx)
    assert np.array_equal(kc[skipped], Kc0[skipped]) and np.array_equal(vc[skipped], Vc0[skipped])


def test_layer_step_f32_tiny_shape(cuda_lib):
    wl = S.TINY_FP32
    grid = wl.grid
    N = grid.N
    shape, bw = _block(13, 256, 1024, False, False)
    idx = S.scattered_mask(14, N, N // 2)
    x = S.normal(15, (N, 256))
    Kc0, Vc0 = S.normal(16, (N, 256)), S.normal(17, (N, 256))
    xA, kc, vc, _ = _run_layer_step(bw, False, grid, idx, x, Kc0, Vc0, None)
    want, Kw, Vw = O.dit_block_active(bw, x[idx], idx, S.token_positions(grid), Kc0, Vc0)
    assert_f32_close(xA - x[idx], want - x[idx], "block output delta")
    assert_f32_close(kc, Kw, "K cache")
    assert_f32_close(vc, Vw, "V cache")


def test_tiny_fp32_loop_matches_oracle(cuda_lib):
    """The tiny single-layer fp32 loop (4x16x16 tokens, T=8, budgets {8,4}, m=1) end to end."""
    wl = S.TINY_FP32
    N, D = wl.grid.N, wl.shape.D
    bw = S.block_weights(wl.seed, wl.shape, False)
    pos = S.token_positions(wl.grid)
    x0, vh0 = S.normal(wl.seed * 10 + 1, (N, D)), S.normal(wl.seed * 10 + 2, (N, D))
    sizes = S.group_sizes(N, wl.fracs)
    model = pipeline.SingleBlockModel(bw, pos, N, bf16=False)
    run = pipeline.HSARun(model, x0, vh0, wl.T, wl.budgets, sizes, wl.m, wl.sigma_kind, wl.shift)
    rec = []
    x_gpu = host(run.run(rec))
    assert hsa.device_status() == 0

    plan = O.make_plan(wl.T, wl.budgets, sizes, wl.m, wl.sigma_kind, wl.shift, N)

    def vel(xA, idx, caches):
        out, Kc, Vc = O.dit_block_active(bw, xA, idx, pos, caches[0], caches[1])
        return out, (Kc, Vc)

    zeros = np.zeros((N, D))
    final, states = O.hsa_denoise(x0, vh0, plan, vel, (zeros, zeros), keep_states=True)
    for r, st in zip(rec, states):
        assert r["M"] == len(st["idx"])
        if r["full"]:
            assert rel_l2(r["score"], st["score"]) < 1e-4
            assert np.array_equal(r["order"], st["order"])
    assert_f32_close(x_gpu, final["x"], "final latent")
    assert_f32_close(x_gpu - x0, final["x"] - x0, "latent displacement")

"""Head parallelism through the CUDA kernels: G ranks' parts of one bf16 block, emulated in one
process on one GPU (EmulatedGroup serves the collectives with device copies and sums), against
the oracle's unsplit block.  The same phases run between real NCCL ranks through
run_collectives; its bookkeeping and algebra are pinned on the CPU (tests/test_sharded.py)."""
import numpy as np
import pytest
import torch

from oracle import hsa_oracle as O
from token_sparse_denoising_b200 import hsa
from token_sparse_denoising_b200 import synthetic as S
from token_sparse_denoising_b200.sharded import EmulatedGroup, HeadParallelBlock, HeadShard, gather_block_output
from tests._util import assert_bf16_close, dev, host

pytestmark = pytest.mark.gpu


def _run(bw, G, grid, idx, x, kc0, vc0, ctx):
    N, D = x.shape
    H, F, M = D // 128, bw.w_1.shape[0], len(idx)
    blocks = [HeadParallelBlock(bw, HeadShard(g, G, H, F, M), N, "cuda", cache_init=(kc0, vc0)) for g in range(G)]
    if ctx is not None:
        EmulatedGroup.run(b.context_kv(ctx) for b in blocks)
    x_d, idx_d, pos_d = dev(x), dev(idx), dev(S.token_positions(grid))
    EmulatedGroup.run(b.step(x_d, idx_d, pos_d) for b in blocks)
    assert hsa.device_status() == 0
    out = host(gather_block_output(blocks))
    kc = np.concatenate([host(b.kc) for b in blocks], axis=1)
    vc = np.concatenate([host(b.vc) for b in blocks], axis=1)
    return out, kc, vc


@pytest.mark.parametrize("G", [2, 4])
@pytest.mark.parametrize("cross,frac", [(False, 0.5), (True, 0.37), (True, 1.0)])
def test_head_parallel_block_matches_oracle(cuda_lib, G, cross, frac):
    grid = S.Grid(3, 10, 10)                       # N = 300 keys: two full 128-key tiles and a ragged one
    N, D, F = grid.N, 512, 1024                    # 4 heads
    shape = S.BlockShape(D, 4, F, cross, 16)
    bw = S.perturb_vectors(S.block_weights(41, shape, True, 0.05), 42)
    M = max(1, int(round(frac * N)))
    idx = S.scattered_mask(43, N, M)
    x = S.normal(44, (N, D))
    kc0, vc0 = S.normal(45, (N, D), 1.0, True), S.normal(46, (N, D), 1.0, True)
    ctx = S.normal(47, (16, D), 1.0, True) if cross else None
    out, kc, vc = _run(bw, G, grid, idx, x, kc0, vc0, ctx)
    want, Kw, Vw = O.dit_block_active(bw, x[idx], idx, S.token_positions(grid), kc0, vc0,
                                      O.context_kv(bw, ctx) if cross else None)
    assert_bf16_close(out - x[idx], want - x[idx], "block output delta")
    assert_bf16_close(out, want, "block output")
    assert_bf16_close(kc[idx], Kw[idx], "fresh K rows")
    assert_bf16_close(vc[idx], Vw[idx], "fresh V rows")
    skipped = np.setdiff1d(np.arange(N), idx)
    assert np.array_equal(kc[skipped], kc0[skipped]) and np.array_equal(vc[skipped], vc0[skipped])


def test_head_parallel_matches_the_unsplit_layer_step(cuda_lib):
    """Two ranks against one hsa_layer_step on the same inputs: the same arithmetic split two
    ways, so the outputs agree to bf16 rounding of the operands they exchange."""
    grid = S.Grid(2, 8, 8)
    N, D, F = grid.N, 512, 1024
    shape = S.BlockShape(D, 4, F, True, 16)
    bw = S.perturb_vectors(S.block_weights(51, shape, True, 0.05), 52)
    idx = S.scattered_mask(53, N, 77)
    x = S.normal(54, (N, D))
    kc0, vc0 = S.normal(55, (N, D), 1.0, True), S.normal(56, (N, D), 1.0, True)
    ctx = S.normal(57, (16, D), 1.0, True)
    out, kc, _ = _run(bw, 2, grid, idx, x, kc0, vc0, ctx)
    w = hsa.LayerWeights(bw, "cuda", True)
    kcu, vcu = dev(kc0, torch.bfloat16), dev(vc0, torch.bfloat16)
    xA = torch.empty((77, D), device="cuda")
    ws = torch.empty(hsa.layer_step_workspace_size(77, D, F, hsa.HSA_BF16), dtype=torch.uint8, device="cuda")
    ck = torch.empty((16, D), dtype=torch.bfloat16, device="cuda")
    cv = torch.empty_like(ck)
    cws = torch.empty(hsa.context_kv_workspace_size(16, D), dtype=torch.uint8, device="cuda")
    hsa.context_kv(dev(ctx, torch.bfloat16), w.t["w_kv2"], w.t["b_kv2"], w.t["g_k2"], ck, cv, cws)
    hsa.layer_step(w, kcu, vcu, xA, dev(idx), dev(S.token_positions(grid)), ws, x_src=dev(x), ctx_k=ck, ctx_v=cv)
    assert hsa.device_status() == 0
    assert_bf16_close(out - x[idx], host(xA) - x[idx], "split vs unsplit block output delta")
    assert_bf16_close(kc[idx], host(kcu)[idx], "split vs unsplit fresh K rows")

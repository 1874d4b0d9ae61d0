"""A whole HSA loop recorded as one CUDA graph runs the same kernels on the same buffers as the
eager loop, so its final latent must match the eager one bit for bit; a second replay after
reset() must match again (the recording reads the active index lists from device buffers that
the selection kernel rewrites, so the partitions chosen during the replay are the replay's own)."""
import numpy as np
import pytest

from token_sparse_denoising_b200 import pipeline, synthetic as S

pytestmark = pytest.mark.gpu


def _host(t):
    return t.detach().float().cpu().numpy()


def test_loop_graph_replay_is_bitwise_identical_to_eager(cuda_lib):
    hsa = cuda_lib
    wl = S.WAN13_LOOP_SMALL
    N, C = wl.grid.N, wl.C
    pm = S.patch_model_weights(wl.seed, wl.shape, C, wl.n_blocks, True, std=0.05)
    pos = S.token_positions(wl.grid)
    x0, vh0 = S.normal(wl.seed * 10 + 1, (N, C)), S.normal(wl.seed * 10 + 2, (N, C))
    ctx = S.normal(wl.seed * 10 + 3, (wl.shape.ctx_len, wl.shape.D), 1.0, True)
    sizes = S.group_sizes(N, wl.fracs)
    model = pipeline.PatchModel(pm, pos, N, bf16=True, ctx=ctx)
    run = pipeline.HSARun(model, x0, vh0, wl.T, wl.budgets, sizes, wl.m, wl.sigma_kind, wl.shift)
    x_eager = _host(run.run()).copy()
    order_eager = run.order.cpu().numpy().copy()
    assert hsa.device_status() == 0

    launches0 = hsa.launch_count()
    run.reset(x0, vh0)
    g = run.capture()
    recorded = hsa.launch_count() - launches0
    assert recorded > wl.T * wl.n_blocks             # every step's launches went into the graph
    run.replay(g)
    x_graph = _host(run.x).copy()
    assert hsa.device_status() == 0
    assert np.array_equal(x_graph, x_eager)
    assert np.array_equal(run.order.cpu().numpy(), order_eager)

    run.reset(x0, vh0)
    run.replay(g)
    assert hsa.device_status() == 0
    assert np.array_equal(_host(run.x), x_eager)
    assert not np.array_equal(x_eager, x0)            # the loop did move the latent


def test_loop_graph_with_non_nested_budgets(cuda_lib):
    """T = 12 with budgets {12, 6, 4} (periods 1, 2, 3): at i = 3 groups 1 and 3 are active
    without group 2, so that step's active set is not a prefix of the order and is gathered
    with device copies, which the graph records as well."""
    hsa = cuda_lib
    grid = S.Grid(1, 4, 8)
    shape = S.WAN13_LOOP_SMALL.shape
    N, C = grid.N, 64
    pm = S.patch_model_weights(7, shape, C, 2, True, std=0.05)
    pos = S.token_positions(grid)
    x0, vh0 = S.normal(71, (N, C)), S.normal(72, (N, C))
    sizes = S.group_sizes(N, (0.25, 0.25, 0.5))
    ctx = S.normal(73, (shape.ctx_len, shape.D), 1.0, True)
    model = pipeline.PatchModel(pm, pos, N, bf16=True, ctx=ctx)
    run = pipeline.HSARun(model, x0, vh0, 12, (12, 6, 4), sizes, 1, 0, 1.0)
    x_eager = _host(run.run()).copy()
    assert hsa.device_status() == 0
    run.reset(x0, vh0)
    g = run.capture()
    run.replay(g)
    assert hsa.device_status() == 0
    assert np.array_equal(_host(run.x), x_eager)

"""hsa_iteration_host: one HSA iteration with the latent in host memory.  The upload, the same
device calls as the device-pointer path (layer step on A_i, cached Euler with the fused score,
regrouping after a full step) and the download run on three streams ordered by events, with two
slots alternating.  The host results must equal the device-pointer path's latent bit for bit at
every iteration, and the method state (v_hat, KV caches, scores, partition) must match too."""
import numpy as np
import pytest
import torch

from token_sparse_denoising_b200 import pipeline, synthetic as S

pytestmark = pytest.mark.gpu


def _setup(hsa, seed, bf16=True):
    grid = S.Grid(2, 8, 10)
    N, D = grid.N, 256
    shape = S.BlockShape(D, 2, 512, True, 16)
    bw = S.perturb_vectors(S.block_weights(seed, shape, bf16, 0.05), seed + 1)
    pos = S.token_positions(grid)
    ctx = S.normal(seed + 4, (16, D), 1.0, bf16)
    kc0, vc0 = S.normal(seed + 5, (N, D), 1.0, bf16), S.normal(seed + 6, (N, D), 1.0, bf16)
    x0, vh0 = S.normal(seed + 2, (N, D)), S.normal(seed + 3, (N, D))
    model = pipeline.SingleBlockModel(bw, pos, N, bf16=bf16, ctx=ctx, cache_init=(kc0, vc0))
    st = dict(model=model, x=torch.from_numpy(x0).cuda(), vhat=torch.from_numpy(vh0).cuda(),
              score=torch.zeros(N, device="cuda"), group=torch.zeros(N, dtype=torch.int8, device="cuda"),
              order=torch.arange(N, dtype=torch.int32, device="cuda"))
    st["sel_ws"] = torch.empty(max(hsa.select_tokens_workspace_size(N, 2), 16), dtype=torch.uint8, device="cuda")
    return st, x0


@pytest.mark.parametrize("same_stream,bf16", [(False, True), (True, True), (False, False)])
def test_iteration_host_matches_device_path(cuda_lib, same_stream, bf16):
    """bf16 (tensor-core kernels) and fp32 (CUDA-core kernels) blocks, with separate copy streams
    and with everything on one stream."""
    hsa = cuda_lib
    dev, x0 = _setup(hsa, 40, bf16)
    hst, _ = _setup(hsa, 40, bf16)
    N, D = x0.shape
    sizes = [N // 2, N - N // 2]
    # steps: full (regroup), the first group only, full, the first group only
    plan = [N, N // 2, N, N // 2]
    dsig = [-0.25, -0.25, -0.25, -0.25]
    h_in = torch.from_numpy(x0.copy()).pin_memory()
    h_out = [torch.empty_like(h_in).pin_memory() for _ in range(2)]
    slots = [hsa.HostSlot(N, D), hsa.HostSlot(N, D)]
    comp = torch.cuda.current_stream()
    up = comp if same_stream else torch.cuda.Stream()
    down = comp if same_stream else torch.cuda.Stream()
    torch.cuda.synchronize()
    for k, (M, ds) in enumerate(zip(plan, dsig)):
        # device-pointer path
        idx = dev["order"][:M].clone() if M < N else dev["order"]
        vA = dev["model"].velocity(dev["x"], idx)
        full = M == N
        hsa.euler_update(dev["x"], dev["vhat"], vA, idx, ds, score=dev["score"] if full else None)
        if full:
            hsa.select_tokens(dev["score"], sizes, dev["group"], dev["order"], ws=dev["sel_ws"])
        # host path: the latent comes from the previous iteration's download
        m = hst["model"]
        hidx = hst["order"][:M].clone() if M < N else hst["order"]
        src = h_in if k == 0 else h_out[(k - 1) % 2]
        if k > 0:
            down.synchronize()                 # the previous download has landed in host memory
        hsa.iteration_host(m.w, m.kc, m.vc, hidx, m.pos, m.xA[:M], hst["vhat"], ds, src, h_out[k % 2], slots[k % 2],
                           m.ws, ctx_k=m.ctx_k, ctx_v=m.ctx_v, score=hst["score"], group_sizes=sizes,
                           group=hst["group"] if full else None, order=hst["order"], sel_ws=hst["sel_ws"],
                           stream=comp, stream_h2d=up, stream_d2h=down)
        torch.cuda.synchronize()
        assert hsa.device_status() == 0
        got = h_out[k % 2].numpy()
        want = dev["x"].cpu().numpy()
        assert np.array_equal(got, want), f"iteration {k}: host-path latent differs"
        assert torch.equal(hst["vhat"], dev["vhat"])
        assert torch.equal(m.kc, dev["model"].kc) and torch.equal(m.vc, dev["model"].vc)
        assert torch.equal(hst["order"], dev["order"]) and torch.equal(hst["group"], dev["group"])
        if full:
            assert torch.equal(hst["score"], dev["score"])
    assert not np.array_equal(h_out[1].numpy(), x0)       # the latent moved

"""hsa_context_kv_noalloc: the context key/value projection for callers that cannot
allocate device memory (a runtime with a device memory budget fixed at start-up, or
a path where an allocation would synchronise the device).  Its scratch is an array
built into the library, so the test checks that it gives the same keys/values as the
workspace entry point, hsa_context_kv, on two calls in a row (the second call finds
the first call's leftovers in the shared scratch), and that oversize requests are
refused.  This file is collected last, so a run stopping at the first failure has
run every other test already."""
import numpy as np
import pytest
import torch

from token_sparse_denoising_b200 import hsa
from token_sparse_denoising_b200 import synthetic as S
from tests._util import assert_bf16_close, dev, host

pytestmark = pytest.mark.gpu


def _case(seed, L, D):
    shape = S.BlockShape(D, D // 128, 512, True, L)
    bw = S.perturb_vectors(S.block_weights(seed, shape, True, 0.05), seed + 1)
    ctx = S.normal(seed + 2, (L, D), 1.0, True)
    w = hsa.LayerWeights(bw, "cuda", True)
    return dev(ctx, torch.bfloat16), w


def _with_workspace(ctx, w):
    L, D = ctx.shape
    k = torch.empty((L, D), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    ws = torch.empty(hsa.context_kv_workspace_size(L, D), dtype=torch.uint8, device="cuda")
    hsa.context_kv(ctx, w.t["w_kv2"], w.t["b_kv2"], w.t["g_k2"], k, v, ws)
    return host(k), host(v)


def _without_workspace(ctx, w):
    L, D = ctx.shape
    k = torch.empty((L, D), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    hsa.context_kv_noalloc(ctx, w.t["w_kv2"], w.t["b_kv2"], w.t["g_k2"], k, v)
    return host(k), host(v)


def test_no_alloc_context_kv_matches_workspace_version(cuda_lib):
    # calls in a row with different inputs and sizes: each later call reuses the scratch; the
    # last one fills it exactly (bf16: 512 x 2 x 4096 x 2 bytes = 8 MiB)
    for seed, L, D in ((3, 512, 1536), (9, 77, 256), (11, 512, 4096)):
        ctx, w = _case(seed, L, D)
        k_ref, v_ref = _with_workspace(ctx, w)
        k, v = _without_workspace(ctx, w)
        assert hsa.device_status() == 0
        assert_bf16_close(k, k_ref, f"K (L={L}, D={D})")
        assert_bf16_close(v, v_ref, f"V (L={L}, D={D})")


def test_no_alloc_rejects_oversize(cuda_lib):
    assert hsa.lib().hsa_context_kv_noalloc_max_bytes() == 8 << 20
    ctx, w = _case(5, 8192, 512)            # bf16: 8192 x 1024 x 2 bytes = 16 MiB > 8 MiB
    k = torch.empty((8192, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hsa.HsaError) as e:
        hsa.context_kv_noalloc(ctx, w.t["w_kv2"], w.t["b_kv2"], w.t["g_k2"], k, torch.empty_like(k))
    assert e.value.code == hsa.HSA_EINVAL

"""Failure detection on the GPU without a fault: kernels never trap.  A token index outside
[0, N) is recorded in the device status word and its row is skipped; a pipelined wait that
runs out gives up after its bound, records HSA_ETIMEOUT and returns.  In both cases the host
reads the status with hsa_device_status(), which clears it, and the context stays usable."""
import numpy as np
import pytest
import torch

from token_sparse_denoising_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def test_out_of_range_token_index_is_flagged_and_skipped(cuda_lib):
    hsa = cuda_lib
    N, C, M = 64, 64, 6
    guard = 4                                                  # rows past N that no kernel may touch
    x0, vh0, vA = S.normal(91, (N + guard, C)), S.normal(92, (N + guard, C)), S.normal(93, (M, C))
    x = torch.from_numpy(x0).cuda()
    vh = torch.from_numpy(vh0).cuda()
    idx = torch.tensor([3, N, 10, -1, 20, N + 1], dtype=torch.int32, device="cuda")
    hsa.euler_update(x[:N], vh[:N], torch.from_numpy(vA).cuda(), idx, -0.25)
    assert hsa.device_status() == hsa.HSA_EINDEX
    assert hsa.device_status() == hsa.HSA_OK               # reading the status cleared it
    got_v, got_x = vh.cpu().numpy(), x.cpu().numpy()
    want_v = vh0.copy()
    for r, n in enumerate([3, N, 10, -1, 20, N + 1]):
        if 0 <= n < N:
            want_v[n] = vA[r]
    assert np.array_equal(got_v, want_v)                    # valid rows scattered, the bad ones skipped
    want_x = x0.copy()
    want_x[:N] = (x0[:N] + np.float32(-0.25) * want_v[:N]).astype(np.float32)
    assert np.allclose(got_x[:N], want_x[:N], rtol=0, atol=1e-6)
    assert np.array_equal(got_x[N:], x0[N:]) and np.array_equal(got_v[N:], vh0[N:])


def test_bounded_wait_gives_up_and_context_stays_usable(cuda_lib):
    hsa = cuda_lib
    hsa.selftest_wait_timeout()
    assert hsa.device_status() == hsa.HSA_ETIMEOUT
    assert hsa.device_status() == hsa.HSA_OK
    # the abort flag was cleared with the status: a pipelined kernel runs normally again
    q = torch.randn((256, 256), device="cuda").to(torch.bfloat16)
    k = torch.randn((300, 256), device="cuda").to(torch.bfloat16)
    v = torch.randn((300, 256), device="cuda").to(torch.bfloat16)
    o = torch.empty_like(q)
    hsa.attention(q, k, v, 2, o)
    assert hsa.device_status() == hsa.HSA_OK
    ref = torch.softmax(q.float().view(256, 2, 128).transpose(0, 1) @ k.float().view(300, 2, 128).permute(1, 2, 0)
                        / 128 ** 0.5, -1) @ v.float().view(300, 2, 128).transpose(0, 1)
    got = o.float().view(256, 2, 128).transpose(0, 1)
    assert float((got - ref).norm() / ref.norm()) < 2e-2

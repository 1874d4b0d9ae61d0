"""Helpers shared by the parity tests (comparison metrics and host<->device moves)."""
import numpy as np

# Tolerances: float32 paths 1e-4 relative L2; bf16 paths 2e-2 relative L2 and
# 5e-2 max-abs on unit-scale data.
TOL_F32 = 1e-4
TOL_BF16_REL = 2e-2
TOL_BF16_ABS = 5e-2


def rel_l2(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def max_abs(got, want) -> float:
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64)))) if np.size(want) else 0.0


def dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def assert_bf16_close(got, want, what=""):
    r, a = rel_l2(got, want), max_abs(got, want)
    assert r <= TOL_BF16_REL and a <= TOL_BF16_ABS, f"{what}: rel_l2 {r:.3e} max_abs {a:.3e}"


def assert_f32_close(got, want, what=""):
    r = rel_l2(got, want)
    assert r <= TOL_F32, f"{what}: rel_l2 {r:.3e}"

"""ctypes binding of libhsa.so (include/hsa.h): argument marshalling only.

Every function takes torch tensors already on the device (or plain numbers)
and passes their pointers, sizes and the current CUDA stream to the C ABI.
There is no fallback: if libhsa.so cannot be loaded, `load()` raises.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhsa.so")

HSA_OK, HSA_EINVAL, HSA_EINDEX, HSA_ECUDA, HSA_ETIMEOUT, HSA_EWORKSPACE = range(6)
HSA_F32, HSA_BF16 = 0, 1
EPI_STORE, EPI_GELU, EPI_RESID, EPI_F32 = range(4)

_lib = None
vp, i32, u64, f32, sz = C.c_void_p, C.c_int, C.c_uint64, C.c_float, C.c_size_t


class HsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: status {code}: {_lib.hsa_last_error_string().decode()}")
        self.code = code


class LayerWeightsC(C.Structure):
    _fields_ = [("D", i32), ("H", i32), ("F", i32), ("dtype", i32),
                ("w_qkv", vp), ("b_qkv", vp), ("g_q", vp), ("g_k", vp),
                ("w_o", vp), ("b_o", vp), ("w_1", vp), ("b_1", vp), ("w_2", vp), ("b_2", vp),
                ("mod", vp), ("ln_c_g", vp), ("ln_c_b", vp), ("w_q2", vp), ("b_q2", vp), ("g_q2", vp),
                ("w_o2", vp), ("b_o2", vp)]


class IterationArgsC(C.Structure):
    _fields_ = [("w", C.POINTER(LayerWeightsC)), ("d_kcache", vp), ("d_vcache", vp), ("N", i32), ("d_idx", vp),
                ("M", i32), ("d_pos", vp), ("d_ctx_k", vp), ("d_ctx_v", vp), ("ctx_len", i32), ("d_xA", vp),
                ("d_vhat", vp), ("dsigma", f32), ("d_score", vp), ("K", i32), ("h_group_sizes", vp),
                ("d_group", vp), ("d_order", vp), ("d_ws", vp), ("ws_bytes", sz), ("d_sel_ws", vp),
                ("sel_ws_bytes", sz)]


class HostSlotC(C.Structure):
    _fields_ = [("d_x", vp), ("ev_in", vp), ("ev_done", vp), ("ev_free", vp)]


_SIGS = {
    "hsa_last_error_string": (C.c_char_p, []),
    "hsa_device_status": (i32, [vp]),
    "hsa_selftest_wait_timeout": (i32, [vp]),
    "hsa_launch_count": (u64, []),
    "hsa_timing_enable": (i32, [i32]),
    "hsa_timing_read": (i32, [i32, C.POINTER(C.c_double), C.POINTER(i32)]),
    "hsa_timing_reset": (i32, []),
    "hsa_plan_groups": (i32, [i32, i32, vp, vp, i32, i32, i32, f32, vp, vp, vp]),
    "hsa_l1_score": (i32, [vp, vp, i32, i32, vp, vp]),
    "hsa_select_tokens_workspace_size": (sz, [i32, i32]),
    "hsa_select_tokens": (i32, [vp, i32, i32, vp, vp, vp, vp, sz, vp]),
    "hsa_select_tokens_pinned": (i32, [vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]),
    "hsa_active_rows": (i32, [vp, i32, i32, vp, vp, vp, C.POINTER(i32), vp]),
    "hsa_euler_update": (i32, [vp, vp, vp, vp, i32, i32, i32, f32, vp, vp]),
    "hsa_context_kv_workspace_size": (sz, [i32, i32]),
    "hsa_context_kv": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
    "hsa_context_kv_noalloc_max_bytes": (sz, []),
    "hsa_context_kv_noalloc": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
    "hsa_layer_step_workspace_size": (sz, [i32, i32, i32, i32]),
    "hsa_layer_step": (i32, [C.POINTER(LayerWeightsC), vp, vp, i32, vp, vp, vp, i32, vp, vp, vp, i32, vp, sz, vp]),
    "hsa_attention": (i32, [vp, i32, vp, vp, i32, i32, i32, vp, vp]),
    "hsa_attention_workspace_size": (sz, [i32, i32, i32, i32]),
    "hsa_attention_ws": (i32, [vp, i32, vp, vp, i32, i32, i32, vp, vp, sz, vp]),
    "hsa_linear": (i32, [vp, i32, i32, vp, i32, vp, i32, i32, vp, vp, vp]),
    "hsa_patch_workspace_size": (sz, [i32, i32, i32, i32]),
    "hsa_patch_embed": (i32, [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp]),
    "hsa_velocity_head": (i32, [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
    "hsa_layernorm_rows": (i32, [vp, vp, vp, i32, i32, i32, vp, vp, i32, i32, vp, vp]),
    "hsa_row_sumsq": (i32, [vp, i32, i32, i32, i32, vp, i32, vp]),
    "hsa_qk_norm_rope_ext": (i32, [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp]),
    "hsa_rms_rows_ext": (i32, [vp, i32, i32, i32, i32, vp, i32, vp, i32, vp, vp]),
    "hsa_gated_residual": (i32, [vp, vp, i32, i32, vp, vp, vp]),
    "hsa_iteration_host": (i32, [C.POINTER(IterationArgsC), vp, vp, C.POINTER(HostSlotC), vp, vp, vp]),
}


def load(path: str = LIB_PATH):
    """Load libhsa.so (building it first when the in-tree copy is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path) or os.environ.get("HSA_REBUILD"):
        from . import build
        build.build_library()
    if not os.path.exists(path):
        raise RuntimeError(f"libhsa.so not found at {path}; the CUDA path has no fallback")
    lib = C.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def lib():
    return load()


def _check(code: int, what: str):
    if code != HSA_OK:
        raise HsaError(code, what)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return HSA_BF16
    if t.dtype == torch.float32:
        return HSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t, name, dtype=None):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


# ---------------------------------------------------------------- host plan

def plan_groups(T: int, budgets, group_sizes, N: int, m: int, sigma_kind: int, shift: float):
    """Returns (sigmas float32[T+1], active table uint8[T,K], n_active int32[T])."""
    K = len(budgets)
    b = np.ascontiguousarray(budgets, np.int32)
    s = np.ascontiguousarray(group_sizes, np.int32)
    sig = np.zeros(T + 1, np.float32)
    tab = np.zeros((T, K), np.uint8)
    nact = np.zeros(T, np.int32)
    _check(lib().hsa_plan_groups(T, K, b.ctypes.data, s.ctypes.data, N, m, sigma_kind, shift,
                                 sig.ctypes.data, tab.ctypes.data, nact.ctypes.data), "hsa_plan_groups")
    return sig, tab, nact


# ---------------------------------------------------------------- device calls

def device_status(stream=None) -> int:
    return lib().hsa_device_status(_stream(stream))


def selftest_wait_timeout(stream=None) -> None:
    """Diagnostic: a kernel whose bounded wait runs out (see hsa_selftest_wait_timeout)."""
    _check(lib().hsa_selftest_wait_timeout(_stream(stream)), "hsa_selftest_wait_timeout")


def launch_count() -> int:
    return int(lib().hsa_launch_count())


KCLASS_ATTENTION, KCLASS_GEMM, KCLASS_OTHER = 0, 1, 2


def timing_enable(on: bool = True):
    _check(lib().hsa_timing_enable(1 if on else 0), "hsa_timing_enable")


def timing_read(kclass: int):
    """(summed device ms, launch count) of one kernel class since the last reset."""
    ms, n = C.c_double(0.0), i32(0)
    _check(lib().hsa_timing_read(kclass, C.byref(ms), C.byref(n)), "hsa_timing_read")
    return ms.value, n.value


def timing_reset():
    _check(lib().hsa_timing_reset(), "hsa_timing_reset")


def l1_score(v_new, v_prev, score, stream=None):
    N, Cc = v_new.shape
    _check(lib().hsa_l1_score(_ptr(v_new), _ptr(v_prev), N, Cc, _ptr(score), _stream(stream)), "hsa_l1_score")


def select_tokens_workspace_size(N: int, K: int) -> int:
    return int(lib().hsa_select_tokens_workspace_size(N, K))


def select_tokens(score, group_sizes, group, order, stream=None, ws=None, pinned=None):
    """Group partition by score; `pinned` (uint8 [N] on the device, optional) ranks those tokens
    ahead of all others (hsa_select_tokens_pinned)."""
    import torch
    N = score.shape[0]
    K = len(group_sizes)
    sizes = np.ascontiguousarray(group_sizes, np.int32)
    nbytes = lib().hsa_select_tokens_workspace_size(N, K)
    if ws is None:
        ws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=score.device)
    elif ws.numel() * ws.element_size() < nbytes:
        raise ValueError("select_tokens: workspace smaller than hsa_select_tokens_workspace_size")
    if pinned is None:
        _check(lib().hsa_select_tokens(_ptr(score), N, K, sizes.ctypes.data, _ptr(group), _ptr(order), _ptr(ws),
                                       nbytes, _stream(stream)), "hsa_select_tokens")
    else:
        if pinned.dtype != torch.uint8 or pinned.numel() != N:
            raise ValueError("select_tokens: pinned must be a uint8 tensor of N entries")
        _check(lib().hsa_select_tokens_pinned(_ptr(score), _ptr(pinned), N, K, sizes.ctypes.data, _ptr(group),
                                              _ptr(order), _ptr(ws), nbytes, _stream(stream)),
               "hsa_select_tokens_pinned")


def active_rows(order, group_sizes, active, idx, stream=None) -> int:
    """A_i: the active groups' lists of `order`, concatenated into `idx`; returns M."""
    N = order.shape[0]
    K = len(group_sizes)
    sizes = np.ascontiguousarray(group_sizes, np.int32)
    act = np.ascontiguousarray(np.asarray(active, bool).astype(np.uint8))
    m = C.c_int(0)
    _check(lib().hsa_active_rows(_ptr(order), N, K, sizes.ctypes.data, act.ctypes.data, _ptr(idx), C.byref(m),
                                 _stream(stream)), "hsa_active_rows")
    return int(m.value)


def euler_update(x, vhat, vA, idx, dsigma: float, score=None, stream=None):
    N, Cc = x.shape
    M = 0 if idx is None else idx.shape[0]
    _check(lib().hsa_euler_update(_ptr(x), _ptr(vhat), _ptr(vA), _ptr(idx), M, N, Cc, float(dsigma), _ptr(score),
                                  _stream(stream)), "hsa_euler_update")


def linear(x, w, b, epilogue: int, y, gate=None, stream=None):
    M, K = x.shape
    _check(lib().hsa_linear(_ptr(x), M, K, _ptr(w), w.shape[0], _ptr(b), _dtype_code(x), epilogue, _ptr(gate),
                            _ptr(y), _stream(stream)), "hsa_linear")


def attention(q, k, v, H: int, o, stream=None, ws=None):
    """o = softmax(q k^T / sqrt(128)) v per head; with `ws` (uint8 device tensor of at least
    attention_workspace_size bytes) the last wave's units are split over key ranges."""
    if ws is None:
        _check(lib().hsa_attention(_ptr(q), q.shape[0], _ptr(k), _ptr(v), k.shape[0], H, _dtype_code(q), _ptr(o),
                                   _stream(stream)), "hsa_attention")
    else:
        _check(lib().hsa_attention_ws(_ptr(q), q.shape[0], _ptr(k), _ptr(v), k.shape[0], H, _dtype_code(q),
                                      _ptr(o), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
               "hsa_attention_ws")


def attention_workspace_size(M: int, L: int, H: int, dtype: int) -> int:
    return int(lib().hsa_attention_workspace_size(M, L, H, dtype))


def context_kv_workspace_size(L: int, D: int) -> int:
    return int(lib().hsa_context_kv_workspace_size(L, D))


def context_kv(ctx, w_kv2, b_kv2, g_k2, k2, v2, ws, stream=None):
    L, D = ctx.shape
    _check(lib().hsa_context_kv(_ptr(ctx), L, D, _dtype_code(ctx), _ptr(w_kv2), _ptr(b_kv2), _ptr(g_k2), _ptr(k2),
                                _ptr(v2), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hsa_context_kv")


def context_kv_noalloc(ctx, w_kv2, b_kv2, g_k2, k2, v2, stream=None):
    """hsa_context_kv without a workspace: scratch comes from an array built into libhsa."""
    L, D = ctx.shape
    _check(lib().hsa_context_kv_noalloc(_ptr(ctx), L, D, _dtype_code(ctx), _ptr(w_kv2), _ptr(b_kv2), _ptr(g_k2),
                                        _ptr(k2), _ptr(v2), _stream(stream)), "hsa_context_kv_noalloc")


def layer_step_workspace_size(M: int, D: int, F: int, dtype: int) -> int:
    return int(lib().hsa_layer_step_workspace_size(M, D, F, dtype))


def layer_step(w: "LayerWeights", kcache, vcache, xA, idx, pos, ws, x_src=None, ctx_k=None, ctx_v=None,
               stream=None):
    N = kcache.shape[0]
    M = idx.shape[0]
    L = 0 if ctx_k is None else ctx_k.shape[0]
    _check(lib().hsa_layer_step(C.byref(w.c), _ptr(kcache), _ptr(vcache), N, _ptr(xA), _ptr(x_src), _ptr(idx), M,
                                _ptr(pos), _ptr(ctx_k), _ptr(ctx_v), L, _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "hsa_layer_step")


def patch_workspace_size(M: int, D: int, Cc: int, dtype: int) -> int:
    return int(lib().hsa_patch_workspace_size(M, D, Cc, dtype))


def patch_embed(x, idx, w_in, b_in, X, ws, stream=None):
    N, Cc = x.shape
    D = w_in.shape[0]
    _check(lib().hsa_patch_embed(_ptr(x), _ptr(idx), idx.shape[0], N, Cc, D, _dtype_code(w_in), _ptr(w_in),
                                 _ptr(b_in), _ptr(X), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hsa_patch_embed")


def velocity_head(X, head_mod, w_out, b_out, vA, ws, stream=None):
    M, D = X.shape
    _check(lib().hsa_velocity_head(_ptr(X), M, D, w_out.shape[0], _dtype_code(w_out), _ptr(head_mod), _ptr(w_out),
                                   _ptr(b_out), _ptr(vA), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "hsa_velocity_head")


def _device_copy(a, device, dtype):
    """A contiguous device tensor of `dtype` from a numpy array or a torch tensor."""
    import torch
    if isinstance(a, torch.Tensor):
        return a.to(device=device, dtype=dtype).contiguous()
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device).to(dtype)


# ---------------------------------------------------------------- head-parallel building blocks

def layernorm_rows(X, mul, add, out, modulate: bool, x_src=None, idx=None, stream=None):
    """out = LN(X)(1 + mul) + add (modulate) or LN(X) mul + add; with x_src, X = x_src[idx] first."""
    M, D = X.shape
    N = 0 if x_src is None else x_src.shape[0]
    _check(lib().hsa_layernorm_rows(_ptr(X), _ptr(x_src), _ptr(idx), M, N, D, _ptr(mul), _ptr(add),
                                    1 if modulate else 0, _dtype_code(out), _ptr(out), _stream(stream)),
           "hsa_layernorm_rows")


def row_sumsq(x, D: int, ss, ss_stride: int = 1, stream=None):
    """ss[r * ss_stride] = sum of squares of the first D elements of row r of x (2-D, any width)."""
    M = x.shape[0]
    _check(lib().hsa_row_sumsq(_ptr(x), x.stride(0), M, D, _dtype_code(x), _ptr(ss), ss_stride, _stream(stream)),
           "hsa_row_sumsq")


def qk_norm_rope_ext(qkv, M: int, D_total: int, ss, g_q, g_k, idx, pos, Q, kcache, vcache, stream=None):
    Dl = qkv.shape[1] // 3
    N = kcache.shape[0]
    _check(lib().hsa_qk_norm_rope_ext(_ptr(qkv), M, N, Dl, D_total, _ptr(ss), _ptr(g_q), _ptr(g_k), _ptr(idx),
                                      _ptr(pos), _dtype_code(qkv), _ptr(Q), _ptr(kcache), _ptr(vcache),
                                      _stream(stream)), "hsa_qk_norm_rope_ext")


def rms_rows_ext(x, M: int, D: int, D_total: int, ss, g, out, ss_stride: int = 1, stream=None):
    """out[:M] = x[:M, :D] * rsqrt(ss / D_total + eps) * g (ss None: a plain copy)."""
    _check(lib().hsa_rms_rows_ext(_ptr(x), x.stride(0), M, D, D_total, _ptr(ss), ss_stride, _ptr(g),
                                  _dtype_code(x), _ptr(out), _stream(stream)), "hsa_rms_rows_ext")


def gated_residual(X, y, b=None, gate=None, stream=None):
    M, D = X.shape
    _check(lib().hsa_gated_residual(_ptr(X), _ptr(y), M, D, _ptr(b), _ptr(gate), _stream(stream)),
           "hsa_gated_residual")


class HostSlot:
    """A device copy of the latent (N x D float32) and the three events of one hsa_iteration_host
    slot.  Each event is recorded once here, so that it exists and counts as complete."""

    def __init__(self, N: int, D: int, device="cuda"):
        import torch
        self.x = torch.empty((N, D), dtype=torch.float32, device=device)
        self.events = [torch.cuda.Event() for _ in range(3)]
        for e in self.events:
            e.record()
        self.c = HostSlotC(_ptr(self.x), *(e.cuda_event for e in self.events))


def iteration_host(w: "LayerWeights", kcache, vcache, idx, pos, xA, vhat, dsigma: float, h_x_in, h_x_out,
                   slot: HostSlot, ws, ctx_k=None, ctx_v=None, score=None, group_sizes=None, group=None,
                   order=None, sel_ws=None, stream=None, stream_h2d=None, stream_d2h=None):
    """One iteration with the latent in host memory (hsa_iteration_host): h_x_in / h_x_out are CPU
    tensors (N x D float32, pinned for overlap); the device state is as for layer_step,
    euler_update and select_tokens."""
    N, M = kcache.shape[0], idx.shape[0]
    sizes = np.ascontiguousarray(group_sizes if group_sizes is not None else [N], np.int32)
    a = IterationArgsC(C.pointer(w.c), _ptr(kcache), _ptr(vcache), N, _ptr(idx), M, _ptr(pos), _ptr(ctx_k),
                       _ptr(ctx_v), 0 if ctx_k is None else ctx_k.shape[0], _ptr(xA), _ptr(vhat), dsigma,
                       _ptr(score), len(sizes), sizes.ctypes.data, _ptr(group), _ptr(order), _ptr(ws),
                       ws.numel() * ws.element_size(), _ptr(sel_ws),
                       0 if sel_ws is None else sel_ws.numel() * sel_ws.element_size())
    _check(lib().hsa_iteration_host(C.byref(a), h_x_in.data_ptr(), h_x_out.data_ptr(), C.byref(slot.c),
                                    _stream(stream), _stream(stream_h2d), _stream(stream_d2h)),
           "hsa_iteration_host")


class LayerWeights:
    """Device copies of one block's parameters plus the C struct that points at them."""

    MATS = ("w_qkv", "w_o", "w_1", "w_2", "w_q2", "w_o2")
    VECS = ("b_qkv", "g_q", "g_k", "b_o", "b_1", "b_2", "mod", "ln_c_g", "ln_c_b", "b_q2", "g_q2", "b_o2")

    def __init__(self, bw, device, bf16: bool):
        import torch
        self.t = {}
        mat_dtype = torch.bfloat16 if bf16 else torch.float32
        for name in self.MATS:
            a = getattr(bw, name)
            if a is not None:
                self.t[name] = _device_copy(a, device, mat_dtype)
        for name in self.VECS:
            a = getattr(bw, name)
            if a is not None:
                self.t[name] = _device_copy(a, device, torch.float32)
        if bw.w_kv2 is not None:
            self.t["w_kv2"] = _device_copy(bw.w_kv2, device, mat_dtype)
            self.t["b_kv2"] = _device_copy(bw.b_kv2, device, torch.float32)
            self.t["g_k2"] = _device_copy(bw.g_k2, device, torch.float32)
        D, F = bw.w_o.shape[0], bw.w_1.shape[0]
        self.D, self.H, self.F = D, D // 128, F
        self.dtype = HSA_BF16 if bf16 else HSA_F32
        p = lambda n: _ptr(self.t.get(n))
        self.c = LayerWeightsC(D, D // 128, F, self.dtype, p("w_qkv"), p("b_qkv"), p("g_q"), p("g_k"), p("w_o"),
                               p("b_o"), p("w_1"), p("b_1"), p("w_2"), p("b_2"), p("mod"), p("ln_c_g"),
                               p("ln_c_b"), p("w_q2"), p("b_q2"), p("g_q2"), p("w_o2"), p("b_o2"))

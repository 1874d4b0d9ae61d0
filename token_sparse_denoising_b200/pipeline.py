"""One HSA denoising run on the device: the per-iteration sequence of libhsa calls.

This module only orders calls to the C ABI (through the ctypes binding) and
owns the device buffers; every arithmetic step runs in libhsa's kernels.

Iteration i (HSA summary §2.1-§2.4):
  1. A_i = the token lists of the groups that run at i (from hsa_plan_groups);
     with nested budgets (every period divides the next) it is a prefix of
     `order`, otherwise the active segments are copied together;
  2. v_A = model velocity of the active rows (hsa_layer_step per block with the
     per-layer KV caches; patch-embed / head around them for latent models);
  3-5. hsa_euler_update: v_hat[A_i] = v_A and x += (sigma_{i+1} - sigma_i) v_hat,
     with the L1 relative-change score fused in when every token ran;
  6. after such a full step, hsa_select_tokens regroups the tokens.
"""
from __future__ import annotations

import numpy as np
import torch

from . import hsa


def _to_dev(a, dtype=torch.float32, device="cuda"):
    if isinstance(a, torch.Tensor):
        return a.to(device=device, dtype=dtype).contiguous()
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device).to(dtype)


class SingleBlockModel:
    """One DiT block whose output rows are the velocity (latent channels C = D)."""

    def __init__(self, bw, pos, N: int, bf16: bool, ctx=None, device="cuda", cache_init=None):
        self.w = hsa.LayerWeights(bw, device, bf16)
        self.bf16 = bf16
        self.N, self.D, self.F = N, self.w.D, self.w.F
        dt = torch.bfloat16 if bf16 else torch.float32
        self.pos = torch.from_numpy(np.ascontiguousarray(pos, np.int32)).to(device)
        if cache_init is None:
            self.kc = torch.zeros((N, self.D), dtype=dt, device=device)
            self.vc = torch.zeros((N, self.D), dtype=dt, device=device)
        else:
            self.kc, self.vc = _to_dev(cache_init[0], dt, device), _to_dev(cache_init[1], dt, device)
        self.ws = torch.empty(hsa.layer_step_workspace_size(N, self.D, self.F, self.w.dtype), dtype=torch.uint8,
                              device=device)
        self.xA = torch.empty((N, self.D), dtype=torch.float32, device=device)
        self.ctx_k = self.ctx_v = None
        if ctx is not None:
            L = ctx.shape[0]
            c = _to_dev(ctx, dt, device)
            self.ctx_k = torch.empty((L, self.D), dtype=dt, device=device)
            self.ctx_v = torch.empty((L, self.D), dtype=dt, device=device)
            ws = torch.empty(hsa.context_kv_workspace_size(L, self.D), dtype=torch.uint8, device=device)
            hsa.context_kv(c, self.w.t["w_kv2"], self.w.t["b_kv2"], self.w.t["g_k2"], self.ctx_k, self.ctx_v, ws)

    def velocity(self, x, idx):
        M = idx.shape[0]
        xA = self.xA[:M]
        hsa.layer_step(self.w, self.kc, self.vc, xA, idx, self.pos, self.ws, x_src=x, ctx_k=self.ctx_k,
                       ctx_v=self.ctx_v)
        return xA


class PatchModel:
    """Patch-embedding C -> D, a stack of blocks with one KV cache each, output head D -> C."""

    def __init__(self, pm, pos, N: int, bf16: bool, ctx=None, device="cuda"):
        self.bf16 = bf16
        dt = torch.bfloat16 if bf16 else torch.float32
        self.dtype = hsa.HSA_BF16 if bf16 else hsa.HSA_F32
        self.N, self.C, self.D = N, pm.w_in.shape[1], pm.w_in.shape[0]
        self.w_in, self.b_in = _to_dev(pm.w_in, dt, device), _to_dev(pm.b_in, torch.float32, device)
        self.w_out, self.b_out = _to_dev(pm.w_out, dt, device), _to_dev(pm.b_out, torch.float32, device)
        self.head_mod = _to_dev(pm.head_mod, torch.float32, device)
        self.pos = torch.from_numpy(np.ascontiguousarray(pos, np.int32)).to(device)
        self.blocks = [hsa.LayerWeights(bw, device, bf16) for bw in pm.blocks]
        self.F = self.blocks[0].F
        self.kc = [torch.zeros((N, self.D), dtype=dt, device=device) for _ in self.blocks]
        self.vc = [torch.zeros((N, self.D), dtype=dt, device=device) for _ in self.blocks]
        self.ws = torch.empty(hsa.layer_step_workspace_size(N, self.D, self.F, self.dtype), dtype=torch.uint8,
                              device=device)
        self.pws = torch.empty(hsa.patch_workspace_size(N, self.D, self.C, self.dtype), dtype=torch.uint8,
                               device=device)
        self.X = torch.empty((N, self.D), dtype=torch.float32, device=device)
        self.vA = torch.empty((N, self.C), dtype=torch.float32, device=device)
        self.ctx_k, self.ctx_v = [None] * len(self.blocks), [None] * len(self.blocks)
        if ctx is not None:
            L = ctx.shape[0]
            c = _to_dev(ctx, dt, device)
            ws = torch.empty(hsa.context_kv_workspace_size(L, self.D), dtype=torch.uint8, device=device)
            for b, w in enumerate(self.blocks):
                self.ctx_k[b] = torch.empty((L, self.D), dtype=dt, device=device)
                self.ctx_v[b] = torch.empty((L, self.D), dtype=dt, device=device)
                hsa.context_kv(c, w.t["w_kv2"], w.t["b_kv2"], w.t["g_k2"], self.ctx_k[b], self.ctx_v[b], ws)

    def velocity(self, x, idx):
        M = idx.shape[0]
        X, vA = self.X[:M], self.vA[:M]
        hsa.patch_embed(x, idx, self.w_in, self.b_in, X, self.pws)
        for b, w in enumerate(self.blocks):
            hsa.layer_step(w, self.kc[b], self.vc[b], X, idx, self.pos, self.ws, ctx_k=self.ctx_k[b],
                           ctx_v=self.ctx_v[b])
        hsa.velocity_head(X, self.head_mod, self.w_out, self.b_out, vA, self.pws)
        return vA


def conditioning_frame_mask(pos, n_frames: int = 1) -> np.ndarray:
    """Image-to-video: the tokens of the first n_frames latent frames (the conditioning image),
    from the (N, 3) (frame, row, column) position table.  Pass it as HSARun(pinned=...)."""
    return np.asarray(pos)[:, 0] < n_frames


class HSARun:
    """Latent x, cached velocities v_hat and the token grouping of one run, plus its schedule.

    pinned (bool[N], optional): tokens kept in G_1 at every regrouping whatever their score
    (image-to-video: conditioning_frame_mask); see hsa_select_tokens_pinned.
    static_groups (int[N], optional): a fixed partition for the whole run (token n in group
    static_groups[n], group k holding sizes[k] tokens); full steps then do not regroup."""

    def __init__(self, model, x0, vhat0, T: int, budgets, sizes, m: int, sigma_kind: int, shift: float,
                 device="cuda", pinned=None, static_groups=None):
        self.model = model
        N = x0.shape[0]
        self.N, self.T, self.sizes = N, T, list(sizes)
        self.sigmas, self.table, self.n_active = hsa.plan_groups(T, list(budgets), self.sizes, N, m, sigma_kind,
                                                                 shift)
        self.x = _to_dev(x0, torch.float32, device)
        self.vhat = _to_dev(vhat0, torch.float32, device)
        self.static_order = None
        if static_groups is not None:
            g = np.asarray(static_groups, np.int64)
            if g.shape != (N,) or [int(np.sum(g == k)) for k in range(len(self.sizes))] != self.sizes:
                raise ValueError("static groups must give group k exactly sizes[k] tokens")
            self.static_order = np.concatenate([np.nonzero(g == k)[0] for k in range(len(self.sizes))])
        self.order = torch.arange(N, dtype=torch.int32, device=device) if self.static_order is None else \
            torch.from_numpy(self.static_order.astype(np.int32)).to(device)
        self.group = torch.zeros(N, dtype=torch.int8, device=device)
        self.score = torch.zeros(N, dtype=torch.float32, device=device)
        self.idx_buf = torch.empty(N, dtype=torch.int32, device=device)
        self.pinned = None if pinned is None else \
            torch.from_numpy(np.ascontiguousarray(pinned, bool).astype(np.uint8)).to(device)
        self.sel_ws = torch.empty(max(hsa.select_tokens_workspace_size(N, len(self.sizes)), 1), dtype=torch.uint8,
                                  device=device)
        self.starts = np.concatenate([[0], np.cumsum(self.sizes)]).astype(np.int64)
        self.i = 0

    def reset(self, x0, vhat0):
        """Start the run again from (x0, vhat0) in the same device buffers, so a captured graph of
        the loop can be replayed for a new latent."""
        self.x.copy_(torch.as_tensor(np.ascontiguousarray(x0, np.float32)))
        self.vhat.copy_(torch.as_tensor(np.ascontiguousarray(vhat0, np.float32)))
        self.order.copy_(torch.arange(self.N, dtype=torch.int32) if self.static_order is None else
                         torch.from_numpy(self.static_order.astype(np.int32)))
        self.group.zero_()
        self.score.zero_()
        self.i = 0

    def capture(self):
        """Record the remaining steps of the run (every launch of every step, selection included)
        as one CUDA graph and return it; replaying it runs those steps.  The schedule is fixed on
        the host, and the active index lists live at fixed device addresses whose contents the
        selection kernel rewrites, so one recording serves every replay.  Nothing executes
        during the recording: the state stays where it was, and replay(g) then runs the steps."""
        g = torch.cuda.CUDAGraph()
        i0 = self.i
        with torch.cuda.graph(g):
            self.run()
        self.i = i0
        return g

    def replay(self, g):
        """Run a graph from capture() on the current state (reset() first for a new latent)."""
        g.replay()
        self.i = self.T

    def active_index(self, i: int):
        act = self.table[i].astype(bool)
        M = int(self.n_active[i])
        K = len(self.sizes)
        first_off = next((k for k in range(K) if not act[k]), K)
        if not act[first_off:].any():
            return self.order[:M]            # nested budgets: the active groups are a prefix
        hsa.active_rows(self.order, self.sizes, act, self.idx_buf)
        return self.idx_buf[:M]

    def step(self, record: list | None = None):
        i = self.i
        idx = self.active_index(i)
        full = idx.shape[0] == self.N
        # a prefix view of `order`, which the regrouping below rewrites: copy it out first
        idx_rec = idx.cpu().numpy().copy() if record is not None else None
        vA = self.model.velocity(self.x, idx)
        dsig = float(np.float32(self.sigmas[i + 1]) - np.float32(self.sigmas[i]))
        regroup = full and self.static_order is None
        hsa.euler_update(self.x, self.vhat, vA, idx, dsig, score=self.score if regroup else None)
        if regroup:
            hsa.select_tokens(self.score, self.sizes, self.group, self.order, ws=self.sel_ws, pinned=self.pinned)
        if record is not None:
            record.append({"i": i, "M": int(idx.shape[0]), "full": full, "idx": idx_rec,
                           "score": self.score.cpu().numpy().copy() if regroup else None,
                           "order": self.order.cpu().numpy().copy()})
        self.i += 1

    def run(self, record: list | None = None):
        while self.i < self.T:
            self.step(record)
        return self.x

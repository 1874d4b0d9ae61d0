"""Head parallelism: one DiT block of the HSA step split over G GPUs.

The pages run the model on one device; for the Wan-14B shapes (40 heads, D = 5120) one block can
be split by heads.  Rank g of G holds:
  * heads [g H/G, (g+1) H/G): their rows of W_q, W_k, W_v (and b, the q/k RMSNorm gains), the KV
    cache of those heads for all N tokens, the matching columns of W_o (and of the cross-attention
    W_q2 / W_kv2 rows and W_o2 columns, the context K/V of those heads);
  * columns [g F/G, (g+1) F/G) of the FFN: rows of W_1 (and b_1), columns of W_2;
  * rows [g Mp/G, (g+1) Mp/G) of the active tokens' residual stream X (Mp = M rounded up to a
    multiple of G; rows at or past M are padding).

One block on the active rows (HSA summary §2.2), per rank, with the collectives between the
phases (all of them NCCL calls into local buffers; no kernel reads another GPU's memory):
  h = LN_mod(X_g)                      -> all-gather h          (Mp x D bf16)
  qkv = h W_qkv,g^T;  partial sums of q^2, k^2 over local channels
                                       -> all-reduce sums       (Mp x 2 float32)
  q, k <- RMSNorm (global sums) + RoPE; Kc_g[A_i], Vc_g[A_i] <- k, v
  o = attention over all N cached rows of the local heads
  y = o W_o,g^T (partial over heads)   -> reduce-scatter y      (Mp x D float32 -> rows of rank g)
  X_g += mod2 (y + b_o)
  [cross-attention: LN_affine -> all-gather, q2 partial sums -> all-reduce, attention against the
   local heads' context K/V, partial O2 -> reduce-scatter, X_g += y2 + b_o2]
  h = LN_mod(X_g)                      -> all-gather h
  y = GELU(h W_1,g^T + b_1,g) W_2,g^T  -> reduce-scatter y
  X_g += mod5 (y + b_2)

A step is written as a generator that yields each collective it needs (("all_gather", out, in),
("all_reduce", buf), ("reduce_scatter", out, in)); `run_collectives` serves them with
torch.distributed (one process per GPU), and `EmulatedGroup` serves G ranks' generators in one
process on one device, which is how the split is tested where only one GPU is available.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import hsa


@dataclass(frozen=True)
class HeadShard:
    """What rank `rank` of `world` owns of a block with H heads, FFN width F and M active rows."""
    rank: int
    world: int
    H: int
    F: int
    M: int

    def __post_init__(self):
        if self.world < 1 or not 0 <= self.rank < self.world:
            raise ValueError("need 0 <= rank < world")
        if self.H % self.world:
            raise ValueError(f"{self.H} heads do not split over {self.world} ranks")
        if self.F % (64 * self.world):
            raise ValueError(f"FFN width {self.F} does not split over {self.world} ranks in multiples of 64")
        if self.M < 1:
            raise ValueError("need at least one active row")

    @property
    def D(self) -> int:
        return 128 * self.H

    @property
    def heads(self) -> range:
        h = self.H // self.world
        return range(self.rank * h, (self.rank + 1) * h)

    @property
    def channels(self) -> slice:
        """The local heads' channels of q, k, v (and of the attention output)."""
        return slice(128 * self.heads.start, 128 * self.heads.stop)

    @property
    def Dl(self) -> int:
        return 128 * len(self.heads)

    @property
    def ffn(self) -> slice:
        f = self.F // self.world
        return slice(self.rank * f, (self.rank + 1) * f)

    @property
    def Mp(self) -> int:
        """Active rows padded to a multiple of the world size (equal reduce-scatter chunks)."""
        return -(-self.M // self.world) * self.world

    @property
    def rows(self) -> slice:
        """This rank's rows of the residual stream, in the padded row space."""
        r = self.Mp // self.world
        return slice(self.rank * r, (self.rank + 1) * r)

    @property
    def real_rows(self) -> int:
        """How many of this rank's rows are active tokens (the rest is padding)."""
        return max(0, min(self.rows.stop, self.M) - self.rows.start)


def shard_block_weights(bw, shard: HeadShard) -> dict:
    """The rank's slices of one block's parameters (numpy arrays or torch tensors alike).
    Full-width vectors (b_o, b_2, b_o2, mod, the cross-attention LayerNorm) are kept whole: they
    act on the residual stream after the reduction."""
    D, c, f = shard.D, shard.channels, shard.ffn
    cat = (lambda parts: torch.cat(parts)) if isinstance(bw.w_qkv, torch.Tensor) else \
        (lambda parts: np.concatenate(parts))
    qkv_rows = lambda a: cat([a[c], a[D + c.start:D + c.stop], a[2 * D + c.start:2 * D + c.stop]])
    s = {"w_qkv": qkv_rows(bw.w_qkv), "b_qkv": qkv_rows(bw.b_qkv), "g_q": bw.g_q[c], "g_k": bw.g_k[c],
         "w_o": bw.w_o[:, c], "b_o": bw.b_o, "w_1": bw.w_1[f], "b_1": bw.b_1[f], "w_2": bw.w_2[:, f],
         "b_2": bw.b_2, "mod": bw.mod}
    if bw.w_q2 is not None:
        s.update(ln_c_g=bw.ln_c_g, ln_c_b=bw.ln_c_b, w_q2=bw.w_q2[c], b_q2=bw.b_q2[c], g_q2=bw.g_q2[c],
                 w_kv2=cat([bw.w_kv2[c], bw.w_kv2[D + c.start:D + c.stop]]),
                 b_kv2=cat([bw.b_kv2[c], bw.b_kv2[D + c.start:D + c.stop]]), g_k2=bw.g_k2[c],
                 w_o2=bw.w_o2[:, c], b_o2=bw.b_o2)
    return s


def _dev(a, dtype, device):
    if isinstance(a, torch.Tensor):
        return a.to(device=device, dtype=dtype).contiguous()
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device).to(dtype).contiguous()


MATRICES = ("w_qkv", "w_o", "w_1", "w_2", "w_q2", "w_kv2", "w_o2")


class HeadParallelBlock:
    """One rank's part of a bf16 block: its weight slices, its heads' KV cache (N x Dl) and the
    buffers of one step for up to M active rows."""

    def __init__(self, bw, shard: HeadShard, N: int, device, cache_init=None):
        self.s = shard
        self.N = N
        self.device = device
        bf = torch.bfloat16
        self.w = {k: _dev(v, bf if k in MATRICES else torch.float32, device)
                  for k, v in shard_block_weights(bw, shard).items()}
        self.cross = "w_q2" in self.w
        D, Dl, Fl, Mp = shard.D, shard.Dl, shard.F // shard.world, shard.Mp
        if cache_init is None:
            self.kc = torch.zeros((N, Dl), dtype=bf, device=device)
            self.vc = torch.zeros((N, Dl), dtype=bf, device=device)
        else:
            self.kc = _dev(cache_init[0][:, shard.channels], bf, device)
            self.vc = _dev(cache_init[1][:, shard.channels], bf, device)
        R = Mp // shard.world
        self.X = torch.zeros((R, D), dtype=torch.float32, device=device)    # rank's rows of the stream
        self.h_full = torch.zeros((Mp, D), dtype=bf, device=device)
        self.qkv = torch.empty((Mp, 3 * Dl), dtype=bf, device=device)
        self.ss = torch.zeros((Mp, 2), dtype=torch.float32, device=device)
        self.q = torch.zeros((Mp, Dl), dtype=bf, device=device)             # padding rows stay zero
        self.q2 = torch.empty((Mp, Dl), dtype=bf, device=device) if "w_q2" in self.w else None
        self.o = torch.zeros((Mp, Dl), dtype=bf, device=device)
        self.y_full = torch.empty((Mp, D), dtype=torch.float32, device=device)
        self.y_loc = torch.empty((R, D), dtype=torch.float32, device=device)
        self.hid = torch.empty((Mp, Fl), dtype=bf, device=device)
        self.attn_ws = torch.empty(max(hsa.attention_workspace_size(shard.M, N, len(shard.heads), hsa.HSA_BF16), 16),
                                   dtype=torch.uint8, device=device)
        self.ctx_k = self.ctx_v = None

    # ---------------------------------------------------------------- once per run
    def context_kv(self, ctx):
        """Generator: the local heads' context keys/values (k RMSNorm over all D channels)."""
        L, Dl, D = ctx.shape[0], self.s.Dl, self.s.D
        c = _dev(ctx, torch.bfloat16, self.device)
        kv = torch.empty((L, 2 * Dl), dtype=torch.bfloat16, device=self.device)
        hsa.linear(c, self.w["w_kv2"], self.w["b_kv2"], hsa.EPI_STORE, kv)
        ss = torch.zeros((L, 1), dtype=torch.float32, device=self.device)
        hsa.row_sumsq(kv, Dl, ss)
        yield ("all_reduce", ss)
        self.ctx_k = torch.empty((L, Dl), dtype=torch.bfloat16, device=self.device)
        self.ctx_v = torch.empty((L, Dl), dtype=torch.bfloat16, device=self.device)
        hsa.rms_rows_ext(kv, L, Dl, D, ss, self.w["g_k2"], self.ctx_k)
        hsa.rms_rows_ext(kv[:, Dl:], L, Dl, D, None, None, self.ctx_v)

    # ---------------------------------------------------------------- one step
    def _gathered_ln(self, mul, add, modulate):
        s = self.s
        R = s.real_rows
        loc = self.h_full[s.rows]
        if R:
            hsa.layernorm_rows(self.X[:R], mul, add, loc[:R], modulate)
        return ("all_gather", self.h_full, loc)

    def _reduced_residual(self, b, gate):
        R = self.s.real_rows
        if R:
            hsa.gated_residual(self.X[:R], self.y_loc[:R], b, gate)

    def step(self, x_src, idx, pos):
        """Generator: one block on the active rows idx (length M) of the latent x_src (N x D
        float32).  On return self.X[:real_rows] holds this rank's rows of the block output."""
        s, w = self.s, self.w
        M, D, Dl = s.M, s.D, s.Dl
        assert idx.shape[0] == M
        r0, R = s.rows.start, s.real_rows
        mod = w["mod"]
        # a1: this rank's rows of the residual stream gathered from the latent, LN + modulation
        if R:
            hsa.layernorm_rows(self.X[:R], mod[1], mod[0], self.h_full[s.rows][:R], True, x_src=x_src,
                               idx=idx[r0:r0 + R])
        yield ("all_gather", self.h_full, self.h_full[s.rows])
        # a2: local heads' q/k/v of every active row; q/k RMS over all D channels
        hsa.linear(self.h_full, w["w_qkv"], w["b_qkv"], hsa.EPI_STORE, self.qkv)
        hsa.row_sumsq(self.qkv, Dl, self.ss[:, 0:], ss_stride=2)
        hsa.row_sumsq(self.qkv[:, Dl:], Dl, self.ss[:, 1:], ss_stride=2)
        yield ("all_reduce", self.ss)
        hsa.qk_norm_rope_ext(self.qkv, M, D, self.ss, w["g_q"], w["g_k"], idx, pos, self.q, self.kc, self.vc)
        # a3: the local heads attend over all N cached rows
        hsa.attention(self.q[:M], self.kc, self.vc, len(s.heads), self.o[:M], ws=self.attn_ws)
        # a4: partial output projection, reduced onto the row owners, gated residual
        hsa.linear(self.o, w["w_o"], None, hsa.EPI_F32, self.y_full)
        yield ("reduce_scatter", self.y_loc, self.y_full)
        self._reduced_residual(w["b_o"], mod[2])
        if self.cross:
            yield self._gathered_ln(w["ln_c_g"], w["ln_c_b"], False)
            q2 = self.q2
            hsa.linear(self.h_full, w["w_q2"], w["b_q2"], hsa.EPI_STORE, q2)
            ss = self.ss[:, 0:1]
            hsa.row_sumsq(q2, Dl, ss, ss_stride=2)
            yield ("all_reduce", self.ss)
            hsa.rms_rows_ext(q2, M, Dl, D, ss, w["g_q2"], self.q, ss_stride=2)
            hsa.attention(self.q[:M], self.ctx_k, self.ctx_v, len(s.heads), self.o[:M], ws=self.attn_ws)
            hsa.linear(self.o, w["w_o2"], None, hsa.EPI_F32, self.y_full)
            yield ("reduce_scatter", self.y_loc, self.y_full)
            self._reduced_residual(w["b_o2"], None)
        # a4: the FFN columns of this rank, partial FFN2 reduced onto the row owners
        yield self._gathered_ln(mod[4], mod[3], True)
        hsa.linear(self.h_full, w["w_1"], w["b_1"], hsa.EPI_GELU, self.hid)
        hsa.linear(self.hid, w["w_2"], None, hsa.EPI_F32, self.y_full)
        yield ("reduce_scatter", self.y_loc, self.y_full)
        self._reduced_residual(w["b_2"], mod[5])


def run_collectives(gen, dist, group=None):
    """Drive one rank's generator with torch.distributed collectives (NCCL on GPUs, gloo on CPU)."""
    for op in gen:
        kind = op[0]
        if kind == "all_gather":
            dist.all_gather_into_tensor(op[1], op[2].contiguous(), group=group)
        elif kind == "all_reduce":
            dist.all_reduce(op[1], group=group)
        elif kind == "reduce_scatter":
            dist.reduce_scatter_tensor(op[1], op[2], group=group)
        else:
            raise ValueError(f"unknown collective {kind}")


class EmulatedGroup:
    """G ranks' generators driven in one process: every collective is performed on the ranks'
    own buffers (device copies and sums), in the order the ranks reach it.  For testing the split
    where one device has to hold every rank."""

    @staticmethod
    def run(gens):
        gens = list(gens)
        G = len(gens)
        while True:
            ops = [next(g, None) for g in gens]
            if all(op is None for op in ops):
                return
            if any(op is None for op in ops) or len({op[0] for op in ops}) != 1:
                raise RuntimeError("ranks reached different collectives")
            kind = ops[0][0]
            if kind == "all_gather":
                parts = [op[2].clone() for op in ops]
                chunk = ops[0][1].shape[0] // G
                for op in ops:
                    for p, part in enumerate(parts):
                        op[1][p * chunk:(p + 1) * chunk].copy_(part)
            elif kind == "all_reduce":
                total = sum(op[1].clone() for op in ops)
                for op in ops:
                    op[1].copy_(total)
            elif kind == "reduce_scatter":
                total = sum(op[2].clone() for op in ops)
                chunk = total.shape[0] // G
                for p, op in enumerate(ops):
                    op[1].copy_(total[p * chunk:(p + 1) * chunk])
            else:
                raise ValueError(f"unknown collective {kind}")


def gather_block_output(blocks) -> torch.Tensor:
    """The active rows' block output from every rank's rows (one process holding all ranks)."""
    return torch.cat([b.X[:b.s.real_rows] for b in blocks])

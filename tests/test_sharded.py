"""Head parallelism on the CPU: the split's bookkeeping, and the split block restated in fp64
over real collectives between two gloo ranks, against the unsplit oracle.

`sharded_block_fp64` below follows the phases of HeadParallelBlock.step one for one (same
collectives in the same order, same buffers' shapes), with the oracle's fp64 primitives in
place of the CUDA kernels.  Driven by the product's `run_collectives` over torch.distributed
(gloo, world size 2) and by `EmulatedGroup` (one process, G = 1, 2, 4), it must reproduce
O.dit_block_active to rounding: that pins the partition of heads, FFN columns and rows, the
placement of biases and gates around the reductions, and the q/k RMS statistics summed over
ranks.  The CUDA path of the same phases is compared with the oracle on the GPU
(tests/test_gpu_sharded.py).
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import hsa_oracle as O  # noqa: E402
from token_sparse_denoising_b200 import synthetic as S  # noqa: E402
from token_sparse_denoising_b200.sharded import (EmulatedGroup, HeadShard, run_collectives,  # noqa: E402
                                                  shard_block_weights)

F64 = torch.float64


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float64))


def sharded_block_fp64(bw, shard: HeadShard, x, idx, pos, kc, vc, ctx_kv_local, out):
    """Generator: rank `shard.rank`'s part of one block in fp64 (mirrors HeadParallelBlock.step).
    kc, vc: the rank's cache columns (N x Dl float64 tensors, updated in place); ctx_kv_local: the
    rank's context K/V columns or None; out: dict receiving the rank's rows of the output."""
    w = {k: _t(v) for k, v in shard_block_weights(bw, shard).items()}
    M, D, Dl, Mp = shard.M, shard.D, shard.Dl, shard.Mp
    rows, R = shard.rows, shard.real_rows
    r0 = rows.start
    mod = w["mod"]
    X = torch.zeros((Mp // shard.world, D), dtype=F64)
    X[:R] = _t(x[idx[r0:r0 + R]])
    h_full = torch.zeros((Mp, D), dtype=F64)
    y_loc = torch.zeros((Mp // shard.world, D), dtype=F64)

    def ln_into_rows(mul, add, modulate):
        loc = h_full[rows]
        if R:
            g = (1.0 + mul) if modulate else mul
            loc[:R] = _t(O.layer_norm(X[:R].numpy())) * g + add
        return ("all_gather", h_full, loc)

    def residual(b, gate):
        if R:
            X[:R] += (1.0 if gate is None else gate) * (y_loc[:R] + b)

    yield ln_into_rows(mod[1], mod[0], True)
    qkv = h_full @ w["w_qkv"].T + w["b_qkv"]
    ss = torch.stack([(qkv[:, :Dl] ** 2).sum(1), (qkv[:, Dl:2 * Dl] ** 2).sum(1)], dim=1)
    yield ("all_reduce", ss)
    q = qkv[:M, :Dl] / torch.sqrt(ss[:M, 0:1] / D + O.RMS_EPS) * w["g_q"]
    k = qkv[:M, Dl:2 * Dl] / torch.sqrt(ss[:M, 1:2] / D + O.RMS_EPS) * w["g_k"]
    q, k = _t(O.rope_3d(q.numpy(), pos[idx])), _t(O.rope_3d(k.numpy(), pos[idx]))
    kc[idx] = k
    vc[idx] = qkv[:M, 2 * Dl:]
    o = torch.zeros((Mp, Dl), dtype=F64)
    o[:M] = _t(O.attention(q.numpy(), kc.numpy(), vc.numpy()))
    y_full = o @ w["w_o"].T
    yield ("reduce_scatter", y_loc, y_full)
    residual(w["b_o"], mod[2])
    if ctx_kv_local is not None:
        yield ln_into_rows(w["ln_c_g"], w["ln_c_b"], False)
        q2 = h_full @ w["w_q2"].T + w["b_q2"]
        ss2 = torch.zeros((Mp, 2), dtype=F64)
        ss2[:, 0] = (q2 ** 2).sum(1)
        yield ("all_reduce", ss2)
        q2 = q2[:M] / torch.sqrt(ss2[:M, 0:1] / D + O.RMS_EPS) * w["g_q2"]
        o = torch.zeros((Mp, Dl), dtype=F64)
        o[:M] = _t(O.attention(q2.numpy(), ctx_kv_local[0], ctx_kv_local[1]))
        y_full = o @ w["w_o2"].T
        yield ("reduce_scatter", y_loc, y_full)
        residual(w["b_o2"], None)
    yield ln_into_rows(mod[4], mod[3], True)
    hid = _t(O.gelu_tanh((h_full @ w["w_1"].T + w["b_1"]).numpy()))
    y_full = hid @ w["w_2"].T
    yield ("reduce_scatter", y_loc, y_full)
    residual(w["b_2"], mod[5])
    out["rows"] = X[:R].numpy().copy()


def context_kv_fp64(bw, shard: HeadShard, ctx):
    """Generator: the rank's context K/V columns (k RMSNorm over all D channels); result in out."""
    w = {k: _t(v) for k, v in shard_block_weights(bw, shard).items()}
    Dl, D = shard.Dl, shard.D
    kv = _t(ctx) @ w["w_kv2"].T + w["b_kv2"]
    ss = (kv[:, :Dl] ** 2).sum(1, keepdim=True)
    yield ("all_reduce", ss)
    k = kv[:, :Dl] / torch.sqrt(ss / D + O.RMS_EPS) * w["g_k2"]
    return k.numpy(), kv[:, Dl:].numpy()


def _case(cross: bool, M: int, seed: int = 3):
    grid = S.Grid(2, 4, 6)                          # N = 48
    N, D, F = grid.N, 512, 1024                     # 4 heads, FFN 1024
    shape = S.BlockShape(D, 4, F, cross, 8)
    bw = S.perturb_vectors(S.block_weights(seed, shape, False, 0.05), seed + 1)
    pos = S.token_positions(grid)
    x = S.normal(seed + 2, (N, D)).astype(np.float64)
    kc0, vc0 = S.normal(seed + 3, (N, D)).astype(np.float64), S.normal(seed + 4, (N, D)).astype(np.float64)
    idx = S.scattered_mask(seed + 5, N, M).astype(np.int64)
    ctx = S.normal(seed + 6, (8, D)).astype(np.float64) if cross else None
    return grid, bw, pos, x, kc0, vc0, idx, ctx


def _reference(bw, pos, x, kc0, vc0, idx, ctx):
    ctx_kv = O.context_kv(bw, ctx) if ctx is not None else None
    return O.dit_block_active(bw, x[idx], idx, pos, kc0, vc0, ctx_kv)


# ---------------------------------------------------------------- bookkeeping

@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_shards_partition_heads_ffn_and_rows(G):
    H, F, M = 40, 13824, 32757
    shards = [HeadShard(g, G, H, F, M) for g in range(G)]
    heads = sorted(h for s in shards for h in s.heads)
    assert heads == list(range(H))
    ch = np.concatenate([np.arange(128 * H)[s.channels] for s in shards])
    assert np.array_equal(ch, np.arange(128 * H))
    ffn = np.concatenate([np.arange(F)[s.ffn] for s in shards])
    assert np.array_equal(ffn, np.arange(F))
    assert all(s.Mp % G == 0 and s.Mp - M < G for s in shards)
    rows = np.concatenate([np.arange(s.Mp)[s.rows] for s in shards])
    assert np.array_equal(rows, np.arange(shards[0].Mp))
    assert sum(s.real_rows for s in shards) == M


def test_shard_rejects_uneven_splits():
    with pytest.raises(ValueError):
        HeadShard(0, 3, 40, 13824, 10)          # 40 heads over 3 ranks
    with pytest.raises(ValueError):
        HeadShard(0, 8, 16, 8960, 10)           # 8960 / 8 = 1120 is not a multiple of 64
    with pytest.raises(ValueError):
        HeadShard(2, 2, 12, 8960, 10)


@pytest.mark.parametrize("G", [2, 4])
def test_weight_slices_reassemble_the_block(G):
    _, bw, *_ = _case(True, 10)
    D = bw.w_o.shape[0]
    parts = [shard_block_weights(bw, HeadShard(g, G, D // 128, bw.w_1.shape[0], 10)) for g in range(G)]
    Dl = D // G
    q = np.concatenate([p["w_qkv"][:Dl] for p in parts])
    k = np.concatenate([p["w_qkv"][Dl:2 * Dl] for p in parts])
    v = np.concatenate([p["w_qkv"][2 * Dl:] for p in parts])
    assert np.array_equal(np.concatenate([q, k, v]), bw.w_qkv)
    assert np.array_equal(np.concatenate([p["w_o"] for p in parts], axis=1), bw.w_o)
    assert np.array_equal(np.concatenate([p["w_1"] for p in parts]), bw.w_1)
    assert np.array_equal(np.concatenate([p["w_2"] for p in parts], axis=1), bw.w_2)
    kk = np.concatenate([p["w_kv2"][:Dl] for p in parts])
    vv = np.concatenate([p["w_kv2"][Dl:] for p in parts])
    assert np.array_equal(np.concatenate([kk, vv]), bw.w_kv2)
    assert np.array_equal(np.concatenate([p["g_q"] for p in parts]), bw.g_q)


# ---------------------------------------------------------------- one process, emulated ranks

@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("cross,M", [(False, 17), (True, 17), (True, 48)])
def test_split_block_fp64_equals_oracle_emulated(G, cross, M):
    grid, bw, pos, x, kc0, vc0, idx, ctx = _case(cross, M)
    want, Kw, Vw = _reference(bw, pos, x, kc0, vc0, idx, ctx)
    H, F = bw.w_o.shape[0] // 128, bw.w_1.shape[0]
    shards = [HeadShard(g, G, H, F, M) for g in range(G)]
    ctx_local = [None] * G
    if cross:
        gens = [context_kv_fp64(bw, s, ctx) for s in shards]
        results = [None] * G

        def capture(g, gen):
            results[g] = yield from gen

        EmulatedGroup.run(capture(g, gen) for g, gen in enumerate(gens))
        ctx_local = results
    kcs = [_t(kc0[:, s.channels]) for s in shards]
    vcs = [_t(vc0[:, s.channels]) for s in shards]
    outs = [{} for _ in shards]
    EmulatedGroup.run(sharded_block_fp64(bw, s, x, idx, pos, kcs[g], vcs[g], ctx_local[g], outs[g])
                      for g, s in enumerate(shards))
    got = np.concatenate([o["rows"] for o in outs])
    assert np.max(np.abs(got - want)) < 1e-10
    for g, s in enumerate(shards):
        assert np.max(np.abs(kcs[g].numpy() - Kw[:, s.channels])) < 1e-12
        assert np.max(np.abs(vcs[g].numpy() - Vw[:, s.channels])) < 1e-12


def test_split_block_detects_a_misplaced_bias():
    """Planted mistake: the output-projection bias added by every rank (before the reduction)
    instead of once after it must show up as a difference from the oracle."""
    grid, bw, pos, x, kc0, vc0, idx, ctx = _case(False, 17)
    bw.b_o = bw.b_o + 0.5
    want, _, _ = _reference(bw, pos, x, kc0, vc0, idx, None)
    G = 2
    H, F = bw.w_o.shape[0] // 128, bw.w_1.shape[0]
    shards = [HeadShard(g, G, H, F, 17) for g in range(G)]

    def wrong(bw, s, *a):
        first = True
        for op in sharded_block_fp64(bw, s, *a):
            if op[0] == "reduce_scatter" and first:
                op[2].add_(_t(bw.b_o))            # every rank adds the bias to its partial sum
                first = False
            yield op

    outs = [{} for _ in shards]
    EmulatedGroup.run(wrong(bw, s, x, idx, pos, _t(kc0[:, s.channels]), _t(vc0[:, s.channels]), None, outs[g])
                      for g, s in enumerate(shards))
    got = np.concatenate([o["rows"] for o in outs])
    assert np.max(np.abs(got - want)) > 1e-3


# ---------------------------------------------------------------- two gloo ranks

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, cross):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M = 23
        grid, bw, pos, x, kc0, vc0, idx, ctx = _case(cross, M)
        H, F = bw.w_o.shape[0] // 128, bw.w_1.shape[0]
        s = HeadShard(rank, world, H, F, M)
        ctx_local = None
        if cross:
            gen = context_kv_fp64(bw, s, ctx)
            ctx_local = []

            def keep():
                ctx_local.extend((yield from gen))

            run_collectives(keep(), dist)
        kc, vc = _t(kc0[:, s.channels]), _t(vc0[:, s.channels])
        out = {}
        run_collectives(sharded_block_fp64(bw, s, x, idx, pos, kc, vc, ctx_local, out), dist)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), rows=out["rows"], kc=kc.numpy(), vc=vc.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cross", [False, True])
def test_split_block_over_two_gloo_ranks_equals_oracle(tmp_path, cross):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), cross), nprocs=world, join=True,
                       start_method="spawn")
    M = 23
    grid, bw, pos, x, kc0, vc0, idx, ctx = _case(cross, M)
    want, Kw, Vw = _reference(bw, pos, x, kc0, vc0, idx, ctx)
    parts = [np.load(os.path.join(tmp_path, f"rank{r}.npz")) for r in range(world)]
    got = np.concatenate([p["rows"] for p in parts])
    assert got.shape == want.shape
    assert np.max(np.abs(got - want)) < 1e-10
    H, F = bw.w_o.shape[0] // 128, bw.w_1.shape[0]
    for r, p in enumerate(parts):
        c = HeadShard(r, world, H, F, M).channels
        assert np.max(np.abs(p["kc"] - Kw[:, c])) < 1e-12 and np.max(np.abs(p["vc"] - Vw[:, c])) < 1e-12

"""Parity of each CUDA building block with the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import hsa_oracle as O
from token_sparse_denoising_b200 import synthetic as S
from tests._util import (assert_bf16_close, assert_f32_close, dev, host, max_abs, rel_l2)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ §2.3 cached Euler + §2.1 score

@pytest.mark.parametrize("N,C,M", [(1000, 64, 1000), (1000, 64, 377), (333, 1536, 333), (333, 1536, 100),
                                   (7, 4, 0)])
def test_euler_update(cuda_lib, N, C, M):
    hsa = cuda_lib
    x0, vh0 = S.normal(1, (N, C)), S.normal(2, (N, C))
    vA = S.normal(3, (M, C))
    idx = S.scattered_mask(4, N, M)
    dsig = np.float32(-0.0375)
    x, vh, va, ix = dev(x0), dev(vh0), dev(vA), dev(idx)
    score = torch.full((N,), -1.0, device="cuda")
    hsa.euler_update(x, vh, va if M else None, ix if M else None, float(dsig), score=score if M else None)
    assert hsa.device_status() == 0
    want_x, want_vh = O.cached_euler(x0, vh0, vA, idx, dsig)
    assert_f32_close(host(x), want_x, "x")
    assert np.array_equal(host(vh), want_vh.astype(np.float32))
    if M:
        want_s = O.l1_relative_change(vA, vh0[idx])
        assert rel_l2(host(score)[idx], want_s) < 1e-5
        untouched = np.setdiff1d(np.arange(N), idx)
        assert np.all(host(score)[untouched] == -1.0)


def test_l1_score(cuda_lib):
    N, C = 5000, 1536
    a, b = S.normal(5, (N, C)), S.normal(6, (N, C))
    b[17] = 0.0                                          # zero previous velocity -> eps denominator
    s = torch.empty(N, device="cuda")
    cuda_lib.l1_score(dev(a), dev(b), s)
    want = O.l1_relative_change(a, b)
    got = host(s)
    assert rel_l2(np.delete(got, 17), np.delete(want, 17)) < 1e-5
    assert got[17] == pytest.approx(want[17], rel=1e-5)


# ------------------------------------------------------------------ §2.1 selection: bit-exact

def _select_case(seed, N, K, kind):
    r = np.random.default_rng(seed)
    if kind == "ties":
        scores = r.choice(np.float32([0.0, 0.125, 0.5, 0.5000001, 1.0, np.nan, -1.0]), size=N).astype(np.float32)
    elif kind == "const":
        scores = np.full(N, 0.25, np.float32)
    else:
        scores = r.random(N, dtype=np.float32) * r.choice([1e-3, 1.0, 1e3], size=N).astype(np.float32)
    cuts = np.sort(r.integers(0, N + 1, size=K - 1))
    sizes = [int(v) for v in np.diff(np.concatenate([[0], cuts, [N]]))]
    return scores, sizes


@pytest.mark.parametrize("seed,N,K,kind", [(0, 1, 1, "rand"), (1, 5, 3, "ties"), (2, 1000, 2, "rand"),
                                           (3, 1000, 4, "ties"), (4, 4097, 5, "const"), (5, 32760, 3, "rand"),
                                           (6, 32760, 16, "ties"), (7, 75600, 3, "rand"), (8, 75600, 3, "const"),
                                           (9, 300000, 3, "ties")])
def test_select_tokens_bit_exact(cuda_lib, seed, N, K, kind):
    """Bit-exact against the oracle.  The selection spreads N over the 8 CTAs of a cluster in ranges of
    whole 1024-index blocks: one token, fewer tokens than one CTA's range (CTAs with nothing),
    ragged ranges, all-equal scores (every boundary decided by token index across CTAs), up to 16
    groups, and N = 300000, where each CTA's range exceeds what it stages in shared memory."""
    scores, sizes = _select_case(seed, N, K, kind)
    if seed == 5:
        sizes = S.group_sizes(N, (0.25, 0.25, 0.5))
    group = torch.full((N,), -7, dtype=torch.int8, device="cuda")
    order = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    cuda_lib.select_tokens(dev(scores), sizes, group, order)
    assert cuda_lib.device_status() == 0
    want_g, want_o = O.select_groups(scores, sizes)
    assert np.array_equal(host(group), want_g)
    assert np.array_equal(host(order), want_o)


@pytest.mark.parametrize("seed,N,K,kind,pin", [(10, 6, 3, "ties", "random"), (11, 1000, 3, "ties", "random"),
                                               (12, 32760, 3, "rand", "first_frame"), (13, 32760, 3, "ties", "many"),
                                               (14, 4097, 4, "const", "random"), (15, 75600, 3, "rand", "first_frame"),
                                               (16, 1000, 2, "rand", "all"), (17, 1000, 3, "rand", "none")])
def test_select_tokens_pinned_bit_exact(cuda_lib, seed, N, K, kind, pin):
    """Pinned tokens (image-to-video: the conditioning frame) rank ahead of all others; compared
    bit for bit with the oracle.  'many' pins more tokens than G_1 holds (they continue into G_2
    by index); N = 75600 takes the unstaged path."""
    scores, sizes = _select_case(seed, N, K, kind)
    if K == 3 and pin in ("first_frame", "many"):
        sizes = S.group_sizes(N, (0.25, 0.25, 0.5))
    r = np.random.default_rng(seed + 1000)
    pinned = {"random": r.random(N) < 0.2, "first_frame": np.arange(N) < N // 21,
              "many": r.random(N) < 0.4, "all": np.ones(N, bool), "none": np.zeros(N, bool)}[pin]
    group = torch.full((N,), -7, dtype=torch.int8, device="cuda")
    order = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    cuda_lib.select_tokens(dev(scores), sizes, group, order, pinned=torch.from_numpy(pinned.astype(np.uint8)).cuda())
    assert cuda_lib.device_status() == 0
    want_g, want_o = O.select_groups(scores, sizes, pinned)
    assert np.array_equal(host(group), want_g)
    assert np.array_equal(host(order), want_o)


@pytest.mark.parametrize("seed,N,K", [(0, 1000, 3), (1, 32760, 4), (2, 7, 5), (3, 75600, 16)])
def test_active_rows_bit_exact(cuda_lib, seed, N, K):
    """A_i from the group lists for every active pattern of K groups (nested or not), against the
    oracle's active_rows; includes groups of size 0, nothing active and everything active."""
    r = np.random.default_rng(seed)
    order = r.permutation(N).astype(np.int32)
    cuts = np.sort(r.integers(0, N + 1, size=K - 1))
    sizes = [int(v) for v in np.diff(np.concatenate([[0], cuts, [N]]))]
    masks = [r.random(K) < 0.5 for _ in range(6)] + [np.zeros(K, bool), np.ones(K, bool)]
    d_order = torch.from_numpy(order).cuda()
    for act in masks:
        idx = torch.full((N + 1,), -9, dtype=torch.int32, device="cuda")
        M = cuda_lib.active_rows(d_order, sizes, act, idx)
        want = O.active_rows(order, sizes, act)
        assert M == len(want)
        got = host(idx)
        assert np.array_equal(got[:M], want) and np.all(got[M:] == -9)
    assert cuda_lib.device_status() == 0


# ------------------------------------------------------------------ linear layers

def _lin_case(seed, M, K, Nout, bf16):
    x = S.normal(seed, (M, K), 1.0, bf16)
    w = S.normal(seed + 1, (Nout, K), 1.0 / np.sqrt(K), bf16)
    b = S.normal(seed + 2, (Nout,), 0.1)
    g = S.normal(seed + 3, (Nout,), 0.5)
    y0 = S.normal(seed + 4, (M, Nout))
    return x, w, b, g, y0


@pytest.mark.parametrize("M,K,Nout", [(300, 256, 768), (129, 128, 64), (1000, 512, 384), (1, 64, 128),
                                      (4097, 1536, 512),
                                      # 256-column outputs with more than 128 rows: the two-CTA kernel;
                                      # a pair whose second CTA holds one valid row, a single k-block,
                                      # and a k-loop that wraps the six-stage ring several times
                                      (129, 128, 256), (257, 64, 256), (2048, 1024, 2304)])
@pytest.mark.parametrize("epi", [0, 1, 2, 3])
def test_linear_bf16(cuda_lib, M, K, Nout, epi):
    """bf16 linear layer against the oracle for every epilogue: outputs of 256 columns with more than
    128 rows run the two-CTA (cta_group::2) kernel, the others the one-CTA kernel."""
    hsa = cuda_lib
    x, w, b, g, y0 = _lin_case(11, M, K, Nout, True)
    acc = O.linear(x, w, b)
    if epi in (0, 1):
        y = torch.empty((M, Nout), dtype=torch.bfloat16, device="cuda")
        want = O.gelu_tanh(acc) if epi == 1 else acc
    elif epi == 2:
        y = dev(y0)
        want = y0 + g * acc
    else:
        y = torch.empty((M, Nout), dtype=torch.float32, device="cuda")
        want = acc
    hsa.linear(dev(x, torch.bfloat16), dev(w, torch.bfloat16), dev(b), epi, y, gate=dev(g) if epi == 2 else None)
    assert hsa.device_status() == 0
    got = host(y)
    if epi == 2:
        assert_bf16_close(got - y0, want - y0, "residual delta")
    else:
        assert_bf16_close(got, want, f"epilogue {epi}")


@pytest.mark.parametrize("M,K,Nout,epi", [(300, 256, 768, 0), (70, 128, 64, 1), (65, 256, 1024, 2)])
def test_linear_f32(cuda_lib, M, K, Nout, epi):
    x, w, b, g, y0 = _lin_case(21, M, K, Nout, False)
    acc = O.linear(x, w, b)
    y = dev(y0) if epi == 2 else torch.empty((M, Nout), device="cuda")
    cuda_lib.linear(dev(x), dev(w), dev(b), epi, y, gate=dev(g) if epi == 2 else None)
    want = {0: acc, 1: O.gelu_tanh(acc), 2: y0 + g * acc}[epi]
    assert_f32_close(host(y), want)


# ------------------------------------------------------------------ §2.2 attention

@pytest.mark.parametrize("M,L,H,qscale", [(200, 1000, 2, 1.0), (128, 128, 1, 1.0), (1, 1, 1, 1.0),
                                          (257, 300, 3, 4.0), (130, 256, 2, 1.0), (100, 129, 1, 4.0),
                                          # more than 8 key tiles: the two-parity kernel
                                          (64, 4000, 2, 1.0), (130, 1100, 2, 1.0), (257, 1153, 3, 4.0),
                                          (1, 1025, 1, 1.0), (128, 1152, 1, 1.0),
                                          (256, 1153, 3, 4.0), (512, 3000, 2, 1.0), (250, 1500, 1, 1.0)])
def test_attention_bf16(cuda_lib, M, L, H, qscale):
    """Key ranges of at most 8 tiles (1024 keys) run the one-parity kernel, longer ones the
    two-parity kernel: ragged query and key tiles of both, one query row, one key."""
    D = 128 * H
    q = S.normal(31, (M, D), qscale, True)
    k, v = S.normal(32, (L, D), 1.0, True), S.normal(33, (L, D), 1.0, True)
    o = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    cuda_lib.attention(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), H, o)
    assert cuda_lib.device_status() == 0
    assert_bf16_close(host(o), O.attention(q, k, v), "attention")


@pytest.mark.parametrize("L", [700, 1500])
def test_attention_rescale_across_tiles(cuda_lib, L):
    """Logits that jump in a late key tile force the lazy O rescale (one-parity kernel at 700
    keys, two-parity kernel at 1500)."""
    M, H = 130, 1
    q = S.normal(41, (M, 128), 1.0, True)
    k = S.normal(42, (L, 128), 0.3, True)
    v = S.normal(43, (L, 128), 1.0, True)
    k[L - 100:L - 90] = S.round_bf16(np.repeat(q[:1] * 0.9, 10, 0))   # large logits for rows like q[0] late
    k[300] = S.round_bf16(q[5] * 0.7)
    o = torch.empty((M, 128), dtype=torch.bfloat16, device="cuda")
    cuda_lib.attention(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), H, o)
    assert_bf16_close(host(o), O.attention(q, k, v), "attention with late max")


def test_attention_identical_keys_give_mean_value(cuda_lib):
    M, L = 50, 513
    q = S.normal(51, (M, 128), 1.0, True)
    k = np.tile(S.normal(52, (1, 128), 1.0, True), (L, 1))
    v = S.normal(53, (L, 128), 1.0, True)
    o = torch.empty((M, 128), dtype=torch.bfloat16, device="cuda")
    cuda_lib.attention(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), 1, o)
    assert max_abs(host(o), np.tile(v.astype(np.float64).mean(0), (M, 1))) < 1e-2


@pytest.mark.parametrize("M,L,H", [(1000, 4000, 12), (300, 1100, 2), (100, 1536, 2), (129, 2000, 3)])
def test_attention_split_tail_matches_oracle(cuda_lib, M, L, H):
    """With a workspace the units of the last, incomplete wave are split over key ranges and
    merged by a second kernel (1000 x 4000 x 12 heads: 96 units, 3 ranges each; 300 x 1100: the
    last range holds the ragged key tile; 100 x 1536: one query tile, ranges of two tiles).
    Checked against the oracle, and against the unsplit kernel to fp32-merge rounding."""
    D = 128 * H
    q = S.normal(71, (M, D), 1.0, True)
    k, v = S.normal(72, (L, D), 1.0, True), S.normal(73, (L, D), 1.0, True)
    need = cuda_lib.attention_workspace_size(M, L, H, cuda_lib.HSA_BF16)
    assert need > 0                                    # these shapes do split
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    o1 = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    qd, kd, vd = dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16)
    cuda_lib.attention(qd, kd, vd, H, o, ws=ws)
    cuda_lib.attention(qd, kd, vd, H, o1)
    assert cuda_lib.device_status() == 0
    assert_bf16_close(host(o), O.attention(q, k, v), "split attention")
    assert max_abs(host(o), host(o1)) <= 2 ** -7          # at most a bf16 step apart
    # a workspace one byte short runs every unit whole: bit-identical to hsa_attention
    short = torch.empty(need - 1, dtype=torch.uint8, device="cuda")
    o2 = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    cuda_lib.attention(qd, kd, vd, H, o2, ws=short)
    assert torch.equal(o2, o1)


@pytest.mark.parametrize("M,L,H", [(256, 512, 12), (300, 16, 2), (200, 300, 2), (2000, 1000, 3), (129, 1024, 1),
                                   (640, 129, 2), (100, 512, 2), (1, 64, 1), (4096, 1024, 4), (40000, 64, 1),
                                   (20000, 300, 3)])
def test_attention_short_key_range(cuda_lib, M, L, H):
    """Key ranges of at most 8 tiles (the cross-attention's context) run the persistent
    one-parity kernel, two CTAs per SM, each walking its units: exact query tiles, ragged last
    query tiles (300, 200, 2000, 129, 100, 40000, 20000 rows), a single query row, a single ragged
    key tile (16 keys), the largest range that takes this path (1024 keys), a ragged 129-key
    range, and more units than CTAs (313 and 471 units: some CTAs take two, across heads)."""
    D = 128 * H
    q = S.normal(91, (M, D), 2.0, True)
    k, v = S.normal(92, (L, D), 1.0, True), S.normal(93, (L, D), 1.0, True)
    assert cuda_lib.attention_workspace_size(M, L, H, cuda_lib.HSA_BF16) == 0      # no key-range split
    o = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    cuda_lib.attention(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), H, o)
    assert cuda_lib.device_status() == 0
    assert_bf16_close(host(o), O.attention(q, k, v), "attention, short key range")


def test_attention_short_key_range_wan_cross(cuda_lib):
    """The Wan-1.3B cross-attention shape: 32760 queries against the 512-row context, 12 heads
    (256 query tiles per head, the last one ragged); sampled rows against the oracle."""
    M, L, H = 32760, 512, 12
    D = 128 * H
    q = S.normal(94, (M, D), 1.0, True)
    k, v = S.normal(95, (L, D), 1.0, True), S.normal(96, (L, D), 1.0, True)
    o = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    cuda_lib.attention(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), H, o)
    assert cuda_lib.device_status() == 0
    rows = np.array([0, 127, 128, 255, 256, 16000, 32639, 32640, 32700, 32759])
    assert_bf16_close(host(o)[rows], O.attention(q[rows], k, v), "cross-attention shape, sampled rows")


def test_attention_split_tail_wan_quarter(cuda_lib):
    """The Wan-1.3B shape at |A|/N = 1/4 (8190 queries, 32760 keys, 12 heads): 768 units, the 28
    of the incomplete last wave split 5 ways; sampled rows against the oracle."""
    M, L, H = 8190, 32760, 12
    D = 128 * H
    q = S.normal(81, (M, D), 1.0, True)
    k, v = S.normal(82, (L, D), 1.0, True), S.normal(83, (L, D), 1.0, True)
    need = cuda_lib.attention_workspace_size(M, L, H, cuda_lib.HSA_BF16)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    cuda_lib.attention(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), H, o, ws=ws)
    assert cuda_lib.device_status() == 0
    # rows of whole units, of split units (tail = units 740..767: heads 11 and 12 of the tiles), ragged end
    rows = np.array([0, 1, 4000, 7000, 7424, 7900, 8100, 8189])
    got = host(o)[rows]
    want = O.attention(q[rows], k, v)
    assert_bf16_close(got, want, "split attention, sampled rows")


@pytest.mark.parametrize("M,L,H", [(100, 300, 2), (1, 1024, 1), (33, 65, 1)])
def test_attention_f32(cuda_lib, M, L, H):
    D = 128 * H
    q, k, v = S.normal(61, (M, D)), S.normal(62, (L, D)), S.normal(63, (L, D))
    o = torch.empty((M, D), device="cuda")
    cuda_lib.attention(dev(q), dev(k), dev(v), H, o)
    assert_f32_close(host(o), O.attention(q, k, v))


@pytest.mark.parametrize("M,L,H", [(1024, 1024, 2), (512, 1024, 2), (37, 300, 3), (1, 200, 1)])
def test_attention_f32_key_range_split(cuda_lib, M, L, H):
    """fp32 attention with a workspace: the (32-query block, head) units are split over key ranges
    so that small active sets fill the GPU, and a second kernel merges the ranges (the tiny loop's
    1024- and 512-row steps, a ragged block, a single query row)."""
    D = 128 * H
    q, k, v = S.normal(64, (M, D)), S.normal(65, (L, D)), S.normal(66, (L, D))
    need = cuda_lib.attention_workspace_size(M, L, H, cuda_lib.HSA_F32)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o = torch.empty((M, D), device="cuda")
    cuda_lib.attention(dev(q), dev(k), dev(v), H, o, ws=ws)
    assert cuda_lib.device_status() == 0
    assert_f32_close(host(o), O.attention(q, k, v))

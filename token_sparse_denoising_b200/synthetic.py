"""Seeded synthetic inputs for the HSA hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CUDA path and the CPU oracle consume the arrays
it returns, so a parity test feeds them identical inputs.

The pages evaluate on trained Wan / LTX weights and VBench prompts, which are
not available here.  These generators stand in for them with random-init
weights of the named shapes (N(0, 0.02^2) projections, zero biases, unit norm
gains), unit-normal latents, velocities, contexts and cache contents, and
tokens in raster order over (frames x height x width) latent patches.

Every generator takes an explicit seed and uses numpy's PCG64.  Values are
drawn in float32; the bf16 workloads round them to bf16 (round to nearest
even) and hand the rounded values to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128
ROPE_SPLIT = (44, 42, 42)


# ---------------------------------------------------------------- bf16 marshalling

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # u + 0x7FFF + lsb stays below 2^32 for every non-NaN pattern (the largest, -inf, is
    # 0xFF800000), so 32-bit arithmetic is exact; NaNs are replaced afterwards
    t = (u >> 16) & np.uint32(1)
    t += np.uint32(0x7FFF)
    t += u
    t >>= 16
    out = t.astype(np.uint16)
    out[np.isnan(a)] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """float32 array whose values are exactly representable in bf16."""
    return bf16_bits_to_f32(f32_to_bf16_bits(a))


# ---------------------------------------------------------------- shapes

@dataclass(frozen=True)
class BlockShape:
    D: int            # hidden width
    H: int            # heads (head dim is always 128)
    F: int            # FFN width
    cross: bool       # cross-attention against a text context
    ctx_len: int = 512

    def __post_init__(self):
        if self.D != self.H * HEAD_DIM:
            raise ValueError("hidden width must equal heads x 128")


@dataclass(frozen=True)
class Grid:
    frames: int
    height: int
    width: int

    @property
    def N(self) -> int:
        return self.frames * self.height * self.width


def token_positions(grid: Grid) -> np.ndarray:
    """(N, 3) int32 (frame, row, column) of each token, raster order n = (f*Hp + h)*Wp + w."""
    f, h, w = np.meshgrid(np.arange(grid.frames), np.arange(grid.height),
                          np.arange(grid.width), indexing="ij")
    return np.stack([f.ravel(), h.ravel(), w.ravel()], axis=1).astype(np.int32)


def group_sizes(N: int, fracs) -> list[int]:
    """Group sizes n_k = floor(frac_k * N) for k >= 2; group 1 takes the remainder."""
    sizes = [int(np.floor(fr * N)) for fr in fracs[1:]]
    return [N - sum(sizes)] + sizes


# ---------------------------------------------------------------- draws

def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(seed: int, shape, scale: float = 1.0, bf16: bool = False) -> np.ndarray:
    a = (_rng(seed).standard_normal(size=shape, dtype=np.float32) * np.float32(scale)).astype(np.float32)
    return round_bf16(a) if bf16 else a


@dataclass
class BlockWeights:
    """One DiT block's parameters, float32 arrays ([out, in] layout for matrices).

    Matrices are bf16-representable when the block is bf16.  Vectors (biases,
    gains, modulation) stay float32 in both precisions.
    """
    w_qkv: np.ndarray          # (3D, D): rows [0,D) q, [D,2D) k, [2D,3D) v
    b_qkv: np.ndarray          # (3D,)
    g_q: np.ndarray            # (D,) q RMSNorm gain
    g_k: np.ndarray            # (D,) k RMSNorm gain
    w_o: np.ndarray            # (D, D)
    b_o: np.ndarray            # (D,)
    w_1: np.ndarray            # (F, D)
    b_1: np.ndarray            # (F,)
    w_2: np.ndarray            # (D, F)
    b_2: np.ndarray            # (D,)
    mod: np.ndarray            # (6, D): shift/scale/gate for attention, then for the FFN
    # cross-attention (None when the block has none)
    ln_c_g: np.ndarray | None = None    # (D,) affine LayerNorm before cross-attention
    ln_c_b: np.ndarray | None = None
    w_q2: np.ndarray | None = None      # (D, D)
    b_q2: np.ndarray | None = None
    g_q2: np.ndarray | None = None
    w_kv2: np.ndarray | None = None     # (2D, D): rows [0,D) k, [D,2D) v
    b_kv2: np.ndarray | None = None
    g_k2: np.ndarray | None = None
    w_o2: np.ndarray | None = None
    b_o2: np.ndarray | None = None
    shape: BlockShape | None = field(default=None, repr=False)


def block_weights(seed: int, shape: BlockShape, bf16: bool, std: float = 0.02) -> BlockWeights:
    D, F = shape.D, shape.F
    s = seed * 64
    z = lambda n: np.zeros(n, np.float32)
    one = lambda n: np.ones(n, np.float32)
    bw = BlockWeights(
        w_qkv=normal(s + 0, (3 * D, D), std, bf16), b_qkv=z(3 * D), g_q=one(D), g_k=one(D),
        w_o=normal(s + 1, (D, D), std, bf16), b_o=z(D),
        w_1=normal(s + 2, (F, D), std, bf16), b_1=z(F),
        w_2=normal(s + 3, (D, F), std, bf16), b_2=z(D),
        mod=normal(s + 4, (6, D), std, False), shape=shape)
    if shape.cross:
        bw.ln_c_g, bw.ln_c_b = one(D), z(D)
        bw.w_q2, bw.b_q2, bw.g_q2 = normal(s + 5, (D, D), std, bf16), z(D), one(D)
        bw.w_kv2, bw.b_kv2, bw.g_k2 = normal(s + 6, (2 * D, D), std, bf16), z(2 * D), one(D)
        bw.w_o2, bw.b_o2 = normal(s + 7, (D, D), std, bf16), z(D)
    return bw


def perturb_vectors(bw: BlockWeights, seed: int, std: float = 0.1) -> BlockWeights:
    """Give biases and gains non-trivial values (zero/one defaults hide dropped terms)."""
    r = _rng(seed)
    for name in ("b_qkv", "g_q", "g_k", "b_o", "b_1", "b_2", "ln_c_g", "ln_c_b", "b_q2",
                 "g_q2", "b_kv2", "g_k2", "b_o2"):
        a = getattr(bw, name)
        if a is None:
            continue
        base = 1.0 if name.startswith(("g_", "ln_c_g")) else 0.0
        setattr(bw, name, (base + std * r.standard_normal(a.shape)).astype(np.float32))
    bw.mod = (bw.mod + std * r.standard_normal(bw.mod.shape)).astype(np.float32)
    return bw


@dataclass
class PatchModelWeights:
    """Patch-embedding and output head around a stack of blocks (C latent channels per token)."""
    w_in: np.ndarray     # (D, C)
    b_in: np.ndarray     # (D,)
    head_mod: np.ndarray  # (2, D): shift, scale of the head's LayerNorm
    w_out: np.ndarray    # (C, D)
    b_out: np.ndarray    # (C,)
    blocks: list


def patch_model_weights(seed: int, shape: BlockShape, C: int, n_blocks: int, bf16: bool,
                        std: float = 0.02) -> PatchModelWeights:
    s = 100_000 + seed * 1024
    return PatchModelWeights(
        w_in=normal(s + 0, (shape.D, C), std, bf16), b_in=np.zeros(shape.D, np.float32),
        head_mod=normal(s + 1, (2, shape.D), std, False),
        w_out=normal(s + 2, (C, shape.D), std, bf16), b_out=np.zeros(C, np.float32),
        blocks=[block_weights(s + 8 + b, shape, bf16, std) for b in range(n_blocks)])


# ---------------------------------------------------------------- draws on the device

def device_normal(gen, shape, scale: float, bf16: bool, device):
    """N(0, scale^2) drawn on the device by torch's seeded generator `gen`; bf16 (rounded to
    nearest even) or float32."""
    import torch
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    t.mul_(scale)
    return t.to(torch.bfloat16) if bf16 else t


def block_weights_on_device(seed: int, shape: BlockShape, bf16: bool, device, std: float = 0.02) -> BlockWeights:
    """The recipe of block_weights drawn on the device (torch tensors; other values than the
    numpy draws of the same seed).  For measurements, where only shapes and distributions
    matter and drawing hundreds of millions of values on the host would take minutes."""
    import torch
    D, F = shape.D, shape.F
    gen = torch.Generator(device=device)
    gen.manual_seed(1_000_003 * (seed + 1))
    z = lambda n: torch.zeros(n, dtype=torch.float32, device=device)
    one = lambda n: torch.ones(n, dtype=torch.float32, device=device)
    nrm = lambda shp, b: device_normal(gen, shp, std, b, device)
    bw = BlockWeights(
        w_qkv=nrm((3 * D, D), bf16), b_qkv=z(3 * D), g_q=one(D), g_k=one(D),
        w_o=nrm((D, D), bf16), b_o=z(D), w_1=nrm((F, D), bf16), b_1=z(F),
        w_2=nrm((D, F), bf16), b_2=z(D), mod=nrm((6, D), False), shape=shape)
    if shape.cross:
        bw.ln_c_g, bw.ln_c_b = one(D), z(D)
        bw.w_q2, bw.b_q2, bw.g_q2 = nrm((D, D), bf16), z(D), one(D)
        bw.w_kv2, bw.b_kv2, bw.g_k2 = nrm((2 * D, D), bf16), z(2 * D), one(D)
        bw.w_o2, bw.b_o2 = nrm((D, D), bf16), z(D)
    return bw


def patch_model_weights_on_device(seed: int, shape: BlockShape, C: int, n_blocks: int, bf16: bool, device,
                                  std: float = 0.02) -> PatchModelWeights:
    """patch_model_weights drawn on the device (see block_weights_on_device)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(2_000_003 * (seed + 1))
    return PatchModelWeights(
        w_in=device_normal(gen, (shape.D, C), std, bf16, device),
        b_in=torch.zeros(shape.D, dtype=torch.float32, device=device),
        head_mod=device_normal(gen, (2, shape.D), std, False, device),
        w_out=device_normal(gen, (C, shape.D), std, bf16, device),
        b_out=torch.zeros(C, dtype=torch.float32, device=device),
        blocks=[block_weights_on_device(100 * seed + 8 + b, shape, bf16, device, std) for b in range(n_blocks)])


# ---------------------------------------------------------------- named workloads

@dataclass(frozen=True)
class LoopWorkload:
    name: str
    grid: Grid
    shape: BlockShape
    C: int                 # latent channels per token (= D for single-block workloads)
    n_blocks: int
    T: int
    budgets: tuple
    fracs: tuple
    m: int
    sigma_kind: int        # 0 linear 1 -> 0, 1 shifted
    shift: float
    bf16: bool
    seed: int


# Tiny single-layer fp32 loop: 4x16x16 tokens, D=256, 2 heads, T=8, budgets {8,4}, m=1, linear sigma.
TINY_FP32 = LoopWorkload("tiny-fp32-N1024-D256", Grid(4, 16, 16), BlockShape(256, 2, 1024, False),
                         C=256, n_blocks=1, T=8, budgets=(8, 4), fracs=(0.5, 0.5), m=1,
                         sigma_kind=0, shift=1.0, bf16=False, seed=1)

# Wan-1.3B-shaped block: 21x30x52 tokens, D=1536, 12 heads, FFN 8960, 512-token context.
WAN13_GRID = Grid(21, 30, 52)
WAN13_BLOCK = BlockShape(1536, 12, 8960, True, 512)
# Wan-14B-shaped block: same token grid, D=5120, 40 heads, FFN 13824, no context.
WAN14_BLOCK = BlockShape(5120, 40, 13824, False)

# Wan-1.3B-shaped 30-block loop (latent 16 channels, 1x2x2 patches -> C=64), T=40, budgets
# {40,20,10} sized 25/25/50 %, m=4, shifted sigma (shift 5).
WAN13_LOOP = LoopWorkload("wan1.3b-loop-N32760", WAN13_GRID, WAN13_BLOCK, C=64, n_blocks=30, T=40,
                          budgets=(40, 20, 10), fracs=(0.25, 0.25, 0.5), m=4, sigma_kind=1,
                          shift=5.0, bf16=True, seed=3)
# Reduced stand-in of the loop with the same T/K/s/m/shift that the oracle runs in full.
WAN13_LOOP_SMALL = LoopWorkload("wan-loop-standin-N128", Grid(1, 8, 16), BlockShape(256, 2, 1024, True, 64),
                                C=64, n_blocks=3, T=40, budgets=(40, 20, 10), fracs=(0.25, 0.25, 0.5),
                                m=4, sigma_kind=1, shift=5.0, bf16=True, seed=3)

SWEEP_GRIDS = {8190: Grid(21, 15, 26), 32760: WAN13_GRID, 75600: Grid(21, 45, 80)}


def active_fraction_rows(N: int, frac: float) -> int:
    return int(round(frac * N))


def contiguous_mask(seed: int, N: int, M: int) -> np.ndarray:
    """Ascending indices of the range [o, o+M) (mod N) at a seeded offset o."""
    o = int(_rng(seed).integers(0, N))
    return np.sort((o + np.arange(M)) % N).astype(np.int32)


def scattered_mask(seed: int, N: int, M: int) -> np.ndarray:
    """Ascending indices of a uniform random M-subset of [0, N)."""
    return np.sort(_rng(seed).permutation(N)[:M]).astype(np.int32)

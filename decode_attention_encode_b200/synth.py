"""Seeded synthetic inputs for the LLA decode and encode paths.

This module draws random numbers and names workload shapes. It holds none of
the method's arithmetic (no reconstruction, attention, absorption or
encoding), so the CUDA path and the test oracle can both take their inputs
from it.

Value recipes (the pages publish no data for this path; these stand in for a
looped model's latent cache):
  * latents z ~ N(0, 1), optionally with a decaying spectrum: coordinate i
    (1-based) is scaled by 1/i, the spectrum of SVD coordinates whose singular
    values fall off as 1/i;
  * decoders: QR-orthonormalised Gaussian blocks, orthonormal columns when
    r <= d_h and orthonormal rows when r > d_h;
  * queries q ~ N(0, 1/d_h);
  * stacked per-loop K/V for the latent write ~ N(0, 1).
All draws use torch generators seeded explicitly, on the device the caller
names, so a CUDA-side draw and a CPU re-draw with the same seed differ; tests
therefore copy device draws to the host instead of re-drawing them.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, seed: int, device="cpu", std: float = 1.0,
           dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) draws in fp32, then cast to ``dtype``."""
    t = torch.randn(tuple(shape), generator=_gen(seed, device), device=device,
                    dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def latents(shape, seed: int, device="cpu", decay: bool = False,
            dtype=torch.bfloat16) -> torch.Tensor:
    """Latent draws z ~ N(0, 1) over the last axis; with ``decay`` coordinate
    i (1-based) is scaled by 1/i."""
    t = torch.randn(tuple(shape), generator=_gen(seed, device), device=device,
                    dtype=torch.float32)
    if decay:
        r = shape[-1]
        t.mul_(1.0 / torch.arange(1, r + 1, device=device, dtype=torch.float32))
    return t.to(dtype)


def orthonormal(n: int, rows: int, cols: int, seed: int, device="cpu",
                dtype=torch.float32) -> torch.Tensor:
    """``n`` matrices of shape [rows, cols]: orthonormal columns when
    rows >= cols, orthonormal rows otherwise (QR of a Gaussian draw, with the
    sign fixed by R's diagonal)."""
    tall = rows >= cols
    a, b = (rows, cols) if tall else (cols, rows)
    g = torch.randn((n, a, b), generator=_gen(seed, device), device=device,
                    dtype=torch.float64 if device == "cpu" else torch.float32)
    qm, rm = torch.linalg.qr(g)
    sign = torch.sign(torch.diagonal(rm, dim1=-2, dim2=-1))
    sign[sign == 0] = 1
    qm = qm * sign.unsqueeze(-2)
    if not tall:
        qm = qm.transpose(-1, -2)
    return qm.contiguous().to(dtype)


def queries(shape, d_h: int, seed: int, device="cpu") -> torch.Tensor:
    """q ~ N(0, 1/d_h), fp32."""
    return normal(shape, seed, device, std=d_h ** -0.5)


def ragged_lengths(B: int, n_mean: int, seed: int, spread: float = 0.5) -> np.ndarray:
    """Seeded per-sequence lengths, uniform in [(1 - spread) n, (1 + spread) n]
    (a serving batch's length mix), at least 1. int32."""
    r = np.random.default_rng(seed)
    lo = max(1, int(round((1.0 - spread) * n_mean)))
    hi = max(lo, int(round((1.0 + spread) * n_mean)))
    return r.integers(lo, hi + 1, size=B).astype(np.int32)


def page_table(lens, page_size: int, seed: int, spare: int = 0, max_blocks: int = 0):
    """A shuffled page assignment for sequences of the given lengths: every
    sequence gets ceil(n / page_size) distinct pages drawn from one pool in a
    seeded random order. Unused table entries are -1. Returns (block_table
    [B, max_blocks] int32, num_pages) with num_pages = pages used + spare."""
    lens = np.asarray(lens, dtype=np.int64)
    need = (lens + page_size - 1) // page_size
    max_blocks = max(int(need.max(initial=0)), max_blocks, 1)
    num_pages = int(need.sum()) + spare
    order = np.random.default_rng(seed).permutation(max(num_pages, 1))
    bt = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    k = 0
    for b, nb in enumerate(need):
        bt[b, :nb] = order[k:k + nb]
        k += nb
    return bt, max(num_pages, 1)


# --------------------------------------------------------------------------
# Workload shapes
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class DecodeConfig:
    """One decode workload. ``two_d`` selects LLA-2D (one latent per token
    and layer shared by all heads). ``page_size`` > 0 selects a paged store
    whose sequences have seeded ragged lengths with mean ``N`` (uniform
    within +-``spread`` N). ``d_r`` > 0 adds a decoupled rotary branch of
    that width to every key row."""
    name: str
    L: int           # layers (D in the paper)
    T: int           # loops
    H: int           # heads
    d_h: int         # head width
    r_k: int
    r_v: int
    B: int           # batch
    N: int           # cached tokens per sequence
    dtype: str       # latent storage: "f32" or "bf16"
    decay: bool      # decaying latent spectrum
    two_d: bool = False
    seed: int = 0
    note: str = field(default="", compare=False)
    page_size: int = 0
    spread: float = 0.0
    d_r: int = 0

    @property
    def esz(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def lengths(self) -> np.ndarray:
        """Cached tokens of each sequence (int32)."""
        if self.page_size:
            return ragged_lengths(self.B, self.N, self.seed + 77, self.spread)
        return np.full(self.B, self.N, dtype=np.int32)

    def tokens(self) -> int:
        """Cached tokens attended per (layer, loop) step, all sequences."""
        return int(self.lengths().sum())

    def store_bytes_per_layer(self) -> int:
        per_tok = (self.r_k + self.d_r + self.r_v) * self.esz * (1 if self.two_d else self.H)
        return self.tokens() * per_tok

    def step_bytes(self) -> int:
        """Algorithmic bytes of one (layer, loop) step: every cached latent
        of one layer is read once."""
        return self.store_bytes_per_layer()


C1 = DecodeConfig("tiny_fp32", L=1, T=4, H=2, d_h=16, r_k=8, r_v=8, B=1, N=64,
                  dtype="f32", decay=False)
C2 = DecodeConfig("perhead_4x", L=24, T=4, H=16, d_h=128, r_k=128, r_v=128, B=64,
                  N=4096, dtype="bf16", decay=True)
C3 = DecodeConfig("perhead_21x", L=24, T=4, H=16, d_h=128, r_k=24, r_v=24, B=768,
                  N=4096, dtype="bf16", decay=True)
C4 = DecodeConfig("lla2d_32x", L=24, T=4, H=16, d_h=128, r_k=256, r_v=256, B=256,
                  N=8192, dtype="bf16", decay=True, two_d=True)
C5_DECODE = DecodeConfig("perhead_32x_long", L=24, T=4, H=16, d_h=128, r_k=16, r_v=16,
                         B=32, N=32768, dtype="bf16", decay=False)
# the 4x geometry as a serving batch: 64 sequences of 2048..6144 tokens in a
# pool of 64-token pages
C2_PAGED = DecodeConfig("perhead_4x_paged", L=24, T=4, H=16, d_h=128, r_k=128, r_v=128, B=64,
                        N=4096, dtype="bf16", decay=True, page_size=64, spread=0.5)


@dataclass(frozen=True)
class EncodeConfig:
    """Latent-write workload: ``N`` tokens of ``G`` groups (heads) for each of
    ``L`` layers and both axes; x is [T][N][G][d_loop] per (layer, axis)."""
    name: str
    L: int
    T: int
    G: int
    d_loop: int
    r: int
    N: int
    n_cal: int
    seed: int = 0

    def in_bytes(self) -> int:
        return 2 * self.L * self.T * self.N * self.G * self.d_loop * 2

    def out_bytes(self) -> int:
        return 2 * self.L * self.G * self.N * self.r * 2

    def flops(self) -> int:
        return 2 * self.L * 2 * self.G * self.N * self.T * self.d_loop * self.r


C5_ENCODE = EncodeConfig("encode_32x", L=24, T=4, G=16, d_loop=128, r=16, N=32768,
                         n_cal=2048)
# the LLA-2D latent write of a 32768-token prefill: each token's whole stack
# (T loops x 16 heads x 128 channels = 8192) to one r = 256 latent per
# (layer, axis); a tensor-bound GEMM at about 250 flop/B
C4_ENCODE = EncodeConfig("encode2d_32x", L=24, T=4, G=1, d_loop=2048, r=256, N=32768,
                         n_cal=512)
ENCODE_CONFIGS = {c.name: c for c in (C5_ENCODE, C4_ENCODE)}

# the 4x geometry with a 64-wide decoupled rotary branch on the key side
C2_ROPE = DecodeConfig("perhead_4x_rope", L=24, T=4, H=16, d_h=128, r_k=128, r_v=128, B=64,
                       N=4096, dtype="bf16", decay=True, d_r=64)
# the 32x LLA-2D geometry as a serving batch: 256 sequences of 4096..12288
# tokens in a pool of 256-token pages
C4_PAGED = DecodeConfig("lla2d_32x_paged", L=24, T=4, H=16, d_h=128, r_k=256, r_v=256, B=256,
                        N=8192, dtype="bf16", decay=True, two_d=True, page_size=256, spread=0.5)
# the same batch in 64-token pages: every 128-token tile spans two pages
C4_PAGED64 = DecodeConfig("lla2d_32x_paged64", L=24, T=4, H=16, d_h=128, r_k=256, r_v=256, B=256,
                          N=8192, dtype="bf16", decay=True, two_d=True, page_size=64, spread=0.5)
# the 32x LLA-2D geometry with a 64-wide rotary key shared by every head:
# key rows [256 latent | 64 rotary], 320 wide
C4_ROPE = DecodeConfig("lla2d_32x_rope", L=24, T=4, H=16, d_h=128, r_k=256, r_v=256, B=256,
                       N=8192, dtype="bf16", decay=True, two_d=True, d_r=64)
DECODE_CONFIGS = {c.name: c for c in (C1, C2, C3, C4, C5_DECODE, C2_PAGED, C2_ROPE, C4_PAGED,
                                      C4_PAGED64, C4_ROPE)}


def sample_units(B: int, L: int, T: int, H: int, n_random: int = 32, seed: int = 0):
    """The fixed sample of (b, layer, loop, h) decode units on which the
    CPU baseline times the oracle: ``n_random`` seeded-random units, then the
    16 corners (each index at its first or last value), without repeats."""
    r = np.random.default_rng(seed)
    units = [(int(r.integers(B)), int(r.integers(L)), int(r.integers(T)), int(r.integers(H)))
             for _ in range(n_random)]
    for b in (0, B - 1):
        for l in (0, L - 1):
            for t in (0, T - 1):
                for h in (0, H - 1):
                    units.append((b, l, t, h))
    seen, out = set(), []
    for u in units:
        if u not in seen:
            seen.add(u)
            out.append(u)
    return out

"""The error bound the tensor-core absorb and merge rely on (host-side
check of the arithmetic, no GPU).

Those kernels split every fp32 operand x into hi = bf16(x) and
lo = bf16(x - hi) and form a product as hi.hi + hi.lo + lo.hi. With bf16's
8-bit significand |x - hi| <= 2^-8 |x| and |x - hi - lo| <= 2^-16 |x|, so
the three terms reproduce x y within 3 * 2^-16 |x y|. The check rounds with
torch's bf16 conversion (round to nearest even, as the kernels' conversion
instructions do) and measures the gap in fp64 over magnitudes spanning the
fp32 normal range."""

import numpy as np
import torch


def split(x32: torch.Tensor):
    hi = x32.to(torch.bfloat16).to(torch.float32)
    lo = (x32 - hi).to(torch.bfloat16).to(torch.float32)  # x - hi is exact in fp32
    return hi.double(), lo.double()


def test_three_term_split_product_bound():
    rng = np.random.default_rng(0)
    n = 200_000
    mant = rng.uniform(-2.0, 2.0, size=(2, n))
    expo = rng.integers(-60, 60, size=(2, n))
    x = torch.from_numpy(mant[0] * 2.0 ** expo[0]).float()
    y = torch.from_numpy(mant[1] * 2.0 ** expo[1]).float()
    hx, lx = split(x)
    hy, ly = split(y)
    exact = x.double() * y.double()
    approx = hx * hy + hx * ly + lx * hy
    rel = ((approx - exact).abs() / exact.abs().clamp_min(1e-300)).max().item()
    assert rel <= 3 * 2.0 ** -16, rel
    # the residue of the split itself
    res = ((x.double() - hx - lx).abs() / x.double().abs().clamp_min(1e-300)).max().item()
    assert res <= 2.0 ** -16, res


def test_split_dot_product_matches_fp64_far_inside_the_bf16_rounding():
    # a q' element: a 128-term dot product of split operands against fp64
    rng = np.random.default_rng(1)
    q = torch.from_numpy(rng.normal(size=(512, 128))).float()
    w = torch.from_numpy(rng.normal(size=(128,)) / np.sqrt(128)).float()
    hq, lq = split(q)
    hw, lw = split(w)
    approx = hq @ hw + hq @ lw + lq @ hw
    exact = q.double() @ w.double()
    scale = (q.double().abs() @ w.double().abs())
    assert ((approx - exact).abs() / scale).max().item() <= 3 * 2.0 ** -16
    # against plain bf16 operands the split is far more accurate
    plain = hq @ hw
    assert ((approx - exact).abs().max() < (plain - exact).abs().max() / 100).item()

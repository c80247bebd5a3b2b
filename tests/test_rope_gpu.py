"""GPU parity of the per-head decode with the decoupled rotary branch
(lla_decode_attn_rope) against the fp64 oracle, through the C ABI.

Key rows hold [latent | rotated rotary key]; the rotary query is this loop's
rotated query. Cases: both latent types, several (r_k, d_r) splits
including ones whose row segment counts differ from the value rows, ragged
tails, a rotary-dominated sharp softmax, and the 4x geometry with a 64-wide
rotary branch on sampled units."""

import math

import numpy as np
import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import synth
from lla_cases import TOL_BF16_REL, TOL_F32_ABS, sample_units, to_f64

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32


def make_rope_inputs(B, H, d_h, N, r_k, d_r, r_v, dtype, n_cap=None, mu=False, seed=0,
                     rope_scale=1.0):
    n_cap = N if n_cap is None else n_cap
    zk = synth.latents((B, H, n_cap, r_k + d_r), seed + 1, "cuda", decay=False, dtype=dtype)
    zv = synth.latents((B, H, n_cap, r_v), seed + 2, "cuda", decay=True, dtype=dtype)
    dk = synth.orthonormal(H, d_h, r_k, seed + 3, "cuda")
    dv = synth.orthonormal(H, d_h, r_v, seed + 4, "cuda")
    q = synth.queries((B, H, d_h), d_h, seed + 5, "cuda")
    q_rope = synth.queries((B, H, d_r), d_r, seed + 6, "cuda") * rope_scale
    mu_k = synth.normal((H, d_h), seed + 7, "cuda") if mu else None
    mu_v = synth.normal((H, d_h), seed + 8, "cuda") if mu else None
    return dict(q=q, q_rope=q_rope, zk=zk, zv=zv, dk=dk, dv=dv, mu_k=mu_k, mu_v=mu_v, N=N)


def check(inp, dtype, units=None):
    import oracle  # test infrastructure only
    out, lse = lla.lla_decode_attn_rope(inp["q"], inp["q_rope"], inp["zk"], inp["zv"], inp["dk"],
                                        inp["dv"], N=inp["N"], mu_k_t=inp["mu_k"],
                                        mu_v_t=inp["mu_v"])
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    B, H, _ = inp["q"].shape
    units = [(b, h) for b in range(B) for h in range(H)] if units is None else units
    bs = torch.tensor([u[0] for u in units], device="cuda")
    hs = torch.tensor([u[1] for u in units], device="cuda")
    N = inp["N"]
    opt = lambda t: None if t is None else to_f64(t)
    ref_out, ref_lse = oracle.lla_decode_rope(
        to_f64(inp["q"]), to_f64(inp["q_rope"]), to_f64(inp["zk"][:, :, :N]),
        to_f64(inp["zv"][:, :, :N]), to_f64(inp["dk"]), to_f64(inp["dv"]), opt(inp["mu_k"]),
        opt(inp["mu_v"]), units=units)
    o = to_f64(out)[[u[0] for u in units], [u[1] for u in units]]
    l = to_f64(lse)[[u[0] for u in units], [u[1] for u in units]]
    diff = np.abs(o - ref_out).max()
    if dtype == F32:
        assert diff <= TOL_F32_ABS, diff
    else:
        rel = diff / np.abs(ref_out).max()
        assert rel <= TOL_BF16_REL, rel
        assert rel < 1e-4, f"relative error {rel:.2e} above fp32 accumulation level"
    assert np.abs(l - ref_lse).max() < 1e-3


@pytest.mark.parametrize("r_k, d_r, r_v, dtype", [
    (8, 8, 8, F32), (32, 32, 64, F32), (64, 64, 64, F32),
    (16, 8, 24, BF16), (64, 64, 128, BF16), (128, 64, 128, BF16), (96, 32, 160, BF16),
    (192, 64, 256, BF16)])
def test_rank_and_rotary_splits(r_k, d_r, r_v, dtype):
    check(make_rope_inputs(3, 4, 64, 777, r_k, d_r, r_v, dtype, n_cap=800, mu=True, seed=r_k + d_r),
          dtype)


@pytest.mark.parametrize("N", [1, 2, 63, 1000])
def test_context_lengths(N):
    check(make_rope_inputs(2, 3, 32, N, 16, 16, 16, F32, n_cap=N + 3, seed=N), F32)


def test_rotary_branch_dominates_a_sharp_softmax():
    # rotary queries x12: scores are driven by the rotary keys
    check(make_rope_inputs(4, 4, 128, 3000, 64, 64, 64, BF16, seed=5, rope_scale=12.0), BF16)


def test_full_size_4x_geometry_with_64_wide_rotary_branch():
    inp = make_rope_inputs(64, 16, 128, 4096, 128, 64, 128, BF16, seed=0)
    check(inp, BF16, units=sample_units(64, 16))


# ---------------------------------------------------------------------------
# LLA-2D: the key row [latent | rotary key] shared by every head
# ---------------------------------------------------------------------------

def make_2d(B, H, d_h, N, r_k, d_r, r_v, n_cap=None, mu=False, seed=0, rope_scale=1.0):
    n_cap = N if n_cap is None else n_cap
    return dict(
        q=synth.queries((B, H, d_h), d_h, seed + 5, "cuda"),
        q_rope=synth.queries((B, H, d_r), d_r, seed + 6, "cuda") * rope_scale,
        zk=synth.latents((B, n_cap, r_k + d_r), seed + 1, "cuda", decay=False, dtype=BF16),
        zv=synth.latents((B, n_cap, r_v), seed + 2, "cuda", decay=True, dtype=BF16),
        dk=synth.orthonormal(H, d_h, r_k, seed + 3, "cuda"),
        dv=synth.orthonormal(H, d_h, r_v, seed + 4, "cuda"),
        mu_k=synth.normal((H, d_h), seed + 7, "cuda") if mu else None,
        mu_v=synth.normal((H, d_h), seed + 8, "cuda") if mu else None, N=N)


def check_2d(inp, units=None):
    import oracle  # test infrastructure only
    out, lse = lla.lla2d_decode_attn_rope(inp["q"], inp["q_rope"], inp["zk"], inp["zv"],
                                          inp["dk"], inp["dv"], N=inp["N"], mu_k_t=inp["mu_k"],
                                          mu_v_t=inp["mu_v"])
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    B, H, _ = inp["q"].shape
    units = [(b, h) for b in range(B) for h in range(H)] if units is None else units
    N = inp["N"]
    opt = lambda t: None if t is None else to_f64(t)
    ref_out, ref_lse = oracle.lla2d_decode_rope(
        to_f64(inp["q"]), to_f64(inp["q_rope"]), to_f64(inp["zk"][:, :N]),
        to_f64(inp["zv"][:, :N]), to_f64(inp["dk"]), to_f64(inp["dv"]), opt(inp["mu_k"]),
        opt(inp["mu_v"]), units=units)
    bs, hs = [u[0] for u in units], [u[1] for u in units]
    o, l = to_f64(out)[bs, hs], to_f64(lse)[bs, hs]
    rel = np.abs(o - ref_out).max() / np.abs(ref_out).max()
    assert rel <= TOL_BF16_REL, rel
    assert np.abs(l - ref_lse).max() < 2e-2


@pytest.mark.parametrize("r_k, d_r, r_v", [(192, 64, 256), (256, 64, 256), (128, 64, 128),
                                           (320, 64, 128), (64, 64, 256), (96, 32, 160),
                                           (200, 8, 96)])
def test_lla2d_rotary_key_row_widths(r_k, d_r, r_v):
    check_2d(make_2d(3, 16, 128, 1000, r_k, d_r, r_v, n_cap=1030, mu=True, seed=r_k))


@pytest.mark.parametrize("H", [1, 20, 32])
def test_lla2d_rotary_head_counts(H):
    check_2d(make_2d(2, H, 64, 300, 256, 64, 128, seed=H, rope_scale=4.0))


def test_lla2d_rotary_full_size_32x_sampled():
    inp = make_2d(256, 16, 128, 8192, 256, 64, 256, seed=0)
    check_2d(inp, units=sample_units(256, 16))

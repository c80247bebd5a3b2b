"""GPU parity of the LLA-2D absorbed decode (lla2d_decode_attn: tcgen05 score
and value contractions) against the fp64 oracle, through the C ABI.

The kernel feeds the tensor cores bf16 operands: the latents exactly, the
absorbed query q' and the softmax weights rounded to bf16 (RNE), with fp32
accumulation. The gate is the stated bf16 tolerance
max|o_gpu - o_ref| / max|o_ref| <= 2e-2."""

import pytest
import torch

import decode_attention_encode_b200 as lla
from lla_cases import compare, make_decode_inputs, oracle_reference, sample_units

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def run(B, H, d_h, N, r_k, r_v, units=None, **kw):
    inp = make_decode_inputs(B, H, d_h, N, r_k, r_v, BF16, two_d=True, **kw)
    out, lse = lla.lla2d_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N,
                                     mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"])
    torch.cuda.synchronize()
    if units is None:
        units = [(b, h) for b in range(B) for h in range(H)]
    ref_out, ref_lse = oracle_reference(inp, units, two_d=True)
    err, lse_err = compare(out, lse, units, ref_out, ref_lse, BF16)
    assert lse_err < 5e-2, f"lse error {lse_err:.2e}"
    assert lla.device_status() == 0
    return err


def test_small_ragged_with_means():
    run(3, 16, 128, 300, 256, 256, n_cap=320, mu=True, decay=True)


@pytest.mark.parametrize("H", [1, 8, 16, 20, 32])
def test_head_counts(H):
    run(2, H, 64, 400, 128, 128, mu=True, seed=H)


@pytest.mark.parametrize("d_h", [16, 32, 96, 256])
def test_head_widths(d_h):
    # d_h of 64 and 128 form Q' on the tensor cores; the others take the
    # CUDA-core absorb, which writes the same swizzled operand
    run(3, 16, d_h, 300, 128, 128, mu=True, seed=d_h)


@pytest.mark.parametrize("r_k, r_v", [(64, 128), (128, 256), (192, 128), (256, 128), (256, 256)])
def test_ranks(r_k, r_v):
    run(2, 16, 128, 333, r_k, r_v, seed=r_k + r_v)


@pytest.mark.parametrize("r_k, r_v", [(96, 160), (192, 192), (8, 8), (24, 40), (136, 200),
                                      (64, 64), (16, 256), (256, 72)])
def test_ranks_padded_to_whole_boxes_and_tiles(r_k, r_v):
    # ranks that are not whole 64-column boxes (K) or 128-row MMA tiles (V):
    # the tensor maps fill the missing columns with zeros and the records
    # keep only the r_v real rows; 96/160 is the paper's asymmetric split
    run(3, 16, 128, 333, r_k, r_v, n_cap=340, mu=True, decay=True, seed=r_k * 7 + r_v)


def test_full_size_asymmetric_96_160_sampled():
    # the 32x geometry with the paper's 96/160 key/value split
    err = run(256, 16, 128, 8192, 96, 160, units=sample_units(256, 16), decay=True, seed=2)
    print(f"lla2d 96/160 full size: rel err {err:.2e}")


@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 1000])
def test_context_lengths(N):
    run(2, 16, 128, N, 256, 256, n_cap=N + 3, mu=True, seed=N)


@pytest.mark.parametrize("B, N", [(37, 1000), (300, 200), (5, 40000), (600, 100), (150, 700)])
def test_sequences_split_across_ctas(B, N):
    run(B, 16, 128, N, 256, 256, units=sample_units(B, 16), decay=True, seed=B)


def test_sharp_softmax_rescales_mid_sequence():
    # Queries x8 and, per (b, h), one planted latent aligned with that head's
    # absorbed query placed after the first tile, so the running maximum
    # jumps while value sums are already accumulated.
    B, H, d_h, N, r = 3, 16, 128, 1200, 256
    inp = make_decode_inputs(B, H, d_h, N, r, r, BF16, two_d=True, q_scale=8.0, seed=9)
    qp = torch.einsum("hdr,bhd->bhr", inp["dk"], inp["q"])
    g = torch.Generator().manual_seed(4)
    for b in range(B):
        pos = 200 + torch.randperm(N - 200, generator=g)[:H]
        for h in range(H):
            inp["zk"][b, pos[h]] = (qp[b, h] / qp[b, h].norm() * 10.0).to(BF16)
    out, lse = lla.lla2d_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N)
    torch.cuda.synchronize()
    units = [(b, h) for b in range(B) for h in range(H)]
    ref_out, ref_lse = oracle_reference(inp, units, two_d=True)
    compare(out, lse, units, ref_out, ref_lse, BF16)


def test_full_size_sampled():
    # LLA-2D workload: H=16, d_h=128, r_k=r_v=256, batch 256, context 8192
    err = run(256, 16, 128, 8192, 256, 256, units=sample_units(256, 16), decay=True, seed=0)
    print(f"lla2d full size: rel err {err:.2e}")


def test_rows_beyond_N_are_never_read():
    B, H, d_h, N, n_cap = 3, 16, 128, 300, 384
    inp = make_decode_inputs(B, H, d_h, N, 256, 256, BF16, two_d=True, n_cap=n_cap, mu=True, seed=13)
    inp["zk"][:, N:] = float("nan")
    inp["zv"][:, N:] = float("nan")
    out, lse = lla.lla2d_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N,
                                     mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"])
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    units = [(b, h) for b in range(B) for h in range(H)]
    ref_out, ref_lse = oracle_reference(inp, units, two_d=True)
    compare(out, lse, units, ref_out, ref_lse, BF16)

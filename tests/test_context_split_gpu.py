"""GPU parity of the context merge (lla_merge_attn): one long sequence batch
is split into parts along the context, each part decoded by the library, the
parts merged on the device, and the result compared with the fp64 oracle
over the whole context and with the unsplit call. Also: empty parts and an
all-empty unit, and the LLA-2D path."""

import numpy as np
import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import synth
from decode_attention_encode_b200.context_split import shard_range
from lla_cases import TOL_BF16_REL, make_decode_inputs, oracle_reference, sample_units, to_f64

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


@pytest.mark.parametrize("parts", [2, 3, 8])
def test_per_head_decode_split_over_the_context(parts):
    B, H, d_h, N, r = 4, 8, 128, 20000, 64
    inp = make_decode_inputs(B, H, d_h, N, r, r, BF16, mu=True, decay=True, seed=parts)
    outs, lses = [], []
    for p in range(parts):
        a, b = shard_range(N, parts, p)
        zk = inp["zk"][:, :, a:b].contiguous()
        zv = inp["zv"][:, :, a:b].contiguous()
        o, l = lla.lla_decode_attn(inp["q"], zk, zv, inp["dk"], inp["dv"], mu_k_t=inp["mu_k"],
                                   mu_v_t=inp["mu_v"])
        outs.append(o)
        lses.append(l)
    out, lse = lla.lla_merge_attn(torch.stack(outs), torch.stack(lses))
    whole_o, whole_l = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"],
                                           mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"])
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    units = [(b, h) for b in range(B) for h in range(H)]
    ref_o, ref_l = oracle_reference(inp, units)
    got = to_f64(out).reshape(B * H, d_h)
    rel = np.abs(got - ref_o).max() / np.abs(ref_o).max()
    assert rel < 1e-4, rel
    assert np.abs(to_f64(lse).reshape(-1) - ref_l).max() < 1e-3
    assert (out - whole_o).abs().max().item() < 1e-4 * whole_o.abs().max().item()


def test_empty_parts_and_all_empty_units():
    U, d = 5, 16
    outs = torch.randn(3, U, d, device="cuda")
    lses = torch.randn(3, U, device="cuda")
    lses[1] = float("-inf")            # part 1 holds no token of any unit
    outs[1] = float("nan")             # and its out is never read as a weight > 0
    lses[:, 4] = float("-inf")         # unit 4: no token anywhere
    out, lse = lla.lla_merge_attn(outs, lses)
    torch.cuda.synchronize()
    import oracle
    ref_o, ref_l = oracle.merge_attn(to_f64(outs[[0, 2]]), to_f64(lses[[0, 2]]))
    np.testing.assert_allclose(to_f64(out)[:4], ref_o[:4], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(to_f64(lse)[:4], ref_l[:4], rtol=1e-6, atol=1e-6)
    assert torch.all(out[4] == 0) and torch.isneginf(lse[4])


def test_lla2d_split_over_the_context():
    B, H, d_h, N, r = 8, 16, 128, 6000, 256
    inp = make_decode_inputs(B, H, d_h, N, r, r, BF16, two_d=True, decay=True, seed=3)
    outs, lses = [], []
    for p in range(4):
        a, b = shard_range(N, 4, p)
        o, l = lla.lla2d_decode_attn(inp["q"], inp["zk"][:, a:b].contiguous(),
                                     inp["zv"][:, a:b].contiguous(), inp["dk"], inp["dv"])
        outs.append(o)
        lses.append(l)
    out, lse = lla.lla_merge_attn(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    units = sample_units(B, H)
    ref_o, ref_l = oracle_reference(inp, units, two_d=True)
    got = to_f64(out)[[u[0] for u in units], [u[1] for u in units]]
    rel = np.abs(got - ref_o).max() / np.abs(ref_o).max()
    assert rel <= TOL_BF16_REL, rel

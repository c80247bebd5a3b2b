"""The decode entry point for callers that cannot allocate device memory
(lla_decode_attn_noalloc), checked against the workspace entry point
(lla_decode_attn) through the C ABI.

Such callers (a plugin inside an engine that owns all device memory, or code
that must not call cudaMalloc after start-up) get the same kernels running
on a fixed scratch array inside the library. Both calls run the same
kernels with the same launch plan on the same inputs, so their outputs must
agree bit for bit; a scratch-offset or layout slip would not. This file runs
last so that a failure here does not hide the other GPU tests. The rejection
of shapes beyond the scratch is checked without a device, in test_abi.py."""

import pytest
import torch

import decode_attention_encode_b200 as lla
from lla_cases import make_decode_inputs

pytestmark = pytest.mark.gpu


def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    # the 4x per-head step: 64 sequences x 16 heads x 4096 tokens, r = 128
    inp = make_decode_inputs(64, 16, 128, 4096, 128, 128, torch.bfloat16, mu=True, decay=True,
                             seed=21)
    args = (inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"])
    kw = dict(mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"])
    ref_out, ref_lse = lla.lla_decode_attn(*args, **kw)
    torch.cuda.synchronize()
    for _ in range(2):
        out, lse = lla.lla_decode_attn_noalloc(*args, **kw)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        assert torch.equal(lse, ref_lse)
    assert lla.device_status() == 0


def test_noalloc_matches_on_a_second_shape_after_the_first():
    # the scratch keeps the previous call's contents: a different plan (fewer
    # streaming pieces, another rank) must not read any of it
    inp = make_decode_inputs(3, 5, 64, 777, 24, 40, torch.bfloat16, mu=False, seed=22)
    args = (inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"])
    ref_out, ref_lse = lla.lla_decode_attn(*args)
    out, lse = lla.lla_decode_attn_noalloc(*args)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)
    assert lla.device_status() == 0

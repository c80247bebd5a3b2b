"""The decode entry point for callers that cannot allocate device memory
(lla_decode_attn_noalloc), checked against the workspace entry point
(lla_decode_attn) through the C ABI.

Such callers (a plugin inside an engine that owns all device memory, or code
that must not call cudaMalloc after start-up) get the same kernels running
on a fixed scratch array inside the library. This file runs last so that a
failure here does not hide the other GPU tests."""

import ctypes

import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import _lib
from lla_cases import TOL_BF16_REL, make_decode_inputs

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
        err = ((out - ref_out).abs().max() / ref_out.abs().max()).item()
        assert err <= TOL_BF16_REL, f"relative error {err:.3e}"
        assert (lse - ref_lse).abs().max().item() < 1e-3
    assert lla.device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch_before_launching():
    # 1024 x 16 units with r = 128 need 8 MiB of absorbed queries alone.
    need = lla.lla_decode_attn_workspace(1024, 16, 4096, 128, 128)
    assert need > 4 << 20
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: rejected on the host
    st = lla.lib().lla_decode_attn_noalloc(fake, fake, fake, 1, 1024, 16, 128, 4096, 4096, 128,
                                           128, fake, fake, None, None, 0.1, fake, None, None)
    assert st == _lib.LLA_ERR_WORKSPACE
    assert b"scratch" in lla.lib().lla_last_error()

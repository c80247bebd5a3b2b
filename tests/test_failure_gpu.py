"""The failure path of the bounded device waits, exercised without a fault:
a self-test kernel waits on a barrier nothing arrives at, gives up after a
short limit and reports through the device status word. The context must
stay usable afterwards."""

import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import _lib, synth

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_sets_the_status_and_returns():
    lla.device_status(clear=True)
    stream = torch.cuda.current_stream().cuda_stream
    assert lla.lib().lla_selftest_wait_timeout(20000, stream) == _lib.LLA_OK  # 20 ms
    torch.cuda.synchronize()
    st = lla.device_status(clear=True)
    assert st & _lib.LLA_DEVICE_WAIT_TIMEOUT
    assert lla.device_status() == 0
    # the context is intact: a decode call still runs and reports nothing
    q = synth.queries((1, 2, 16), 16, 1, "cuda")
    zk = synth.latents((1, 2, 64, 8), 2, "cuda", dtype=torch.float32)
    zv = synth.latents((1, 2, 64, 8), 3, "cuda", dtype=torch.float32)
    dk = synth.orthonormal(2, 16, 8, 4, "cuda")
    dv = synth.orthonormal(2, 16, 8, 5, "cuda")
    out, lse = lla.lla_decode_attn(q, zk, zv, dk, dv)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    assert lla.device_status() == 0

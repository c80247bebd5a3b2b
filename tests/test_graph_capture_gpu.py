"""The library calls inside a CUDA graph.

A call allocates nothing and never synchronises, so a serving loop can
capture a whole decode step once and replay it. Each family is captured
here with caller-owned workspaces and outputs, the outputs are cleared,
and one replay must give the eager call's results bit for bit (the same
kernels on the same inputs)."""

import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import synth
from lla_cases import make_decode_inputs, make_paged_inputs

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def capture_matches_eager(run, outputs):
    """run() writes `outputs`; eager results, then a captured replay."""
    run()
    torch.cuda.synchronize()
    ref = [t.clone() for t in outputs]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    for t in outputs:
        t.fill_(float("nan") if t.is_floating_point() else 0)
    graph.replay()
    torch.cuda.synchronize()
    for got, want in zip(outputs, ref):
        assert torch.equal(got, want)
    assert lla.device_status() == 0


def test_per_head_decode_step():
    inp = make_decode_inputs(6, 4, 64, 300, 24, 40, BF16, mu=True, seed=1)
    ws = torch.empty(lla.lla_decode_attn_workspace(6, 4, 300, 24, 40), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(6, 4, 64, device="cuda")
    lse = torch.empty(6, 4, device="cuda")
    capture_matches_eager(
        lambda: lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"],
                                    mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"], out=out, lse=lse,
                                    workspace=ws), [out, lse])


def test_lla2d_decode_step():
    inp = make_decode_inputs(5, 16, 128, 700, 256, 256, BF16, two_d=True, seed=2)
    ws = torch.empty(lla.lla2d_decode_attn_workspace(5, 16, 700, 256, 256), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(5, 16, 128, device="cuda")
    lse = torch.empty(5, 16, device="cuda")
    capture_matches_eager(
        lambda: lla.lla2d_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"],
                                      out=out, lse=lse, workspace=ws), [out, lse])


def test_paged_plan_then_planned_calls():
    lens = [5, 64, 300, 1]
    inp = make_paged_inputs(lens, 3, 64, 24, 24, BF16, 64, seed=3)
    ws = torch.empty(lla.lla_decode_attn_paged_workspace(4, 3, 24, 24), dtype=torch.uint8,
                     device="cuda")
    outs = [torch.empty(4, 3, 64, device="cuda") for _ in range(2)]

    def step():
        lla.lla_decode_attn_paged_plan(inp["zk"], inp["zv"], inp["block_table"], inp["seq_lens"],
                                       ws)
        for o in outs:
            lla.lla_decode_attn_paged(inp["q"], inp["zk"], inp["zv"], inp["block_table"],
                                      inp["seq_lens"], inp["dk"], inp["dv"], out=o, workspace=ws,
                                      want_lse=False, planned=True)

    capture_matches_eager(step, outs)


def test_encode_split_over_k():
    T, N, G, d_loop, r = 4, 256, 1, 2048, 256
    x = synth.normal((T, N, G, d_loop), 4, "cuda", dtype=BF16)
    w_t = synth.orthonormal(G, T * d_loop, r, 5, "cuda").to(BF16).transpose(1, 2).contiguous()
    muw = lla.lla_encode_bias(w_t, synth.normal((G, T * d_loop), 6, "cuda", std=0.5))
    need = lla.lla_encode_with_bias_workspace_bytes(T, N, G, d_loop, r)
    assert need > 0  # this shape splits over K
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    z = torch.empty(G, N, r, device="cuda", dtype=BF16)
    capture_matches_eager(
        lambda: lla.lla_encode_with_bias(x, w_t, muw, z=z, z_row_stride=r, z_group_stride=N * r,
                                         workspace=ws), [z])

"""A paged decode step planned once (lla_decode_attn_paged_plan /
lla_decode_attn_paged_planned and the LLA-2D pair) against the unplanned
paged calls and the fp64 oracle, through the C ABI.

A looped model makes T x L calls per step over the same lengths and block
table; the plan (length and page checks, the split of the ragged range) is
made once and reused. The planned calls run the same kernels on the same
plan as the unplanned ones, so their outputs must agree bit for bit. A
planned call whose workspace holds no plan for it must decode nothing and
say so; a table changed after planning must not move a copy outside the
pool."""

import numpy as np
import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import synth
from lla_cases import (add_undeclared_pages, compare_paged, make_paged_inputs,
                       oracle_paged_reference)

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def layer_inputs(inp, n, seed):
    """n (layer, loop) calls' queries and decoders over the same store."""
    B, H, d = inp["q"].shape
    r_k, r_v = inp["zk"].shape[-1], inp["zv"].shape[-1]
    return [dict(q=synth.queries((B, H, d), d, seed + 10 * i, "cuda"),
                 dk=synth.orthonormal(H, d, r_k, seed + 10 * i + 1, "cuda"),
                 dv=synth.orthonormal(H, d, r_v, seed + 10 * i + 2, "cuda")) for i in range(n)]


@pytest.mark.parametrize("sink, window", [(0, 0), (4, 256)])
def test_per_head_planned_calls_equal_unplanned_calls(sink, window):
    lens = [0, 1, 64, 65, 700, 2000, 333]
    inp = make_paged_inputs(lens, 8, 128, 64, 64, BF16, 64, seed=5)
    ws = torch.empty(lla.lla_decode_attn_paged_workspace(len(lens), 8, 64, 64), dtype=torch.uint8,
                     device="cuda")
    calls = layer_inputs(inp, 3, seed=31)
    args = (inp["zk"], inp["zv"], inp["block_table"], inp["seq_lens"])
    refs = [lla.lla_decode_attn_paged(c["q"], *args, c["dk"], c["dv"], sink=sink, window=window)
            for c in calls]
    lla.lla_decode_attn_paged_plan(*args, ws, sink=sink, window=window)
    for c, (ro, rl) in zip(calls, refs):
        out, lse = lla.lla_decode_attn_paged_planned(c["q"], *args, c["dk"], c["dv"], sink=sink,
                                                     window=window, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(out, ro) and torch.equal(lse, rl)
    assert lla.device_status() == 0
    # and the last one against the oracle
    inp2 = dict(inp, q=calls[-1]["q"], dk=calls[-1]["dk"], dv=calls[-1]["dv"])
    ref_out, ref_lse = oracle_paged_reference(inp2, sink, window)
    compare_paged(out, lse, ref_out, ref_lse, lens, BF16)


def test_lla2d_planned_calls_equal_unplanned_calls():
    lens = np.array([1, 127, 128, 129, 0, 1000, 4000], dtype=np.int32)
    H, d, r, ps = 16, 128, 256, 64
    bt, P = synth.page_table(lens, ps, seed=7, spare=1)
    zk = synth.latents((P, ps, r), 1, "cuda", decay=True, dtype=BF16)
    zv = synth.latents((P, ps, r), 2, "cuda", decay=True, dtype=BF16)
    bt = torch.from_numpy(bt).cuda()
    sl = torch.from_numpy(lens).cuda()
    inp = dict(q=synth.queries((len(lens), H, d), d, 3, "cuda"), zk=zk, zv=zv)
    calls = layer_inputs(inp, 3, seed=41)
    ws = torch.empty(lla.lla2d_decode_attn_paged_workspace(len(lens), H, r, r),
                     dtype=torch.uint8, device="cuda")
    refs = [lla.lla2d_decode_attn_paged(c["q"], zk, zv, bt, sl, c["dk"], c["dv"]) for c in calls]
    lla.lla2d_decode_attn_paged_plan(zk, zv, bt, sl, H, ws)
    for c, (ro, rl) in zip(calls, refs):
        out, lse = lla.lla2d_decode_attn_paged_planned(c["q"], zk, zv, bt, sl, c["dk"], c["dv"],
                                                       workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(out, ro) and torch.equal(lse, rl)
    assert lla.device_status() == 0


@pytest.mark.parametrize("two_d", [False, True])
def test_planned_call_without_a_plan_decodes_nothing(two_d):
    # A zero-filled workspace holds no plan (its stamp is 0, which no plan
    # has): nothing is read, out = 0, lse = -inf, and the mismatch is
    # reported. A workspace planned for other lengths' pointer mismatches too.
    lens = [100, 300]
    H, d, r, ps = 16, 64, 128, 64
    if two_d:
        bt, P = synth.page_table(lens, ps, seed=9)
        zk = synth.latents((P, ps, r), 1, "cuda", dtype=BF16)
        zv = synth.latents((P, ps, r), 2, "cuda", dtype=BF16)
        ws = torch.zeros(lla.lla2d_decode_attn_paged_workspace(2, H, r, r), dtype=torch.uint8,
                         device="cuda")
        fn = lla.lla2d_decode_attn_paged_planned
    else:
        bt, P = synth.page_table(lens, ps, seed=9)
        zk = synth.latents((P, H, ps, r), 1, "cuda", dtype=BF16)
        zv = synth.latents((P, H, ps, r), 2, "cuda", dtype=BF16)
        ws = torch.zeros(lla.lla_decode_attn_paged_workspace(2, H, r, r), dtype=torch.uint8,
                         device="cuda")
        fn = lla.lla_decode_attn_paged_planned
    bt = torch.from_numpy(bt).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q = synth.queries((2, H, d), d, 3, "cuda")
    dk, dv = synth.orthonormal(H, d, r, 4, "cuda"), synth.orthonormal(H, d, r, 5, "cuda")
    lla.device_status(clear=True)
    out, lse = fn(q, zk, zv, bt, sl, dk, dv, workspace=ws)
    torch.cuda.synchronize()
    assert lla.device_status(clear=True) == lla._lib.LLA_DEVICE_PAGED_PLAN_MISMATCH
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    # planned for one lengths array, called with another: also a mismatch
    sl2 = sl.clone()
    plan = lla.lla2d_decode_attn_paged_plan if two_d else lla.lla_decode_attn_paged_plan
    if two_d:
        plan(zk, zv, bt, sl, H, ws)
    else:
        plan(zk, zv, bt, sl, ws)
    out, lse = fn(q, zk, zv, bt, sl2, dk, dv, workspace=ws)
    torch.cuda.synchronize()
    assert lla.device_status(clear=True) == lla._lib.LLA_DEVICE_PAGED_PLAN_MISMATCH
    assert torch.all(out == 0)
    assert lla.device_status() == 0


def test_table_changed_after_planning_stays_inside_the_pool():
    # The plan checked the table; afterwards one used entry is changed to a
    # page past the declared pool (allocated and NaN-filled, so even a
    # missed check would stay in bounds). The planned call reads page 0 in
    # its place and reports the bad index.
    lens = [200, 300]
    inp = make_paged_inputs(lens, 4, 64, 32, 32, BF16, 32, seed=13)
    extra = add_undeclared_pages(inp)
    ws = torch.empty(lla.lla_decode_attn_paged_workspace(2, 4, 32, 32), dtype=torch.uint8,
                     device="cuda")
    args = (inp["zk"], inp["zv"], inp["block_table"], inp["seq_lens"])
    lla.lla_decode_attn_paged_plan(*args, ws)
    inp["block_table"][1, 3] = extra[0]   # in place: the plan's pointer is unchanged
    lla.device_status(clear=True)
    out, lse = lla.lla_decode_attn_paged_planned(inp["q"], *args, inp["dk"], inp["dv"],
                                                 workspace=ws)
    torch.cuda.synchronize()
    assert lla.device_status(clear=True) & lla._lib.LLA_DEVICE_BAD_PAGED_INPUT
    assert torch.isfinite(out).all()
    assert lla.device_status() == 0

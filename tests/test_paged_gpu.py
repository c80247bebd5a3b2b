"""GPU parity of the paged, ragged per-head decode (lla_decode_attn_paged)
against the fp64 oracle, through the C ABI.

Cases: ragged length mixes (1 token, page-boundary lengths, empty
sequences), page sizes that do and do not divide the stage tile, both latent
types and several ranks, the attention-sink + window eviction set (with the
table entries of evicted blocks out of the declared pool and their pages
NaN), device-side
rejection of bad lengths and page indices, agreement with the dense kernel
on a dense-equivalent layout, and a full-size ragged batch."""

import numpy as np
import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import synth
from lla_cases import (add_undeclared_pages, compare_paged, make_paged_inputs,
                       oracle_paged_reference, pad_block_table, to_f64)

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32


def run_paged(inp, dtype, sink=0, window=0, fp32_tight=True, lens=None):
    out, lse = lla.lla_decode_attn_paged(inp["q"], inp["zk"], inp["zv"], inp["block_table"],
                                         inp["seq_lens"], inp["dk"], inp["dv"], inp["mu_k"],
                                         inp["mu_v"], sink=sink, window=window)
    torch.cuda.synchronize()
    lens = inp["seq_lens"].cpu().numpy() if lens is None else lens
    ref_out, ref_lse = oracle_paged_reference(inp, sink, window)
    err, lse_err = compare_paged(out, lse, ref_out, ref_lse, lens, dtype)
    if fp32_tight and dtype == BF16:
        assert err < 1e-4, f"relative error {err:.2e} above fp32 accumulation level"
    assert lse_err < 1e-3, f"lse error {lse_err:.2e}"
    assert lla.device_status() == 0
    return out, lse


@pytest.mark.parametrize("page_size", [1, 7, 16, 64, 100])
def test_ragged_lengths_page_sizes(page_size):
    lens = [1, page_size - 1 if page_size > 1 else 2, page_size, page_size + 1, 0, 333, 2 * page_size,
            57]
    inp = make_paged_inputs(lens, 3, 64, 24, 24, BF16, page_size, mu=True, seed=page_size)
    run_paged(inp, BF16)


@pytest.mark.parametrize("r_k, r_v, dtype", [(8, 8, F32), (32, 32, F32), (128, 128, F32),
                                              (16, 16, BF16), (48, 80, BF16), (128, 128, BF16),
                                              (256, 256, BF16), (96, 160, BF16)])
def test_ranks_and_types(r_k, r_v, dtype):
    lens = synth.ragged_lengths(9, 300, seed=r_k + r_v)
    inp = make_paged_inputs(lens, 4, 128, r_k, r_v, dtype, 32, mu=True, seed=r_k)
    run_paged(inp, dtype)


def test_all_empty_and_single_long_sequence():
    inp = make_paged_inputs([0, 0, 0], 2, 32, 16, 16, BF16, 16, seed=3)
    out, lse = lla.lla_decode_attn_paged(inp["q"], inp["zk"], inp["zv"], inp["block_table"],
                                         inp["seq_lens"], inp["dk"], inp["dv"])
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    assert lla.device_status() == 0
    # one sequence spread over every streaming warp
    inp = make_paged_inputs([50000], 2, 64, 16, 16, BF16, 256, seed=4)
    run_paged(inp, BF16)


@pytest.mark.parametrize("sink, window", [(4, 256), (0, 100), (3, 1), (16, 0), (5, 2000)])
def test_sink_window_eviction(sink, window):
    lens = [1000, 260, 261, 3, 0, 4000, 257]
    ps = 32
    inp = make_paged_inputs(lens, 3, 64, 24, 24, BF16, ps, mu=True, seed=sink + window)
    # Blocks that hold no kept token: their pages become NaN and their table
    # entries name a page past the declared pool (out of range for the call,
    # but allocated and NaN-filled by add_undeclared_pages), so reading or
    # checking an evicted block fails the test without leaving the allocation.
    import oracle
    extra = add_undeclared_pages(inp)
    bt = inp["block_table"].cpu().numpy()
    for b, n in enumerate(lens):
        kept = set((oracle.kept_positions(n, sink, window) // ps).tolist())
        for blk in range((n + ps - 1) // ps):
            if blk not in kept:
                inp["zk"][int(bt[b, blk])] = float("nan")
                inp["zv"][int(bt[b, blk])] = float("nan")
                bt[b, blk] = extra[blk % len(extra)]
    inp["block_table"] = torch.from_numpy(bt).cuda()
    out, lse = run_paged(inp, BF16, sink=sink, window=window)
    assert torch.isfinite(out).all()


def test_bad_lengths_and_pages_are_rejected_on_the_device():
    # Every planted error stays inside allocated memory, so a regressed check
    # gives a wrong number or status, not an illegal access:
    # - sequence 1 names a page one past the declared pool, which is an
    #   allocated NaN page (add_undeclared_pages);
    # - sequence 3, the table's last row, is one token longer than the table;
    #   its extra block lies in the padding row of the table's allocation,
    #   which names declared page 0 (pad_block_table).
    # A negative length has no in-bounds place to land, so none is planted.
    lens = [40, 50, 60, 70]
    inp = make_paged_inputs(lens, 2, 32, 16, 16, BF16, 16, seed=9)
    extra = add_undeclared_pages(inp)
    bt = inp["block_table"].cpu().numpy()
    bt[1, 2] = extra[0]           # a used block past the declared pool
    pad_block_table(inp, bt)
    inp["seq_lens"] = torch.tensor([40, 50, 60, bt.shape[1] * 16 + 1], dtype=torch.int32,
                                   device="cuda")
    lla.device_status(clear=True)
    out, lse = lla.lla_decode_attn_paged(inp["q"], inp["zk"], inp["zv"], inp["block_table"],
                                         inp["seq_lens"], inp["dk"], inp["dv"])
    torch.cuda.synchronize()
    st = lla.device_status(clear=True)
    assert st & lla._lib.LLA_DEVICE_BAD_PAGED_INPUT
    assert lla.device_status() == 0
    # sequences 1 and 3 are treated as empty; sequences 0 and 2 are intact
    o, l = out.cpu(), lse.cpu()
    for b in (1, 3):
        assert torch.all(o[b] == 0) and torch.all(torch.isneginf(l[b]))
    inp["seq_lens"] = torch.tensor([40, 0, 60, 0], dtype=torch.int32, device="cuda")
    ref_out, ref_lse = oracle_paged_reference(inp)
    for b in (0, 2):
        np.testing.assert_allclose(to_f64(out)[b], ref_out[b],
                                   atol=2e-2 * np.abs(ref_out[b]).max())


def test_dense_equivalent_layout_matches_the_dense_kernel():
    # page_size = n_cap, one page per sequence in order: the dense store
    B, H, d_h, N, r = 6, 4, 64, 777, 32
    zk = synth.latents((B, H, N, r), 1, "cuda", dtype=BF16)
    zv = synth.latents((B, H, N, r), 2, "cuda", dtype=BF16)
    dk = synth.orthonormal(H, d_h, r, 3, "cuda")
    dv = synth.orthonormal(H, d_h, r, 4, "cuda")
    q = synth.queries((B, H, d_h), d_h, 5, "cuda")
    o1, l1 = lla.lla_decode_attn(q, zk, zv, dk, dv)
    bt = torch.arange(B, dtype=torch.int32, device="cuda").reshape(B, 1)
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    o2, l2 = lla.lla_decode_attn_paged(q, zk, zv, bt, sl, dk, dv)
    torch.cuda.synchronize()
    assert (o1 - o2).abs().max().item() <= 1e-5 * o1.abs().max().item()
    assert (l1 - l2).abs().max().item() <= 1e-5


def test_full_size_ragged_batch_sampled():
    # the perhead_4x_paged workload: a serving batch at the 4x geometry, 64
    # sequences of 2k..6k tokens, 64-token pages; checked on sampled sequences
    lens = synth.C2_PAGED.lengths()
    inp = make_paged_inputs(lens, 16, 128, 128, 128, BF16, 64, seed=0)
    out, lse = lla.lla_decode_attn_paged(inp["q"], inp["zk"], inp["zv"], inp["block_table"],
                                         inp["seq_lens"], inp["dk"], inp["dv"])
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    pick = [0, 1, 31, 63]
    sub = dict(inp)
    sub["q"] = inp["q"][pick]
    sub["block_table"] = inp["block_table"][pick]
    sub["seq_lens"] = inp["seq_lens"][pick]
    ref_out, ref_lse = oracle_paged_reference(sub)
    compare_paged(out[pick], lse[pick], ref_out, ref_lse, lens[pick], BF16)

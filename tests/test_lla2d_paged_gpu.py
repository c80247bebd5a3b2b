"""GPU parity of the paged, ragged LLA-2D decode (lla2d_decode_attn_paged)
against the fp64 oracle, through the C ABI.

Cases: ragged length mixes around the 128-token tile (0, 1, 127, 128, 129,
page boundaries), page sizes 64, 128, 192 and 256 (64-token pages split
a tile over two pages), shuffled pools, more sequences
than CTAs and sequences spread over many CTAs, device-side rejection of bad
lengths and page indices, agreement with the dense kernel on a
dense-equivalent layout, and the 32x geometry as a ragged serving batch."""

import numpy as np
import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import synth
from lla_cases import TOL_BF16_REL, add_undeclared_pages, pad_block_table, to_f64

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


def make(lens, H, d_h, r_k, r_v, page_size, mu=False, seed=0, spare=2):
    bt, num_pages = synth.page_table(lens, page_size, seed + 11, spare=spare)
    B = len(lens)
    zk = synth.latents((num_pages, page_size, r_k), seed + 1, "cuda", decay=True, dtype=BF16)
    zv = synth.latents((num_pages, page_size, r_v), seed + 2, "cuda", decay=True, dtype=BF16)
    return dict(q=synth.queries((B, H, d_h), d_h, seed + 5, "cuda"), zk=zk, zv=zv,
                dk=synth.orthonormal(H, d_h, r_k, seed + 3, "cuda"),
                dv=synth.orthonormal(H, d_h, r_v, seed + 4, "cuda"),
                mu_k=synth.normal((H, d_h), seed + 6, "cuda") if mu else None,
                mu_v=synth.normal((H, d_h), seed + 7, "cuda") if mu else None,
                block_table=torch.from_numpy(bt).cuda(),
                seq_lens=torch.tensor(np.asarray(lens, dtype=np.int32), device="cuda"))


def run(inp, sink=0, window=0):
    return lla.lla2d_decode_attn_paged(inp["q"], inp["zk"], inp["zv"], inp["block_table"],
                                       inp["seq_lens"], inp["dk"], inp["dv"], inp["mu_k"],
                                       inp["mu_v"], sink=sink, window=window)


def reference(inp, pick=None, sink=0, window=0):
    import oracle  # test infrastructure only
    opt = lambda t: None if t is None else to_f64(t)
    sel = slice(None) if pick is None else pick
    return oracle.paged2d_decode(to_f64(inp["q"][sel]), to_f64(inp["zk"]), to_f64(inp["zv"]),
                                 inp["block_table"][sel].cpu().numpy().astype(np.int64),
                                 inp["seq_lens"][sel].cpu().numpy(), to_f64(inp["dk"]),
                                 to_f64(inp["dv"]), opt(inp["mu_k"]), opt(inp["mu_v"]),
                                 sink=sink, window=window)


def compare(out, lse, ref_out, ref_lse, lens):
    o, l = to_f64(out), to_f64(lse)
    lens = np.asarray(lens)
    empty = lens == 0
    assert np.all(o[empty] == 0) and np.all(np.isneginf(l[empty]))
    full = ~empty
    err = np.abs(o[full] - ref_out[full]).max() / np.abs(ref_out[full]).max()
    assert err <= TOL_BF16_REL, f"bf16 relative error {err:.3e}"
    assert np.abs(l[full] - ref_lse[full]).max() < 2e-2
    return err


@pytest.mark.parametrize("page_size", [64, 128, 192, 256])
def test_ragged_lengths_around_the_tile(page_size):
    lens = [1, 127, 128, 129, 0, 255, 256, 257, 1000, 3]
    inp = make(lens, 16, 128, 256, 256, page_size, mu=True, seed=page_size)
    out, lse = run(inp)
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    compare(out, lse, *reference(inp), lens)


@pytest.mark.parametrize("H, r_k, r_v", [(8, 64, 128), (20, 128, 256), (32, 192, 128),
                                         (16, 96, 160), (4, 200, 8)])
def test_heads_and_ranks(H, r_k, r_v):
    lens = synth.ragged_lengths(7, 700, seed=H)
    inp = make(lens, H, 64, r_k, r_v, 128, seed=H + r_k)
    out, lse = run(inp)
    torch.cuda.synchronize()
    compare(out, lse, *reference(inp), lens)


def test_many_short_and_one_long_sequence():
    # more sequences than CTAs, and one spread over many CTAs
    lens = list(synth.ragged_lengths(300, 150, seed=3)) + [60000]
    inp = make(lens, 16, 128, 256, 256, 256, seed=9)
    out, lse = run(inp)
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    pick = [0, 1, 150, 299, 300]
    ref_out, ref_lse = reference(inp, pick)
    compare(out[pick], lse[pick], ref_out, ref_lse, np.asarray(lens)[pick])


def test_bad_lengths_and_pages_are_rejected_on_the_device():
    # Planted errors stay inside allocated memory: sequence 1 names a page
    # past the declared pool that is allocated (add_undeclared_pages), and
    # sequence 2, the table's last row, is one token longer than its table
    # row, whose next entry lies in the padding row (pad_block_table).
    lens = [300, 400, 500]
    inp = make(lens, 16, 64, 128, 128, 128, seed=4)
    extra = add_undeclared_pages(inp)
    bt = inp["block_table"].cpu().numpy()
    bt[1, 1] = extra[1]
    pad_block_table(inp, bt)
    inp["seq_lens"] = torch.tensor([300, 400, bt.shape[1] * 128 + 1], dtype=torch.int32,
                                   device="cuda")
    lla.device_status(clear=True)
    out, lse = run(inp)
    torch.cuda.synchronize()
    assert lla.device_status(clear=True) & lla._lib.LLA_DEVICE_BAD_PAGED_INPUT
    assert torch.all(out[1:] == 0) and torch.all(torch.isneginf(lse[1:]))
    inp["seq_lens"] = torch.tensor([300, 0, 0], dtype=torch.int32, device="cuda")
    ref_out, ref_lse = reference(inp)
    compare(out, lse, ref_out, ref_lse, [300, 0, 0])


def test_dense_equivalent_layout_matches_the_dense_kernel():
    B, H, d_h, N, r = 5, 16, 128, 768, 256
    zk = synth.latents((B, N, r), 1, "cuda", decay=True, dtype=BF16)
    zv = synth.latents((B, N, r), 2, "cuda", decay=True, dtype=BF16)
    dk = synth.orthonormal(H, d_h, r, 3, "cuda")
    dv = synth.orthonormal(H, d_h, r, 4, "cuda")
    q = synth.queries((B, H, d_h), d_h, 5, "cuda")
    o1, l1 = lla.lla2d_decode_attn(q, zk, zv, dk, dv)
    bt = torch.arange(B, dtype=torch.int32, device="cuda").reshape(B, 1)
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    o2, l2 = lla.lla2d_decode_attn_paged(q, zk, zv, bt, sl, dk, dv)
    torch.cuda.synchronize()
    assert (o1 - o2).abs().max().item() <= 1e-5 * o1.abs().max().item()
    assert (l1 - l2).abs().max().item() <= 1e-4


@pytest.mark.parametrize("page_size", [256, 64])
def test_full_size_ragged_32x_batch_sampled(page_size):
    # the lla2d_32x_paged and lla2d_32x_paged64 workloads
    lens = synth.ragged_lengths(256, 8192, seed=0)
    inp = make(lens, 16, 128, 256, 256, page_size, seed=0)
    out, lse = run(inp)
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    pick = [0, 1, 127, 255]
    ref_out, ref_lse = reference(inp, pick)
    compare(out[pick], lse[pick], ref_out, ref_lse, lens[pick])


@pytest.mark.parametrize("sink, window, page_size", [(4, 256, 256), (0, 300, 128), (130, 1, 128),
                                                     (4, 5000, 256), (4, 256, 64), (4, 230, 64),
                                                     (70, 100, 192), (0, 300, 192), (130, 1, 64)])
def test_sink_window_eviction(sink, window, page_size):
    import oracle  # test infrastructure only
    lens = [3000, 260, 261, 1, 0, 9000, 257, 700]
    inp = make(lens, 16, 128, 256, 256, page_size, mu=True, seed=sink + window)
    # Pages holding no kept token: NaN latents, and table entries that name a
    # page past the declared pool (allocated and NaN-filled by
    # add_undeclared_pages), so reading or checking them fails the test
    # without leaving the allocation.
    extra = add_undeclared_pages(inp)
    bt = inp["block_table"].cpu().numpy()
    for b, n in enumerate(lens):
        kept_blocks = set((oracle.kept_positions(n, sink, window) // page_size).tolist())
        for blk in range((n + page_size - 1) // page_size):
            if blk not in kept_blocks:
                inp["zk"][int(bt[b, blk])] = float("nan")
                inp["zv"][int(bt[b, blk])] = float("nan")
                bt[b, blk] = extra[blk % len(extra)]
    inp["block_table"] = torch.from_numpy(bt).cuda()
    out, lse = run(inp, sink, window)
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    assert torch.isfinite(out).all()
    compare(out, lse, *reference(inp, sink=sink, window=window), lens)


@pytest.mark.parametrize("H, r_k, r_v", [(32, 192, 128), (8, 64, 256), (16, 96, 160),
                                         (12, 40, 24)])
def test_64_token_pages_heads_and_ranks(H, r_k, r_v):
    # every tile half from its own shuffled page; key rows of one and three boxes
    lens = [64, 65, 128, 1, 191, 640, 333]
    inp = make(lens, H, 64, r_k, r_v, 64, mu=True, seed=H + r_v)
    out, lse = run(inp)
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    compare(out, lse, *reference(inp), lens)


def test_64_token_pages_never_read_past_the_length():
    # a tile half wholly past a sequence's length is zero-filled, not read:
    # its table entry names a NaN-filled spare page
    lens = [64, 192, 320]
    inp = make(lens, 16, 128, 256, 256, 64, mu=True, seed=21, spare=1)
    bt = inp["block_table"].cpu().numpy()
    used = set(bt[bt >= 0].tolist())
    poison = next(p for p in range(inp["zk"].shape[0]) if p not in used)
    inp["zk"][poison] = float("nan")
    inp["zv"][poison] = float("nan")
    bt[bt < 0] = poison
    assert (bt == poison).sum() == 6
    inp["block_table"] = torch.from_numpy(bt).cuda()
    out, lse = run(inp)
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    assert torch.isfinite(out).all()
    compare(out, lse, *reference(inp), lens)

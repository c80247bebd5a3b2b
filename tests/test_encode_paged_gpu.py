"""GPU parity of the latent write into a paged store (lla_encode_paged)
against the oracle's Eq. 2 encode followed by its paged scatter, through the
C ABI.

Cases: a serving step that appends every sequence's newest token to a
shuffled per-head pool (positions at, before and across page boundaries),
key rows wider than the latent (a rotary tail that must survive), the wide
LLA-2D stack written for one decode step (split over K), a chunked prefill
of one sequence across several pages, out-of-range entries that must be
skipped and reported, and a write followed by the paged decode. Rows the
call does not address must stay bit-identical."""

import numpy as np
import pytest
import torch

import decode_attention_encode_b200 as lla
import oracle
from decode_attention_encode_b200 import synth
from lla_cases import check_encoded, to_f64

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


def codec(T, G, d_loop, r, seed, mu=True):
    w = synth.orthonormal(G, T * d_loop, r, seed + 2, "cuda").to(BF16)       # [G, K, r]
    w_t = w.transpose(1, 2).contiguous()                                       # [G, r, K]
    m = synth.normal((G, T * d_loop), seed + 3, "cuda", std=0.5) if mu else None
    muw = lla.lla_encode_bias(w_t, m) if mu else None
    return w, w_t, m, muw


def check_write(pool_before, pool_after, x, w, m, bt, pos, seq=None):
    """Written rows within the rounding bound of the oracle, every other
    element bit-identical."""
    z_ref = oracle.encode(to_f64(x), to_f64(w), None if m is None else to_f64(m))
    ref_pool, skipped = oracle.paged_write(to_f64(pool_before), z_ref, bt.cpu().numpy(),
                                           pos.cpu().numpy(),
                                           None if seq is None else seq.cpu().numpy())
    marker, _ = oracle.paged_write(np.zeros(pool_before.shape), np.ones_like(z_ref),
                                   bt.cpu().numpy(), pos.cpu().numpy(),
                                   None if seq is None else seq.cpu().numpy())
    written = marker != 0
    after = to_f64(pool_after)
    check_encoded(after[written], ref_pool[written])
    keep = torch.from_numpy(~written).cuda()
    assert torch.equal(pool_after[keep], pool_before[keep]), "a row the call does not address changed"
    return skipped


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("page_size", [16, 64, 100])
def test_serving_step_appends_each_sequences_newest_token(page_size, split):
    # per-head pool [P][H][page_size][r]: token b is sequence b's newest,
    # written at position seq_lens[b]
    T, H, d, r = 4, 16, 128, 128
    lens = np.array([0, 1, page_size - 1, page_size, page_size + 1, 3 * page_size, 777, 5],
                    dtype=np.int32)
    B = len(lens)
    bt_np, P = synth.page_table(lens + 1, page_size, seed=page_size, spare=3)
    bt = torch.from_numpy(bt_np).cuda()
    pool = synth.latents((P, H, page_size, r), 7, "cuda", dtype=BF16)
    before = pool.clone()
    x = synth.normal((T, B, H, d), 8, "cuda", dtype=BF16)
    w, w_t, m, muw = codec(T, H, d, r, seed=page_size)
    pos = torch.from_numpy(lens).cuda()
    # split: a few tokens split the contraction over K (k_encode_reduce
    # places the rows); unsplit, the tensor-core epilogue places them
    lla.lla_encode_paged(x, w_t, muw, pool, bt, pos, split=split)
    torch.cuda.synchronize()
    assert check_write(before, pool, x, w, m, bt, pos) == []
    assert lla.device_status() == 0


def test_key_rows_keep_their_rotary_tail():
    T, H, d, r, dr, ps = 4, 4, 64, 48, 16, 32
    lens = np.array([10, 31, 32, 100], dtype=np.int32)
    bt_np, P = synth.page_table(lens + 1, ps, seed=3, spare=1)
    bt = torch.from_numpy(bt_np).cuda()
    pool = synth.latents((P, H, ps, r + dr), 4, "cuda", dtype=BF16)
    before = pool.clone()
    x = synth.normal((T, len(lens), H, d), 5, "cuda", dtype=BF16)
    w, w_t, m, muw = codec(T, H, d, r, seed=6)
    pos = torch.from_numpy(lens).cuda()
    lla.lla_encode_paged(x, w_t, muw, pool, bt, pos)
    torch.cuda.synchronize()
    check_write(before, pool, x, w, m, bt, pos)
    assert lla.device_status() == 0


@pytest.mark.parametrize("B", [3, 256])
def test_lla2d_stack_of_one_decode_step(B):
    # LLA-2D: each token's whole stack (T x 16 heads x 128) to one r = 256
    # latent, in a [P][page_size][256] pool; B = 256 splits over K
    T, HD, r, ps = 4, 16 * 128, 256, 256
    lens = synth.ragged_lengths(B, 700, seed=B)
    bt_np, P = synth.page_table(lens + 1, ps, seed=B + 1, spare=2)
    bt = torch.from_numpy(bt_np).cuda()
    pool = synth.latents((P, ps, r), 9, "cuda", dtype=BF16)
    before = pool.clone()
    x = synth.normal((T, B, 1, HD), 10, "cuda", dtype=BF16)
    w, w_t, m, muw = codec(T, 1, HD, r, seed=11)
    pos = torch.from_numpy(lens).cuda()
    assert lla.lla_encode_with_bias_workspace_bytes(T, B, 1, HD, r) > 0   # split over K
    lla.lla_encode_paged(x, w_t, muw, pool, bt, pos)
    torch.cuda.synchronize()
    check_write(before, pool, x, w, m, bt, pos)
    assert lla.device_status() == 0


def test_chunked_prefill_of_one_sequence_across_pages():
    # 300 tokens of sequence 2 at positions 50..349 of 64-token pages
    T, H, d, r, ps = 4, 3, 64, 16, 64
    lens = np.array([10, 20, 350, 5], dtype=np.int32)
    bt_np, P = synth.page_table(lens, ps, seed=12, spare=2)
    bt = torch.from_numpy(bt_np).cuda()
    pool = synth.latents((P, H, ps, r), 13, "cuda", dtype=BF16)
    before = pool.clone()
    n = 300
    x = synth.normal((T, n, H, d), 14, "cuda", dtype=BF16)
    w, w_t, m, muw = codec(T, H, d, r, seed=15, mu=False)
    pos = torch.arange(50, 50 + n, dtype=torch.int32, device="cuda")
    seq = torch.full((n,), 2, dtype=torch.int32, device="cuda")
    lla.lla_encode_paged(x, w_t, muw, pool, bt, pos, seq_idx=seq)
    torch.cuda.synchronize()
    check_write(before, pool, x, w, m, bt, pos, seq)
    assert lla.device_status() == 0


@pytest.mark.parametrize("split", [True, False])
def test_out_of_range_entries_are_skipped_and_reported(split):
    # Every bad entry stays inside allocated memory, so a regressed device
    # check gives a wrong row or status, never an illegal access:
    # - token 1's position is one page past its table row; that row is the
    #   table's last and its allocation has a padding row behind it naming a
    #   declared page;
    # - token 2's table entry names a page allocated after the declared pool;
    # - token 3's sequence index is one past the declared rows, which is the
    #   padding row.
    T, H, d, r, ps = 4, 2, 64, 16, 8
    n_seq, mb = 4, 3
    P_decl, P_alloc = 10, 12
    alloc = synth.latents((P_alloc, H, ps, r), 16, "cuda", dtype=BF16)
    pool = alloc[:P_decl]
    bt_all = torch.tensor([[0, 1, 2], [3, 4, 11], [5, 6, 7], [8, 9, 0], [0, 0, 0]],
                          dtype=torch.int32, device="cuda")
    bt = bt_all[:n_seq]
    before = alloc.clone()
    x = synth.normal((T, 4, H, d), 17, "cuda", dtype=BF16)
    w, w_t, m, muw = codec(T, H, d, r, seed=18)
    seq = torch.tensor([0, 3, 1, 4], dtype=torch.int32, device="cuda")
    pos = torch.tensor([5, mb * ps, 2 * ps + 1, 0], dtype=torch.int32, device="cuda")
    lla.device_status(clear=True)
    lla.lla_encode_paged(x, w_t, muw, pool, bt, pos, seq_idx=seq, split=split)
    torch.cuda.synchronize()
    assert lla.device_status(clear=True) & lla._lib.LLA_DEVICE_BAD_PAGED_INPUT
    assert lla.device_status() == 0
    # the undeclared pages and the padding row's page 0 beyond token 0's row
    # are untouched; token 0 landed
    assert torch.equal(alloc[P_decl:], before[P_decl:])
    skipped = check_write(before[:P_decl], pool, x, w, m, bt, pos, seq)
    assert skipped == [1, 2, 3]


def test_write_then_paged_decode_matches_the_oracle():
    # a serving step: append the newest token, then decode with the longer
    # lengths; the new token is attended with the rest
    T, H, d, r, ps = 4, 8, 128, 64, 32
    lens = np.array([31, 64, 100, 1], dtype=np.int32)
    bt_np, P = synth.page_table(lens + 1, ps, seed=20, spare=1)
    bt = torch.from_numpy(bt_np).cuda()
    zk = synth.latents((P, H, ps, r), 21, "cuda", dtype=BF16)
    zv = synth.latents((P, H, ps, r), 22, "cuda", dtype=BF16)
    xk = synth.normal((T, len(lens), H, d), 23, "cuda", dtype=BF16)
    xv = synth.normal((T, len(lens), H, d), 24, "cuda", dtype=BF16)
    wk, wk_t, mk, muwk = codec(T, H, d, r, seed=25)
    wv, wv_t, mv, muwv = codec(T, H, d, r, seed=26)
    pos = torch.from_numpy(lens).cuda()
    zk_ref, _ = oracle.paged_write(to_f64(zk), oracle.encode(to_f64(xk), to_f64(wk), to_f64(mk)),
                                   bt_np, lens)
    zv_ref, _ = oracle.paged_write(to_f64(zv), oracle.encode(to_f64(xv), to_f64(wv), to_f64(mv)),
                                   bt_np, lens)
    lla.lla_encode_paged(xk, wk_t, muwk, zk, bt, pos)
    lla.lla_encode_paged(xv, wv_t, muwv, zv, bt, pos)
    new_lens = torch.from_numpy(lens + 1).cuda()
    dk = synth.orthonormal(H, d, r, 27, "cuda")
    dv = synth.orthonormal(H, d, r, 28, "cuda")
    q = synth.queries((len(lens), H, d), d, 29, "cuda")
    out, lse = lla.lla_decode_attn_paged(q, zk, zv, bt, new_lens, dk, dv)
    torch.cuda.synchronize()
    assert lla.device_status() == 0
    # the oracle decodes its own write (exact Eq. 2 rows): the gap is the
    # bf16 rounding of the new rows plus fp32 accumulation
    ref_o, ref_l = oracle.paged_decode(to_f64(q), zk_ref, zv_ref, bt_np, lens + 1, to_f64(dk),
                                       to_f64(dv), scale=d ** -0.5)
    err = np.abs(to_f64(out) - ref_o).max() / np.abs(ref_o).max()
    assert err <= 2e-2, err
    assert np.abs(to_f64(lse) - ref_l).max() < 2e-2

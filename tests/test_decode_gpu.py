"""GPU parity of the per-head absorbed decode (lla_decode_attn) against the
fp64 oracle, through the C ABI.

Cases span the 16-byte segment layouts the kernel selects (lanes per token
1, 2, 4, 8; exact and masked), tiles with ragged tails, units split across
several warps, the degenerate contexts (N = 1, N not a multiple of anything),
non-zero codec means, a sharp softmax, and the full-size workloads in the
launch configuration the benchmark times."""

import math

import numpy as np
import pytest
import torch

import decode_attention_encode_b200 as lla
from lla_cases import compare, make_decode_inputs, oracle_reference, sample_units

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32


def run_case(B, H, d_h, N, r_k, r_v, dtype, units=None, fp32_tight=True, **kw):
    inp = make_decode_inputs(B, H, d_h, N, r_k, r_v, dtype, **kw)
    out, lse = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N,
                                   mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"])
    torch.cuda.synchronize()
    if units is None:
        units = [(b, h) for b in range(B) for h in range(H)]
    ref_out, ref_lse = oracle_reference(inp, units)
    err, lse_err = compare(out, lse, units, ref_out, ref_lse, dtype)
    # The per-head kernel rounds nothing below fp32 (latents are widened
    # exactly, q' and the value sums are fp32), so it sits far inside the
    # bf16 tolerance; a regression to bf16-level error would show here.
    if fp32_tight and dtype == BF16:
        assert err < 1e-4, f"relative error {err:.2e} above fp32 accumulation level"
    assert lse_err < 1e-3, f"lse error {lse_err:.2e}"
    assert lla.device_status() == 0
    return err, lse_err


def test_tiny_fp32_config():
    # 1 layer, T=4, H=2, d_h=16, r=8 (8x), batch 1, 64 cached tokens, seed 0
    for t in range(4):
        run_case(1, 2, 16, 64, 8, 8, F32, seed=100 * t)


@pytest.mark.parametrize("N", [1, 2, 7, 63, 64, 65, 127, 1000])
def test_tiny_fp32_context_lengths(N):
    run_case(1, 2, 16, N, 8, 8, F32, n_cap=N + 5, mu=True)


@pytest.mark.parametrize("r", [8, 16, 24, 32, 48, 64, 128, 256])
def test_bf16_ranks_multi_tile_ragged(r):
    run_case(3, 5, 64, 1000, r, r, BF16, n_cap=1030, mu=True, decay=True, seed=r)


@pytest.mark.parametrize("r", [8, 16, 24, 32, 64, 128])
def test_fp32_ranks(r):
    run_case(2, 3, 32, 333, r, r, F32, mu=True, seed=r)


@pytest.mark.parametrize("r_k, r_v", [(96, 160), (160, 96), (160, 160), (80, 80), (24, 40),
                                      (16, 24), (8, 256), (40, 40), (192, 128), (128, 64)])
def test_asymmetric_and_odd_ranks(r_k, r_v):
    run_case(2, 4, 128, 517, r_k, r_v, BF16, mu=True, seed=r_k + r_v)


@pytest.mark.parametrize("d_h", [1, 4, 100, 256])
def test_head_widths(d_h):
    run_case(2, 3, d_h, 200, 16, 24, BF16, mu=True)


def test_sharp_softmax_with_planted_token():
    # Queries scaled x8 and, per unit, one cached key latent aligned with the
    # absorbed query, so one token holds most of the softmax mass.
    B, H, d_h, N, r = 4, 6, 128, 3000, 128
    inp = make_decode_inputs(B, H, d_h, N, r, r, BF16, q_scale=8.0, seed=7)
    qp = torch.einsum("hdr,bhd->bhr", inp["dk"], inp["q"])
    pos = torch.randint(0, N, (B, H), generator=torch.Generator().manual_seed(3)).cuda()
    planted = (qp / qp.norm(dim=-1, keepdim=True) * 12.0).to(BF16)
    inp["zk"][torch.arange(B)[:, None], torch.arange(H)[None, :], pos] = planted
    out, lse = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N)
    torch.cuda.synchronize()
    units = [(b, h) for b in range(B) for h in range(H)]
    ref_out, ref_lse = oracle_reference(inp, units)
    err, lse_err = compare(out, lse, units, ref_out, ref_lse, BF16)
    assert err < 1e-4 and lse_err < 1e-3


def test_many_units_few_tokens_and_repeat_calls():
    # B*H much larger than the warp count: each warp crosses many units.
    inp = make_decode_inputs(64, 16, 64, 40, 24, 24, BF16, mu=True, seed=11)
    ws = torch.empty(lla.lla_decode_attn_workspace(64, 16, 40, 24, 24), dtype=torch.uint8,
                     device="cuda")
    o1, l1 = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"],
                                 mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"], workspace=ws)
    o2, l2 = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"],
                                 mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)  # deterministic
    units = sample_units(64, 16)
    ref_out, ref_lse = oracle_reference(inp, units)
    compare(o1, l1, units, ref_out, ref_lse, BF16)


@pytest.mark.parametrize("d_h, r_k, r_v", [(64, 40, 24), (128, 128, 256), (16, 8, 8), (48, 16, 16),
                                           (64, 256, 192), (40, 200, 40), (16, 192, 8)])
def test_large_batch_absorb_and_combine(d_h, r_k, r_v):
    # From B = 256 with a rank of 192 or more the per-head path forms q' and
    # W^V ubar on the tensor cores with split bf16 operands (the others stay
    # on the CUDA cores); 300 rows leave a ragged 64-row block, d_h = 16
    # and 40 keep the CUDA-core absorb (the tensor-core one stages d_h of 64
    # or 128) with the tensor-core combine, and the fp32-level bound of
    # run_case holds for the split products.
    B, H = 300, 3
    pick = [(b, h) for b in (0, 1, 63, 64, 255, 256, 299) for h in range(H)]
    run_case(B, H, d_h, 200, r_k, r_v, BF16, units=pick, mu=True, decay=True, seed=d_h + r_k)


# ---------------------------------------------------------------------------
# full-size workloads, one (layer, loop) step each, sampled units
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name, B, H, N, r, decay", [
    ("perhead_4x", 64, 16, 4096, 128, True),
    ("perhead_21x", 768, 16, 4096, 24, True),
    ("perhead_32x_long", 32, 16, 32768, 16, False),
])
def test_full_size_sampled(name, B, H, N, r, decay):
    err, lse_err = run_case(B, H, 128, N, r, r, BF16, units=sample_units(B, H), decay=decay,
                            seed=0)
    print(f"{name}: rel err {err:.2e}, lse err {lse_err:.2e}")
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype", [BF16, F32])
def test_rows_beyond_N_are_never_read(dtype):
    # Every cached row at or past N is NaN: one read of it would poison the
    # softmax or the value sum.
    B, H, d_h, N, n_cap, r = 3, 4, 64, 777, 900, 24
    inp = make_decode_inputs(B, H, d_h, N, r, r, dtype, n_cap=n_cap, mu=True, seed=31)
    inp["zk"][:, :, N:] = float("nan")
    inp["zv"][:, :, N:] = float("nan")
    out, lse = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N,
                                   mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"])
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    units = [(b, h) for b in range(B) for h in range(H)]
    ref_out, ref_lse = oracle_reference(inp, units)
    compare(out, lse, units, ref_out, ref_lse, dtype)


def test_launch_timers_bracket_each_streaming_kernel_without_syncs():
    inp = make_decode_inputs(64, 16, 128, 2048, 128, 128, BF16, seed=6)
    args = (inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"])
    lla.lla_decode_attn(*args)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with lla.launch_timers(4) as lt:
        ev[0].record()
        for _ in range(3):
            lt.next()
            lla.lla_decode_attn(*args)
        lt.pause()
        lla.lla_decode_attn(*args)  # not timed
        ev[1].record()
    assert lt.used == 3 and len(lt.ms) == 3
    total = ev[0].elapsed_time(ev[1])
    assert all(m > 0 for m in lt.ms) and sum(lt.ms) < total
    with pytest.raises(lla.LLAError):
        with lla.launch_timers(1) as lt:
            lt.next()
            lt.next()


def test_kernel_timer_brackets_the_streaming_kernel():
    inp = make_decode_inputs(64, 16, 128, 2048, 128, 128, BF16, seed=5)
    args = (inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"])
    lla.lla_decode_attn(*args)
    call0, call1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with lla.kernel_timer() as kt:
        call0.record()
        lla.lla_decode_attn(*args)
        call1.record()
    torch.cuda.synchronize()
    call_ms = call0.elapsed_time(call1)
    assert 0 < kt.ms <= call_ms
    # after the block the hook is cleared: a plain call records nothing new
    lla.lla_decode_attn(*args)
    torch.cuda.synchronize()

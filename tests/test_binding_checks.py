"""The Python binding rejects mismatched operands before the C call.

The kernels trust the element types and shapes they are given: an fp32 zk
with a bf16 zv, for instance, would be read at the wrong width. The binding
therefore checks every operand's dtype and shape against q (or x) and raises
LLAError(LLA_ERR_INVALID_ARG). These checks run before the CUDA-placement
check, so CPU tensors exercise them here; nothing reaches the library."""

import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import _lib

F32, BF16 = torch.float32, torch.bfloat16
B, H, D, N, RK, RV = 2, 3, 16, 5, 8, 16


def dense(**over):
    a = dict(q=torch.zeros(B, H, D), zk=torch.zeros(B, H, N, RK, dtype=BF16),
             zv=torch.zeros(B, H, N, RV, dtype=BF16), dk_t=torch.zeros(H, D, RK),
             dv_t=torch.zeros(H, D, RV))
    a.update(over)
    return a


def dense2d(**over):
    a = dict(q=torch.zeros(B, H, D), zk=torch.zeros(B, N, RK, dtype=BF16),
             zv=torch.zeros(B, N, RV, dtype=BF16), dk_t=torch.zeros(H, D, RK),
             dv_t=torch.zeros(H, D, RV))
    a.update(over)
    return a


def rejects(fn, match, **kw):
    with pytest.raises(lla.LLAError, match=match) as e:
        fn(**kw)
    assert e.value.status == _lib.LLA_ERR_INVALID_ARG


@pytest.mark.parametrize("over, match", [
    (dict(zv=torch.zeros(B, H, N, RV, dtype=F32)), "zv must have zk's dtype"),
    (dict(q=torch.zeros(B, H, D, dtype=torch.float64)), "q must be float32"),
    (dict(dk_t=torch.zeros(H, D, RK, dtype=BF16)), "dk_t must be float32"),
    (dict(dv_t=torch.zeros(H, D, RV + 8)), "dv_t must have shape"),
    (dict(dk_t=torch.zeros(H, D + 1, RK)), "dk_t must have shape"),
    (dict(zv=torch.zeros(B, H, N + 1, RV, dtype=BF16)), "do not match q"),
    (dict(zk=torch.zeros(B + 1, H, N, RK, dtype=BF16)), "do not match q"),
    (dict(zk=torch.zeros(B, H, N, RK, dtype=torch.float16)), "unsupported latent dtype"),
    (dict(mu_k_t=torch.zeros(H, D + 2)), "mu_k_t must have shape"),
    (dict(mu_v_t=torch.zeros(H, D, dtype=BF16)), "mu_v_t must be float32"),
    (dict(out=torch.zeros(B, H, D + 1)), "out must have shape"),
    (dict(lse=torch.zeros(B, H, 1)), "lse must have shape"),
])
@pytest.mark.parametrize("fn", [lla.lla_decode_attn, lla.lla_decode_attn_noalloc])
def test_per_head_decode_checks_operands(fn, over, match):
    rejects(fn, match, **dense(**over))


def test_well_formed_cpu_operands_reach_the_placement_check():
    rejects(lla.lla_decode_attn, "contiguous CUDA", **dense())
    rejects(lla.lla2d_decode_attn, "contiguous CUDA", **dense2d())


@pytest.mark.parametrize("over, match", [
    (dict(zv=torch.zeros(B, N, RV, dtype=F32)), "zv must have zk's dtype"),
    (dict(zk=torch.zeros(B, H, N, RK, dtype=BF16)), "latents must be"),
    (dict(zv=torch.zeros(B, N + 3, RV, dtype=BF16)), "do not match q"),
    (dict(dv_t=torch.zeros(H, D, RK)), "dv_t must have shape"),
])
def test_lla2d_decode_checks_operands(over, match):
    rejects(lla.lla2d_decode_attn, match, **dense2d(**over))


def test_rotary_decodes_check_the_rotary_query_and_rows():
    dr = 8
    kw = dense(zk=torch.zeros(B, H, N, RK + dr, dtype=BF16), q_rope=torch.zeros(B, H, dr))
    rejects(lla.lla_decode_attn_rope, "q_rope must be float32",
            **dict(kw, q_rope=torch.zeros(B, H, dr, dtype=BF16)))
    rejects(lla.lla_decode_attn_rope, "zv must have zk's dtype",
            **dict(kw, zv=torch.zeros(B, H, N, RV, dtype=F32)))
    rejects(lla.lla_decode_attn_rope, "contiguous CUDA", **kw)
    kw2 = dense2d(zk=torch.zeros(B, N, RK + dr, dtype=BF16), q_rope=torch.zeros(B, H, dr))
    rejects(lla.lla2d_decode_attn_rope, "q_rope must be", **dict(kw2, q_rope=torch.zeros(B, dr)))
    rejects(lla.lla2d_decode_attn_rope, "contiguous CUDA", **kw2)


def paged(two_d=False, **over):
    P, ps, mb = 6, 4, 3
    pool = (P, ps) if two_d else (P, H, ps)
    a = dict(q=torch.zeros(B, H, D), zk_pages=torch.zeros(*pool, RK, dtype=BF16),
             zv_pages=torch.zeros(*pool, RV, dtype=BF16),
             block_table=torch.zeros(B, mb, dtype=torch.int32),
             seq_lens=torch.zeros(B, dtype=torch.int32), dk_t=torch.zeros(H, D, RK),
             dv_t=torch.zeros(H, D, RV))
    a.update(over)
    return a


@pytest.mark.parametrize("two_d", [False, True])
def test_paged_decodes_check_pools_tables_and_lengths(two_d):
    fn = lla.lla2d_decode_attn_paged if two_d else lla.lla_decode_attn_paged
    pool = (6, 4) if two_d else (6, H, 4)
    rejects(fn, "zv must have zk's dtype",
            **paged(two_d, zv_pages=torch.zeros(*pool, RV, dtype=F32)))
    rejects(fn, "int32", **paged(two_d, block_table=torch.zeros(B, 3, dtype=torch.int64)))
    rejects(fn, "block_table must be", **paged(two_d, block_table=torch.zeros(B + 1, 3,
                                                                              dtype=torch.int32)))
    rejects(fn, "seq_lens must have shape",
            **paged(two_d, seq_lens=torch.zeros(B + 2, dtype=torch.int32)))
    rejects(fn, "disagree", **paged(two_d, zv_pages=torch.zeros(7, *pool[1:], RV, dtype=BF16)))
    rejects(fn, "dk_t must have shape", **paged(two_d, dk_t=torch.zeros(H, D, RK + 8)))
    rejects(fn, "contiguous CUDA", **paged(two_d))
    if not two_d:
        rejects(fn, "H heads", **paged(two_d, zk_pages=torch.zeros(6, H + 1, 4, RK, dtype=BF16),
                                       zv_pages=torch.zeros(6, H + 1, 4, RV, dtype=BF16)))


def test_encode_checks_operands_and_the_output_extent():
    T, Nt, G, dl, r = 2, 3, 2, 64, 8
    x = torch.zeros(T, Nt, G, dl, dtype=BF16)
    w = torch.zeros(G, r, T * dl, dtype=BF16)
    rejects(lla.lla_encode, "x must be bfloat16", x=x.float(), w_down_t=w)
    rejects(lla.lla_encode, "w_down_t must be", x=x, w_down_t=torch.zeros(G, r, dl, dtype=BF16))
    rejects(lla.lla_encode, "w_down_t must be bfloat16", x=x, w_down_t=w.float())
    rejects(lla.lla_encode, "mu must have shape", x=x, w_down_t=w, mu=torch.zeros(G, dl))
    rejects(lla.lla_encode_with_bias, "muw must have shape", x=x, w_down_t=w,
            muw=torch.zeros(G, r + 8))
    rejects(lla.lla_encode_with_bias, "muw must be float32", x=x, w_down_t=w,
            muw=torch.zeros(G, r, dtype=BF16))
    rejects(lla.lla_encode_bias, "mu must have shape", w_down_t=w, mu=torch.zeros(G, T * dl + 8))
    rejects(lla.lla_encode, "contiguous CUDA", x=x, w_down_t=w)


def test_encode_output_strides_must_stay_inside_z(monkeypatch):
    # the extent check itself, on CPU tensors (the placement check is
    # bypassed here so that z's extent is what is tested)
    G, Nt, r = 2, 3, 8
    x = torch.zeros(1, Nt, G, 64, dtype=BF16)
    store = torch.zeros(G, Nt + 1, r, dtype=BF16)
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    _lib._check_z(store[:, 1], x, G, Nt, r, r, (Nt + 1) * r)       # rows 1..3 of each group
    with pytest.raises(lla.LLAError, match="storage holds"):
        _lib._check_z(store[:, 2], x, G, Nt, r, r, (Nt + 1) * r)   # one row past the end
    with pytest.raises(lla.LLAError, match="must be bfloat16"):
        _lib._check_z(store.float(), x, G, Nt, r, r, Nt * r)


def test_merge_checks_parts():
    outs, lses = torch.zeros(3, 4, 5), torch.zeros(3, 4)
    rejects(lla.lla_merge_attn, "without its last axis", out_parts=outs,
            lse_parts=torch.zeros(3, 5))
    rejects(lla.lla_merge_attn, "lse_parts must be float32", out_parts=outs,
            lse_parts=lses.double())
    rejects(lla.lla_merge_attn, "out must have shape", out_parts=outs, lse_parts=lses,
            out=torch.zeros(4, 6))
    rejects(lla.lla_merge_attn, "contiguous CUDA", out_parts=outs, lse_parts=lses)

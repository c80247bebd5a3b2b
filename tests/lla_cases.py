"""Shared builders for the GPU parity tests: seeded inputs on the device, the
same values copied to the host for the oracle, and the tolerance checks."""

from __future__ import annotations

import math

import numpy as np
import torch

from decode_attention_encode_b200 import synth

# Tolerances (max over each checked output tensor):
#   fp32 latents: max |o_gpu - o_ref| <= 1e-4
#   bf16 latents: max |o_gpu - o_ref| / max |o_ref| <= 2e-2
TOL_F32_ABS = 1e-4
TOL_BF16_REL = 2e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of device values for the oracle."""
    return t.detach().to("cpu", torch.float64).numpy()


def make_decode_inputs(B, H, d_h, N, r_k, r_v, dtype, *, n_cap=None, two_d=False, decay=False,
                       mu=False, seed=0, q_scale=1.0, device="cuda"):
    """Seeded inputs of one (layer, loop) decode step on `device`."""
    n_cap = N if n_cap is None else n_cap
    zshape_k = (B, n_cap, r_k) if two_d else (B, H, n_cap, r_k)
    zshape_v = (B, n_cap, r_v) if two_d else (B, H, n_cap, r_v)
    zk = synth.latents(zshape_k, seed + 1, device, decay=decay, dtype=dtype)
    zv = synth.latents(zshape_v, seed + 2, device, decay=decay, dtype=dtype)
    dk = synth.orthonormal(H, d_h, r_k, seed + 3, device)
    dv = synth.orthonormal(H, d_h, r_v, seed + 4, device)
    q = synth.queries((B, H, d_h), d_h, seed + 5, device)
    if q_scale != 1.0:
        q = q * q_scale
    mu_k = synth.normal((H, d_h), seed + 6, device) if mu else None
    mu_v = synth.normal((H, d_h), seed + 7, device) if mu else None
    return dict(q=q, zk=zk, zv=zv, dk=dk, dv=dv, mu_k=mu_k, mu_v=mu_v, N=N)


def sample_units(B, H, n_random=32, seed=0):
    """32 seeded-random (b, h) units plus up to 16 corner units."""
    corners_b = sorted({0, min(1, B - 1), B // 2, B - 1})
    corners_h = sorted({0, min(1, H - 1), H // 2, H - 1})
    units = [(b, h) for b in corners_b for h in corners_h]
    r = np.random.default_rng(seed)
    for _ in range(n_random):
        units.append((int(r.integers(B)), int(r.integers(H))))
    seen, out = set(), []
    for u in units:
        if u not in seen:
            seen.add(u)
            out.append(u)
    return out


def oracle_reference(inp, units, two_d=False, scale=None):
    """Runs the oracle on the given units, reading only those units' data
    back from the device."""
    import oracle  # test infrastructure only

    q = inp["q"]
    d_h = q.shape[-1]
    N = inp["N"]
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    bs = torch.tensor([u[0] for u in units], device=q.device)
    hs = torch.tensor([u[1] for u in units], device=q.device)
    if two_d:
        zk = to_f64(inp["zk"][bs, :N])
        zv = to_f64(inp["zv"][bs, :N])
    else:
        zk = to_f64(inp["zk"][bs, hs, :N])
        zv = to_f64(inp["zv"][bs, hs, :N])
    out, lse = oracle.decode_units(
        to_f64(q[bs, hs]), zk, zv, to_f64(inp["dk"][hs]), to_f64(inp["dv"][hs]),
        None if inp["mu_k"] is None else to_f64(inp["mu_k"][hs]),
        None if inp["mu_v"] is None else to_f64(inp["mu_v"][hs]), scale)
    return out, lse


def compare(out_gpu, lse_gpu, units, ref_out, ref_lse, dtype):
    """Returns (err, lse_err) and asserts the stated tolerance."""
    bs = [u[0] for u in units]
    hs = [u[1] for u in units]
    o = to_f64(out_gpu)[bs, hs]
    diff = np.abs(o - ref_out).max()
    if dtype == torch.float32:
        err = diff
        assert err <= TOL_F32_ABS, f"fp32 max-abs error {err:.3e} > {TOL_F32_ABS}"
    else:
        err = diff / np.abs(ref_out).max()
        assert err <= TOL_BF16_REL, f"bf16 relative error {err:.3e} > {TOL_BF16_REL}"
    lse_err = None
    if lse_gpu is not None:
        lse_err = np.abs(to_f64(lse_gpu)[bs, hs] - ref_lse).max()
    return err, lse_err


def make_paged_inputs(lens, H, d_h, r_k, r_v, dtype, page_size, *, spare=2, mu=False, seed=0,
                      max_blocks=0, device="cuda"):
    """Seeded paged store: a shuffled page pool [P, H, page_size, r] holding
    sequences of the given lengths, with its block table and lengths as
    int32 device arrays."""
    bt, num_pages = synth.page_table(lens, page_size, seed + 11, spare=spare,
                                     max_blocks=max_blocks)
    B = len(lens)
    zk = synth.latents((num_pages, H, page_size, r_k), seed + 1, device, dtype=dtype)
    zv = synth.latents((num_pages, H, page_size, r_v), seed + 2, device, dtype=dtype)
    dk = synth.orthonormal(H, d_h, r_k, seed + 3, device)
    dv = synth.orthonormal(H, d_h, r_v, seed + 4, device)
    q = synth.queries((B, H, d_h), d_h, seed + 5, device)
    mu_k = synth.normal((H, d_h), seed + 6, device) if mu else None
    mu_v = synth.normal((H, d_h), seed + 7, device) if mu else None
    return dict(q=q, zk=zk, zv=zv, dk=dk, dv=dv, mu_k=mu_k, mu_v=mu_v,
                block_table=torch.from_numpy(bt).to(device),
                seq_lens=torch.from_numpy(np.asarray(lens, dtype=np.int32)).to(device))


def oracle_paged_reference(inp, sink=0, window=0, scale=None):
    """The oracle's paged decode on the exact device values."""
    import oracle  # test infrastructure only

    d_h = inp["q"].shape[-1]
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    opt = lambda t: None if t is None else to_f64(t)
    bt = inp["block_table"].cpu().numpy().astype(np.int64)
    return oracle.paged_decode(to_f64(inp["q"]), to_f64(inp["zk"]), to_f64(inp["zv"]), bt,
                               inp["seq_lens"].cpu().numpy(), to_f64(inp["dk"]), to_f64(inp["dv"]),
                               opt(inp["mu_k"]), opt(inp["mu_v"]), scale, sink, window)


def compare_paged(out, lse, ref_out, ref_lse, lens, dtype):
    """Element-wise check of every (b, h): empty sequences exactly 0 / -inf,
    the others within the stated tolerance. Returns (err, lse_err)."""
    o = to_f64(out)
    l = to_f64(lse)
    lens = np.asarray(lens)
    empty = lens == 0
    assert np.all(o[empty] == 0.0) and np.all(np.isneginf(l[empty]))
    full = ~empty
    if not full.any():
        return 0.0, 0.0
    diff = np.abs(o[full] - ref_out[full]).max()
    if dtype == torch.float32:
        err = diff
        assert err <= TOL_F32_ABS, f"fp32 max-abs error {err:.3e} > {TOL_F32_ABS}"
    else:
        err = diff / np.abs(ref_out[full]).max()
        assert err <= TOL_BF16_REL, f"bf16 relative error {err:.3e} > {TOL_BF16_REL}"
    lse_err = np.abs(l[full] - ref_lse[full]).max()
    return err, lse_err


def add_undeclared_pages(inp, extra=2):
    """Moves the page pool into an allocation with `extra` NaN-filled pages
    after the declared ones. The calls see only the declared pool (the
    binding takes num_pages from zk.shape[0]), so a table entry naming one of
    the extra pages is out of range for the library, yet still lands in
    allocated memory: if a device check regressed, the test would see NaN
    output or a wrong status, never an out-of-bounds access. Returns the
    extra pages' indices."""
    P = inp["zk"].shape[0]
    for key in ("zk", "zv"):
        z = inp[key]
        full = torch.full((P + extra,) + tuple(z.shape[1:]), float("nan"), dtype=z.dtype,
                          device=z.device)
        full[:P] = z
        inp[key + "_alloc"] = full
        inp[key] = full[:P]
    return list(range(P, P + extra))


def pad_block_table(inp, bt, fill_page=0):
    """Installs the [B, max_blocks] table `bt` as the first B rows of a
    [B + 1, max_blocks] allocation whose last row names `fill_page` (a
    declared page). A read one block past the end of any row, even the last,
    then stays inside the allocation and names a real page."""
    B, mb = bt.shape
    full = np.full((B + 1, mb), fill_page, dtype=np.int32)
    full[:B] = bt
    t = torch.from_numpy(full).to(inp["q"].device)
    inp["block_table_alloc"] = t
    inp["block_table"] = t[:B]


def check_encoded(z_gpu, z_ref):
    """A latent write against the oracle's Eq. 2: the kernel rounds its fp32
    result to bf16 once (round to nearest even), so each element may differ
    from the exact value by half a bf16 ulp (2^-9 relative) plus fp32
    accumulation error. Checks the stated gate max|z_gpu - z_ref| / max|z_ref|
    <= 2e-2 and the tighter element-wise bound 2^-8 |z_ref| + 1e-4 max|z_ref|.
    Returns the relative error."""
    zg = to_f64(z_gpu) if isinstance(z_gpu, torch.Tensor) else np.asarray(z_gpu)
    scale = np.abs(z_ref).max()
    err = np.abs(zg - z_ref).max() / scale
    assert err <= TOL_BF16_REL, f"relative error {err:.3e}"
    bound = 2.0 ** -8 * np.abs(z_ref) + 1e-4 * scale
    bad = np.abs(zg - z_ref) > bound
    assert not bad.any(), f"{bad.sum()} elements outside rounding bound; max rel {err:.2e}"
    return err

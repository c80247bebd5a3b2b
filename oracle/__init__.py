"""Reference oracle for Looped Latent Attention (LLA) decode and encode.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The CUDA library never
calls it, and it never calls the CUDA library.

Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
Transformers" (O'Neill & Reid, arXiv 2607.15456).

What is here, each in fp64:
  * ``attend``: textbook softmax attention (the uncompressed per-loop path).
  * ``decode_unit`` / ``decode_units`` / ``lla_decode`` / ``lla2d_decode``:
    explicit reconstruction, k_t = W^K_up,t z^K + mu^K_t and the same for V
    (§3 Eq. 3), then textbook attention. Per-head LLA reads one latent per
    (token, head); LLA-2D (§3 "The LLA-2D variant") reads one latent per token
    shared by every head, with decoders per (head, loop).
  * ``decode_unit_absorbed``: the §7 bilinear identities, kept only so the
    tests can compare the two forms by brute force.
  * ``encode``: the latent write c = (x - mu) W_down (§3 Eq. 2) over a
    loop-major stack (§3 Eq. 1); ``paged_write`` places its rows in a paged
    store through a block table (the layout ``paged_decode`` reads).
  * ``svd_init``: §3 "Initialization and conversion": centre by the
    per-loop mean, take the top-r right singular vectors of the stacked-loop
    matrix as W_down, and its loop slices as the initial W_up,t.
  * ``compression_ratio``: §3 Eq. 4.
  * ``rope_rotate`` / ``decode_unit_rope`` / ``lla_decode_rope``: the
    decoupled-RoPE split of §7 (NoPE latent content path plus an explicit
    rotary branch), as attention over concatenated content and rotary keys;
    ``lla2d_decode_rope`` with the key row shared by every head.
  * ``paged2d_decode``: the same gather for the LLA-2D store.
  * ``merge_attn``: the log-sum-exp merge of attention over disjoint parts
    of a context (how a context split over GPUs recombines).
  * ``kept_positions`` / ``paged_decode``: the per-head decode over a paged
    store with per-sequence lengths (a gather of each unit's rows, then the
    explicit-reconstruction unit), with the attention-sink + window eviction
    the pages compose with LLA (§7 "Memory", App. C).

The decode and encode arithmetic lives in ``lla_oracle.c`` (plain C, no
BLAS). ``svd_init`` uses numpy's LAPACK SVD as a library step.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, special cases and invariants the pages fix; none is
left unpinned.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblla_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile ``lla_oracle.c`` into ``liblla_oracle.so`` (gcc, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_attend.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          _dp, _dp, _dp, ctypes.c_double, _dp, _dp]
            lib.oracle_attend.restype = ctypes.c_int
            unit_args = [ctypes.c_int] * 4 + [_dp] * 7 + [ctypes.c_double, _dp, _dp]
            lib.oracle_decode_unit.argtypes = unit_args
            lib.oracle_decode_unit.restype = ctypes.c_int
            lib.oracle_decode_unit_absorbed.argtypes = unit_args
            lib.oracle_decode_unit_absorbed.restype = ctypes.c_int
            lib.oracle_decode_units.argtypes = ([ctypes.c_int] * 5 + [_dp] * 7 +
                                                [ctypes.c_double, _dp, _dp, ctypes.c_int])
            lib.oracle_decode_units.restype = ctypes.c_int
            lib.oracle_encode.argtypes = [ctypes.c_int] * 5 + [_dp] * 4 + [ctypes.c_int]
            lib.oracle_encode.restype = None
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.cast(None, _dp)
    return a.ctypes.data_as(_dp)


def max_threads() -> int:
    """Threads an OpenMP region of the oracle uses by default."""
    return int(_load().oracle_max_threads())


# --------------------------------------------------------------------------
# attention and decode
# --------------------------------------------------------------------------

def attend(q, K, V, scale):
    """Textbook attention of one query over rows of K and V.

    Returns (out [dv], lse) with lse = ln sum_j exp(scale q.K_j)."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    N, d = K.shape
    dv = V.shape[1]
    out = np.zeros(dv)
    lse = np.zeros(1)
    rc = _load().oracle_attend(d, dv, N, _ptr(q), _ptr(K), _ptr(V), float(scale),
                               _ptr(out), _ptr(lse))
    if rc:
        raise ValueError("oracle_attend: empty context or out of memory")
    return out, float(lse[0])


def _unit(fn, q, zk, zv, dk, dv, mu_k, mu_v, scale):
    q, zk, zv, dk, dv = map(_f64, (q, zk, zv, dk, dv))
    mu_k = None if mu_k is None else _f64(mu_k)
    mu_v = None if mu_v is None else _f64(mu_v)
    N, r_k = zk.shape
    r_v = zv.shape[1]
    d = q.shape[0]
    assert dk.shape == (d, r_k) and dv.shape == (d, r_v) and zv.shape[0] == N
    out = np.zeros(d)
    lse = np.zeros(1)
    rc = fn(d, N, r_k, r_v, _ptr(q), _ptr(zk), _ptr(zv), _ptr(dk), _ptr(dv),
            _ptr(mu_k), _ptr(mu_v), float(scale), _ptr(out), _ptr(lse))
    if rc:
        raise ValueError("oracle decode: empty context or out of memory")
    return out, float(lse[0])


def decode_unit(q, zk, zv, dk, dv, mu_k=None, mu_v=None, scale=None):
    """One (batch row, head, layer, loop) unit, explicit reconstruction.

    q [d]; zk [N, r_k]; zv [N, r_v]; dk = W^K_up,t [d, r_k];
    dv = W^V_up,t [d, r_v]; mu_k, mu_v = mu_t slices [d] or None."""
    if scale is None:
        scale = 1.0 / np.sqrt(np.asarray(q).shape[0])
    return _unit(_load().oracle_decode_unit, q, zk, zv, dk, dv, mu_k, mu_v, scale)


def decode_unit_absorbed(q, zk, zv, dk, dv, mu_k=None, mu_v=None, scale=None):
    """The same unit through the §7 absorbed identities (pins only)."""
    if scale is None:
        scale = 1.0 / np.sqrt(np.asarray(q).shape[0])
    return _unit(_load().oracle_decode_unit_absorbed, q, zk, zv, dk, dv, mu_k,
                 mu_v, scale)


def decode_units(q, zk, zv, dk, dv, mu_k=None, mu_v=None, scale=None,
                 nthreads: int = 0):
    """Many independent units at once (OpenMP over units).

    q [U, d]; zk [U, N, r_k]; zv [U, N, r_v]; dk [U, d, r_k];
    dv [U, d, r_v]; mu_k, mu_v [U, d] or None. Returns out [U, d], lse [U]."""
    q, zk, zv, dk, dv = map(_f64, (q, zk, zv, dk, dv))
    mu_k = None if mu_k is None else _f64(mu_k)
    mu_v = None if mu_v is None else _f64(mu_v)
    U, d = q.shape
    N, r_k = zk.shape[1], zk.shape[2]
    r_v = zv.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((U, d))
    lse = np.zeros(U)
    bad = _load().oracle_decode_units(U, d, N, r_k, r_v, _ptr(q), _ptr(zk), _ptr(zv),
                                      _ptr(dk), _ptr(dv), _ptr(mu_k), _ptr(mu_v),
                                      float(scale), _ptr(out), _ptr(lse), int(nthreads))
    if bad:
        raise ValueError(f"oracle decode: {bad} units failed")
    return out, lse


def lla_decode(q, zk, zv, dk, dv, mu_k=None, mu_v=None, scale=None, N=None,
               units=None, nthreads: int = 0):
    """Per-head LLA decode for one (layer, loop) step.

    q [B, H, d]; zk [B, H, n_cap, r_k]; zv [B, H, n_cap, r_v] (first N rows
    used); dk [H, d, r_k]; dv [H, d, r_v]; mu_k, mu_v [H, d] or None.
    ``units`` restricts the work to a list of (b, h) pairs; the result then
    holds one row per listed unit. Returns out, lse."""
    return _decode(q, zk, zv, dk, dv, mu_k, mu_v, scale, N, units, nthreads,
                   shared_latent=False)


def lla2d_decode(q, zk, zv, dk, dv, mu_k=None, mu_v=None, scale=None, N=None,
                 units=None, nthreads: int = 0):
    """LLA-2D decode for one (layer, loop) step: zk [B, n_cap, r_k] and
    zv [B, n_cap, r_v] are shared by every head; dk [H, d, r_k] and
    dv [H, d, r_v] are this loop's per-head decoders."""
    return _decode(q, zk, zv, dk, dv, mu_k, mu_v, scale, N, units, nthreads,
                   shared_latent=True)


def _decode(q, zk, zv, dk, dv, mu_k, mu_v, scale, N, units, nthreads, shared_latent):
    q = np.asarray(q)
    B, H, d = q.shape
    if N is None:
        N = zk.shape[-2]
    if units is None:
        units = [(b, h) for b in range(B) for h in range(H)]
    bs = np.array([u[0] for u in units], dtype=np.int64)
    hs = np.array([u[1] for u in units], dtype=np.int64)
    if shared_latent:
        zk_u = np.asarray(zk)[bs, :N]
        zv_u = np.asarray(zv)[bs, :N]
    else:
        zk_u = np.asarray(zk)[bs, hs, :N]
        zv_u = np.asarray(zv)[bs, hs, :N]
    out, lse = decode_units(
        q[bs, hs], zk_u, zv_u, np.asarray(dk)[hs], np.asarray(dv)[hs],
        None if mu_k is None else np.asarray(mu_k)[hs],
        None if mu_v is None else np.asarray(mu_v)[hs], scale, nthreads)
    if len(units) == B * H and list(units) == [(b, h) for b in range(B) for h in range(H)]:
        return out.reshape(B, H, d), lse.reshape(B, H)
    return out, lse


# --------------------------------------------------------------------------
# decoupled RoPE: a NoPE latent content path plus an explicit rotary branch
# --------------------------------------------------------------------------

def rope_rotate(x, pos, theta=10000.0):
    """Rotary position embedding (Su et al., 2021, the work §3 "RoPE and
    reconstruction" cites) of the last axis of x (even length d) at integer
    positions ``pos`` (broadcast against x[..., 0]): the pair (x_2i, x_2i+1)
    turns by the angle pos * theta^(-2i/d)."""
    x = _f64(x)
    d = x.shape[-1]
    assert d % 2 == 0
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta ** (-np.arange(0, d, 2) / d)
    c, s_ = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s_
    out[..., 1::2] = x[..., 0::2] * s_ + x[..., 1::2] * c
    return out


def decode_unit_rope(q, q_rope, zk, k_rope, zv, dk, dv, mu_k=None, mu_v=None, scale=None):
    """One unit with the decoupled-RoPE split of §7 ("Per-head LLA versus
    LLA-2D at inference": RoPE blocks exact absorption of the positional
    part, so the latent carries the NoPE content and a small explicit rotary
    branch, shared across loops for a token, carries position).

    q [d] content query; q_rope [d_r] this loop's rotated rotary query;
    zk [N, r_k], zv [N, r_v] latents; k_rope [N, d_r] the tokens' rotated
    rotary keys. Scores are scale * (q . khat_j + q_rope . k_rope_j) with
    khat_j = dk zk_j + mu_k (§3 Eq. 3): textbook attention over keys that
    concatenate the reconstructed content key and the rotary key."""
    q, q_rope, zk, k_rope, zv = map(_f64, (q, q_rope, zk, k_rope, zv))
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[0])
    khat = zk @ _f64(dk).T + (0.0 if mu_k is None else _f64(mu_k))
    vhat = zv @ _f64(dv).T + (0.0 if mu_v is None else _f64(mu_v))
    return attend(np.concatenate([q, q_rope]), np.concatenate([khat, k_rope], axis=1), vhat,
                  scale)


def lla_decode_rope(q, q_rope, zk, zv, dk, dv, mu_k=None, mu_v=None, scale=None, N=None,
                    units=None):
    """Per-head decode with the decoupled rotary branch for one (layer,
    loop) step. The store keeps each key row as [latent (r_k) | rotated
    rotary key (d_r)]: zk [B, H, n_cap, r_k + d_r]; q_rope [B, H, d_r].
    Returns out, lse for the listed (b, h) units (all by default)."""
    q, q_rope = np.asarray(q), np.asarray(q_rope)
    B, H, d = q.shape
    d_r = q_rope.shape[-1]
    zk, zv = np.asarray(zk), np.asarray(zv)
    r_k = zk.shape[-1] - d_r
    N = zk.shape[2] if N is None else N
    full = units is None
    units = [(b, h) for b in range(B) for h in range(H)] if full else units
    out = np.zeros((len(units), d))
    lse = np.zeros(len(units))
    for i, (b, h) in enumerate(units):
        out[i], lse[i] = decode_unit_rope(
            q[b, h], q_rope[b, h], zk[b, h, :N, :r_k], zk[b, h, :N, r_k:], zv[b, h, :N],
            np.asarray(dk)[h], np.asarray(dv)[h],
            None if mu_k is None else np.asarray(mu_k)[h],
            None if mu_v is None else np.asarray(mu_v)[h], scale)
    if full:
        return out.reshape(B, H, d), lse.reshape(B, H)
    return out, lse


def lla2d_decode_rope(q, q_rope, zk, zv, dk, dv, mu_k=None, mu_v=None, scale=None, N=None,
                      units=None):
    """LLA-2D decode with the decoupled rotary branch: the key row of each
    token [latent (r_k) | rotated rotary key (d_r)] is shared by every head,
    as MLA shares its rotary key (zk [B, n_cap, r_k + d_r], zv [B, n_cap,
    r_v]); q_rope [B, H, d_r] is each head's rotated rotary query. Per unit
    this is ``decode_unit_rope`` on the shared rows."""
    q, q_rope = np.asarray(q), np.asarray(q_rope)
    B, H, d = q.shape
    d_r = q_rope.shape[-1]
    zk, zv = np.asarray(zk), np.asarray(zv)
    r_k = zk.shape[-1] - d_r
    N = zk.shape[1] if N is None else N
    full = units is None
    units = [(b, h) for b in range(B) for h in range(H)] if full else units
    out = np.zeros((len(units), d))
    lse = np.zeros(len(units))
    for i, (b, h) in enumerate(units):
        out[i], lse[i] = decode_unit_rope(
            q[b, h], q_rope[b, h], zk[b, :N, :r_k], zk[b, :N, r_k:], zv[b, :N],
            np.asarray(dk)[h], np.asarray(dv)[h],
            None if mu_k is None else np.asarray(mu_k)[h],
            None if mu_v is None else np.asarray(mu_v)[h], scale)
    if full:
        return out.reshape(B, H, d), lse.reshape(B, H)
    return out, lse


def merge_attn(outs, lses):
    """Merges attention results over disjoint parts of one context: with
    L = ln sum_r exp(lse_r), out = sum_r exp(lse_r - L) out_r and lse = L.
    Each part's out_r is its softmax-weighted value sum and lse_r its log
    normaliser (the decode calls' outputs), so the merge is exact; a part
    with lse_r = -inf (no token) has weight 0, and if every part is empty
    the result is out = 0, lse = -inf. outs [R, ..., d], lses [R, ...]."""
    outs, lses = _f64(outs), _f64(lses)
    L = np.max(lses, axis=0)
    finite = np.isfinite(L)
    Ls = np.where(finite, L, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - Ls), 0.0)
    tot = w.sum(axis=0)
    lse = np.where(finite, Ls + np.log(np.where(finite, tot, 1.0)), -np.inf)
    out = np.where(finite[..., None], (w[..., None] * outs).sum(axis=0) /
                   np.where(finite, tot, 1.0)[..., None], 0.0)
    return out, lse


# --------------------------------------------------------------------------
# ragged and paged latent stores, sequence-axis eviction
# --------------------------------------------------------------------------

def kept_positions(N, sink=0, window=0):
    """Cached-token positions a sequence of N tokens attends.

    With window > 0 this is the attention-sink + recent-window index set that
    the pages stack on LLA (§7 "Memory"; App. C Table 9: a 260-token budget
    of 4 sink tokens plus a 256-token window): the first ``sink`` tokens and
    the last ``window`` tokens, or all N when N <= sink + window. With
    window <= 0 nothing is evicted and all N positions are kept."""
    N, sink, window = int(N), max(0, int(sink)), int(window)
    if window <= 0 or N <= sink + window:
        return np.arange(N, dtype=np.int64)
    return np.concatenate([np.arange(sink, dtype=np.int64),
                           np.arange(N - window, N, dtype=np.int64)])


def paged_decode(q, zk_pages, zv_pages, block_table, seq_lens, dk, dv, mu_k=None,
                 mu_v=None, scale=None, sink=0, window=0, nthreads: int = 0):
    """Per-head LLA decode over a paged latent store with per-sequence lengths.

    q [B, H, d]; zk_pages [P, H, page_size, r_k]; zv_pages [P, H, page_size,
    r_v]; block_table [B, max_blocks] page indices; seq_lens [B]. Token j of
    sequence b, head h is row j % page_size of head h in page
    block_table[b, j // page_size]. Sequence b attends the positions
    ``kept_positions(seq_lens[b], sink, window)``: each (b, h) unit gathers
    those rows and goes through the explicit-reconstruction unit (§3 Eq. 3,
    then textbook attention). The pages leave attention over an empty set
    undefined; this oracle reads it as no attention mass: out = 0 and
    lse = -inf, the neutral element of a log-sum-exp merge.
    Returns out [B, H, d], lse [B, H]."""
    q = np.asarray(q)
    B, H, d = q.shape
    zk_pages, zv_pages = np.asarray(zk_pages), np.asarray(zv_pages)
    block_table, seq_lens = np.asarray(block_table), np.asarray(seq_lens)
    ps = zk_pages.shape[2]
    out = np.zeros((B, H, d))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        pos = kept_positions(int(seq_lens[b]), sink, window)
        if pos.size == 0:
            continue
        pages = block_table[b, pos // ps]
        rows = pos % ps
        # gathered [n, H, r] -> per-head [H, n, r]
        zk_u = np.transpose(zk_pages[pages, :, rows], (1, 0, 2))
        zv_u = np.transpose(zv_pages[pages, :, rows], (1, 0, 2))
        o, l = decode_units(q[b], zk_u, zv_u, dk, dv, mu_k, mu_v, scale, nthreads)
        out[b], lse[b] = o, l
    return out, lse


def paged2d_decode(q, zk_pages, zv_pages, block_table, seq_lens, dk, dv, mu_k=None, mu_v=None,
                   scale=None, nthreads: int = 0, sink=0, window=0):
    """LLA-2D decode over a paged store with per-sequence lengths.

    zk_pages [P, page_size, r_k], zv_pages [P, page_size, r_v]: one latent
    per token shared by every head (§3 "The LLA-2D variant"); token j of
    sequence b is row j % page_size of page block_table[b, j // page_size].
    Sequence b attends ``kept_positions(seq_lens[b], sink, window)`` (all
    its tokens when window is 0): it gathers those rows and goes through the
    LLA-2D explicit reconstruction; an empty set gives out = 0, lse = -inf
    (the same reading as ``paged_decode``). Returns out [B, H, d], lse [B, H]."""
    q = np.asarray(q)
    B, H, d = q.shape
    zk_pages, zv_pages = np.asarray(zk_pages), np.asarray(zv_pages)
    block_table, seq_lens = np.asarray(block_table), np.asarray(seq_lens)
    ps = zk_pages.shape[1]
    out = np.zeros((B, H, d))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        pos = kept_positions(int(seq_lens[b]), sink, window)
        if pos.size == 0:
            continue
        pages = block_table[b, pos // ps]
        zk = zk_pages[pages, pos % ps][None]
        zv = zv_pages[pages, pos % ps][None]
        o, l = lla2d_decode(q[b:b + 1], zk, zv, dk, dv, mu_k, mu_v, scale, nthreads=nthreads)
        out[b], lse[b] = o[0], l[0]
    return out, lse


# --------------------------------------------------------------------------
# encode and codec initialisation
# --------------------------------------------------------------------------

def encode(x, w, mu=None, nthreads: int = 0):
    """Latent write, Eq. 2: x [T, N, G, d_loop] loop-major; w [G, T*d_loop, r];
    mu [G, T*d_loop] or None. Returns z [G, N, r]. ``nthreads`` > 0 sets the
    OpenMP thread count (as for ``decode_units``)."""
    x, w = _f64(x), _f64(w)
    mu = None if mu is None else _f64(mu)
    T, N, G, d_loop = x.shape
    r = w.shape[2]
    assert w.shape == (G, T * d_loop, r)
    z = np.zeros((G, N, r))
    _load().oracle_encode(T, N, G, d_loop, r, _ptr(x), _ptr(w), _ptr(mu), _ptr(z),
                          int(nthreads))
    return z


def paged_write(pool, z, block_table, positions, seq_idx=None):
    """Places encoded latent rows in a paged store: the write side of the
    paged layout ``paged_decode`` and ``paged2d_decode`` read.

    Token n belongs to sequence s = seq_idx[n] (s = n when seq_idx is None)
    at position p = positions[n]; its row lands in row p % page_size of page
    block_table[s, p // page_size]. pool is [P, G, page_size, r_row] for a
    per-head store (G heads) or [P, page_size, r_row] for LLA-2D (G = 1);
    z is [G, N, r] as ``encode`` returns it, and only the first r values of
    a row (the latent part of a [latent | rotary key] row) are written. A
    token whose sequence index, position or page lies outside the table or
    the pool is not written. Returns (new pool, list of skipped tokens)."""
    pool = np.array(pool, dtype=np.float64, copy=True)
    z = _f64(z)
    block_table = np.asarray(block_table)
    two_d = pool.ndim == 3
    ps = pool.shape[1] if two_d else pool.shape[2]
    G, N, r = z.shape
    n_seq, max_blocks = block_table.shape
    skipped = []
    for n in range(N):
        s = n if seq_idx is None else int(seq_idx[n])
        p = int(positions[n])
        if not (0 <= s < n_seq and 0 <= p < max_blocks * ps):
            skipped.append(n)
            continue
        page = int(block_table[s, p // ps])
        if not 0 <= page < pool.shape[0]:
            skipped.append(n)
            continue
        if two_d:
            pool[page, p % ps, :r] = z[0, n]
        else:
            pool[page, :, p % ps, :r] = z[:, n]
    return pool, skipped


def svd_init(X, r, T):
    """Codec initialisation of §3 "Initialization and conversion".

    X [n_cal, T*d] holds one stacked-loop vector per row (Eq. 1). Returns
    (w_down [T*d, r], w_up [T, d, r], mu [T*d]): mu is the column mean, which
    is the per-loop mean of every loop stacked; w_down holds the top-r right
    singular vectors of the centred matrix; w_up[t] is w_down's loop-t row
    slice, so Eq. 3 gives xhat_t = c w_up[t]^T + mu_t."""
    X = _f64(X)
    n, K = X.shape
    assert K % T == 0
    d = K // T
    mu = X.mean(axis=0)
    _, _, vt = np.linalg.svd(X - mu, full_matrices=False)
    w_down = np.ascontiguousarray(vt[:r].T)
    w_up = np.ascontiguousarray(w_down.reshape(T, d, r))
    return w_down, w_up, mu


def reconstruct(z, w_up, mu=None):
    """Eq. 3 for every loop: z [..., r], w_up [T, d, r], mu [T*d] or None.
    Returns xhat [..., T, d]."""
    z = _f64(z)
    w_up = _f64(w_up)
    T, d, r = w_up.shape
    xhat = np.einsum("tdr,...r->...td", w_up, z)
    if mu is not None:
        xhat = xhat + _f64(mu).reshape(T, d)
    return xhat


def compression_ratio(T, d_head, r_k, r_v, H=1, two_d=False):
    """Eq. 4: per-head rho = 2 T H d_head / ((r_k + r_v) H) = 2 T d_head /
    (r_k + r_v). LLA-2D stores (r_k + r_v) scalars per token and layer for
    all H heads, so its ratio is 2 T H d_head / (r_k + r_v)."""
    if two_d:
        return 2.0 * T * H * d_head / (r_k + r_v)
    return (2.0 * T * H * d_head) / ((r_k + r_v) * H)

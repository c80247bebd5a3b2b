"""ctypes binding of liblla.so (the C ABI declared in include/lla.h).

Argument marshalling only: every step of the decode and encode paths runs in
the library's CUDA kernels. Torch supplies device memory and the current
stream. If the library cannot be loaded the calls raise; there is no
fallback.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

from . import build as _build

LLA_OK = 0
LLA_ERR_INVALID_ARG = 1
LLA_ERR_UNSUPPORTED = 2
LLA_ERR_WORKSPACE = 3
LLA_ERR_CUDA = 4

LLA_F32 = 0
LLA_BF16 = 1

LLA_DEVICE_WAIT_TIMEOUT = 0x1
LLA_DEVICE_BAD_PAGED_INPUT = 0x2
LLA_DEVICE_PAGED_PLAN_MISMATCH = 0x4
LLA_DEVICE_OUT_OF_BOUNDS = 0x8

# Every symbol include/lla.h declares.
EXPORTS = (
    "lla_status_string", "lla_last_error", "lla_version", "lla_device_status",
    "lla_selftest_wait_timeout", "lla_set_timing_events", "lla_merge_attn",
    "lla_decode_attn_workspace", "lla_decode_attn", "lla_decode_attn_noalloc",
    "lla_decode_attn_rope",
    "lla_decode_attn_paged_workspace", "lla_decode_attn_paged",
    "lla_decode_attn_paged_plan", "lla_decode_attn_paged_planned",
    "lla2d_decode_attn_workspace", "lla2d_decode_attn", "lla2d_decode_attn_rope",
    "lla2d_decode_attn_paged_workspace", "lla2d_decode_attn_paged",
    "lla2d_decode_attn_paged_plan", "lla2d_decode_attn_paged_planned",
    "lla_encode", "lla_encode_bias", "lla_encode_with_bias_workspace", "lla_encode_with_bias",
    "lla_encode_paged",
)

_lock = threading.Lock()
_lib = None


class LLAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_c_int, _c_size, _c_float, _c_ll, _vp = (ctypes.c_int, ctypes.c_size_t, ctypes.c_float,
                                         ctypes.c_longlong, ctypes.c_void_p)

_SIGS = {
    "lla_status_string": ([_c_int], ctypes.c_char_p),
    "lla_last_error": ([], ctypes.c_char_p),
    "lla_version": ([], _c_int),
    "lla_device_status": ([ctypes.POINTER(ctypes.c_uint), _c_int], _c_int),
    "lla_set_timing_events": ([_vp, _vp], None),
    "lla_selftest_wait_timeout": ([ctypes.c_uint, _vp], _c_int),
    "lla_merge_attn": ([_vp, _vp, _c_int, _c_ll, _c_int, _vp, _vp, _vp], _c_int),
    "lla_decode_attn_workspace": ([_c_int] * 5, _c_size),
    "lla_decode_attn_rope": ([_vp, _vp, _vp, _vp, _c_int] + [_c_int] * 8 + [_vp] * 4 +
                             [_c_float, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "lla_decode_attn_paged_workspace": ([_c_int] * 4, _c_size),
    "lla_decode_attn_paged": ([_vp, _vp, _vp, _c_int] + [_c_int] * 7 + [_vp, _c_int, _vp] +
                              [_c_int] * 2 + [_vp] * 4 + [_c_float, _vp, _vp, _vp, _c_size, _vp],
                              _c_int),
    "lla_decode_attn_paged_plan": ([_c_int] * 7 + [_vp, _c_int, _vp, _c_int, _c_int, _vp,
                                                    _c_size, _vp], _c_int),
    "lla2d_decode_attn_paged_plan": ([_c_int] * 6 + [_vp, _c_int, _vp, _c_int, _c_int, _vp,
                                                      _c_size, _vp], _c_int),
    "lla2d_decode_attn_workspace": ([_c_int] * 5, _c_size),
    "lla2d_decode_attn_rope": ([_vp, _vp, _vp, _vp, _c_int] + [_c_int] * 8 + [_vp] * 4 +
                               [_c_float, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "lla2d_decode_attn_paged_workspace": ([_c_int] * 4, _c_size),
    "lla_decode_attn_paged_planned": ([_vp, _vp, _vp, _c_int] + [_c_int] * 7 +
                                      [_vp, _c_int, _vp] + [_c_int] * 2 + [_vp] * 4 +
                                      [_c_float, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "lla2d_decode_attn_paged_planned": ([_vp, _vp, _vp, _c_int] + [_c_int] * 7 +
                                        [_vp, _c_int, _vp] + [_c_int] * 2 + [_vp] * 4 +
                                        [_c_float, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "lla2d_decode_attn_paged": ([_vp, _vp, _vp, _c_int] + [_c_int] * 7 + [_vp, _c_int, _vp] +
                                [_c_int] * 2 + [_vp] * 4 + [_c_float, _vp, _vp, _vp, _c_size, _vp],
                                _c_int),
    "lla_decode_attn": ([_vp, _vp, _vp, _c_int] + [_c_int] * 7 + [_vp] * 4 +
                        [_c_float, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "lla_decode_attn_noalloc": ([_vp, _vp, _vp, _c_int] + [_c_int] * 7 + [_vp] * 4 +
                                [_c_float, _vp, _vp, _vp], _c_int),
    "lla2d_decode_attn": ([_vp, _vp, _vp, _c_int] + [_c_int] * 7 + [_vp] * 4 +
                          [_c_float, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "lla_encode": ([_vp, _c_int] + [_c_int] * 5 + [_vp, _vp, _vp, _c_ll, _c_ll, _vp], _c_int),
    "lla_encode_bias": ([_vp, _vp, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
    "lla_encode_with_bias_workspace": ([_c_int] * 5, _c_size),
    "lla_encode_with_bias": ([_vp, _c_int] + [_c_int] * 5 + [_vp, _vp, _vp, _c_ll, _c_ll, _vp,
                                                              _c_size, _vp], _c_int),
    "lla_encode_paged": ([_vp, _c_int] + [_c_int] * 5 + [_vp, _vp, _vp, _c_ll, _c_ll, _c_ll,
                                                          _c_int, _c_int, _vp, _c_int, _c_int,
                                                          _vp, _vp, _vp, _c_size, _vp], _c_int),
}


def library_variant() -> str:
    """The build this process loads: "release" (liblla.so), or "check"
    (liblla_check.so, the bounds-check build) when LLA_LIBRARY_VARIANT=check."""
    return os.environ.get("LLA_LIBRARY_VARIANT", "release") or "release"


def library_path() -> str:
    return _build.lib_path(library_variant())


def lib(build_if_missing: bool = True):
    """Loads the library (building it with nvcc if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            variant = library_variant()
            path = (_build.build(variant=variant) if build_if_missing
                    else _build.lib_path(variant))
            if not os.path.exists(path):
                raise LLAError(LLA_ERR_CUDA, f"library not found at {path}")
            h = ctypes.CDLL(path)
            for name, (args, res) in _SIGS.items():
                fn = getattr(h, name)
                fn.argtypes = args
                fn.restype = res
            _lib = h
    return _lib


def _check(status: int):
    if status != LLA_OK:
        h = lib()
        raise LLAError(status, f"{h.lla_status_string(status).decode()}: "
                               f"{h.lla_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return LLA_BF16
    if t.dtype == torch.float32:
        return LLA_F32
    raise LLAError(LLA_ERR_INVALID_ARG, f"unsupported latent dtype {t.dtype}")


def _need_cuda(*ts):
    """Every given tensor is a contiguous CUDA tensor on one device, and that
    device is the current one (the call's stream and kernels run there)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise LLAError(LLA_ERR_INVALID_ARG, "tensors must be contiguous CUDA tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise LLAError(LLA_ERR_INVALID_ARG, f"tensors on {dev} and {t.device}: use one device")
    if dev is not None and dev.index != torch.cuda.current_device():
        raise LLAError(LLA_ERR_INVALID_ARG, f"tensors are on {dev} but the current device is "
                                            f"cuda:{torch.cuda.current_device()}")


def _expect(cond, msg):
    if not cond:
        raise LLAError(LLA_ERR_INVALID_ARG, msg)


def _shape(name, t, shape):
    """t has exactly this shape (None: t is optional and absent)."""
    if t is None:
        return
    _expect(tuple(t.shape) == tuple(shape),
            f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _f32(name, t, shape=None):
    if t is None:
        return
    _expect(t.dtype == torch.float32, f"{name} must be float32, got {t.dtype}")
    if shape is not None:
        _shape(name, t, shape)


def _same_latent_type(zk, zv):
    _dtype_code(zk)
    _expect(zv.dtype == zk.dtype, f"zv must have zk's dtype {zk.dtype}, got {zv.dtype}")


def _check_query_side(q, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, r_k, r_v, q_rope=None):
    """fp32 operands of a decode call against q [B,H,d_h]: decoders
    [H,d_h,r_k] and [H,d_h,r_v], means [H,d_h], out [B,H,d_h], lse [B,H],
    and the rotary query [B,H,d_r] when there is one."""
    _f32("q", q)
    _expect(q.dim() == 3, f"q must be [B, H, d_h], got {tuple(q.shape)}")
    B, H, d_h = q.shape
    if q_rope is not None:
        _f32("q_rope", q_rope)
        _expect(q_rope.dim() == 3 and tuple(q_rope.shape[:2]) == (B, H),
                f"q_rope must be [B, H, d_r], got {tuple(q_rope.shape)}")
    _f32("dk_t", dk_t, (H, d_h, r_k))
    _f32("dv_t", dv_t, (H, d_h, r_v))
    _f32("mu_k_t", mu_k_t, (H, d_h))
    _f32("mu_v_t", mu_v_t, (H, d_h))
    _f32("out", out, (B, H, d_h))
    _f32("lse", lse, (B, H))


def _check_decode(q, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, *, two_d, r_k=None,
                  q_rope=None):
    """Shapes and element types of a dense decode call's operands, checked
    before anything reaches the library (whose kernels trust them): latents
    [B,(H,)n_cap,r] of one type matching q [B,H,d_h], plus the fp32 operands
    of _check_query_side. r_k, when given, is the latent part of a key row
    that also holds a rotary key."""
    _expect(q.dim() == 3, f"q must be [B, H, d_h], got {tuple(q.shape)}")
    B, H = q.shape[0], q.shape[1]
    _same_latent_type(zk, zv)
    lead = 2 if two_d else 3
    _expect(zk.dim() == lead + 1 and zv.dim() == lead + 1,
            "latents must be [B, n_cap, r]" if two_d else "latents must be [B, H, n_cap, r]")
    want = (B, zk.shape[-2]) if two_d else (B, H, zk.shape[-2])
    _expect(tuple(zk.shape[:lead]) == want and tuple(zv.shape[:lead]) == want,
            f"zk {tuple(zk.shape)} and zv {tuple(zv.shape)} do not match q {tuple(q.shape)}")
    _check_query_side(q, dk_t, dv_t, mu_k_t, mu_v_t, out, lse,
                      zk.shape[-1] if r_k is None else r_k, zv.shape[-1], q_rope)


def _check_paged(q, zk_pages, zv_pages, block_table, seq_lens, *, two_d):
    """Page pools [P,(H,)page_size,r] of one latent type, an int32
    [B,max_blocks] block table and int32 [B] lengths."""
    _expect(q.dim() == 3, f"q must be [B, H, d_h], got {tuple(q.shape)}")
    B = q.shape[0]
    _same_latent_type(zk_pages, zv_pages)
    lead = 2 if two_d else 3
    _expect(zk_pages.dim() == lead + 1 and zv_pages.dim() == lead + 1,
            "page pools must be [P, page_size, r]" if two_d
            else "page pools must be [P, H, page_size, r]")
    _expect(tuple(zk_pages.shape[:lead]) == tuple(zv_pages.shape[:lead]),
            f"zk_pages {tuple(zk_pages.shape)} and zv_pages {tuple(zv_pages.shape)} disagree")
    if not two_d:
        _expect(zk_pages.shape[1] == q.shape[1], "page pools must hold q's H heads")
    _expect(block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32,
            "block_table and seq_lens must be int32")
    _expect(block_table.dim() == 2 and block_table.shape[0] == B,
            f"block_table must be [B, max_blocks] with B = {B}, got {tuple(block_table.shape)}")
    _shape("seq_lens", seq_lens, (B,))


def device_status(clear: bool = False) -> int:
    v = ctypes.c_uint(0)
    _check(lib().lla_device_status(ctypes.byref(v), int(clear)))
    return v.value


class kernel_timer:
    """Context manager that times the main kernel of each library call made
    inside it with CUDA events (lla_set_timing_events). After the block,
    `ms` is the elapsed time of the last timed call's main kernel."""

    def __init__(self):
        self.begin = torch.cuda.Event(enable_timing=True)
        self.end = torch.cuda.Event(enable_timing=True)
        # torch creates the underlying CUDA events on first record
        stream = torch.cuda.current_stream()
        self.begin.record(stream)
        self.end.record(stream)
        self.end.synchronize()
        self.ms = None

    def __enter__(self):
        lib().lla_set_timing_events(ctypes.c_void_p(self.begin.cuda_event),
                                    ctypes.c_void_p(self.end.cuda_event))
        return self

    def __exit__(self, *exc):
        lib().lla_set_timing_events(None, None)
        self.end.synchronize()
        self.ms = self.begin.elapsed_time(self.end)
        return False


class launch_timers:
    """Times the main kernel of each of up to n library calls made inside
    it, with no synchronisation between the calls: next() before a call
    points the library's timing hook at a fresh pair of CUDA events. After
    the block, `ms` lists the elapsed time of every timed kernel."""

    def __init__(self, n):
        stream = torch.cuda.current_stream()
        self.pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(n)]
        for b, e in self.pairs:  # torch creates the CUDA events on first record
            b.record(stream)
            e.record(stream)
        stream.synchronize()
        self.used = 0
        self.ms = None

    def next(self):
        _expect(self.used < len(self.pairs), "launch_timers: more calls than event pairs")
        b, e = self.pairs[self.used]
        self.used += 1
        lib().lla_set_timing_events(ctypes.c_void_p(b.cuda_event), ctypes.c_void_p(e.cuda_event))

    def pause(self):
        """Calls made until the next next() are not timed."""
        lib().lla_set_timing_events(None, None)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        lib().lla_set_timing_events(None, None)
        torch.cuda.synchronize()
        self.ms = [b.elapsed_time(e) for b, e in self.pairs[:self.used]]
        return False


def lla_decode_attn_workspace(B, H, N, r_k, r_v) -> int:
    return int(lib().lla_decode_attn_workspace(B, H, N, r_k, r_v))


def lla2d_decode_attn_workspace(B, H, N, r_k, r_v) -> int:
    return int(lib().lla2d_decode_attn_workspace(B, H, N, r_k, r_v))


def _decode(fn_name, ws_name, q, zk, zv, dk_t, dv_t, N, mu_k_t, mu_v_t, scale, out, lse,
            workspace, stream, want_lse, two_d):
    _check_decode(q, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, two_d=two_d)
    _need_cuda(q, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, workspace)
    B, H, d_h = q.shape
    if two_d:
        n_cap, r_k = zk.shape[1], zk.shape[2]
        r_v = zv.shape[2]
    else:
        n_cap, r_k = zk.shape[2], zk.shape[3]
        r_v = zv.shape[3]
    if N is None:
        N = n_cap
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    if out is None:
        out = torch.empty((B, H, d_h), device=q.device, dtype=torch.float32)
    if lse is None and want_lse:
        lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    h = lib()
    need = int(getattr(h, ws_name)(B, H, N, r_k, r_v))
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    st = getattr(h, fn_name)(_ptr(q), _ptr(zk), _ptr(zv), _dtype_code(zk), B, H, d_h, N, n_cap,
                             r_k, r_v, _ptr(dk_t), _ptr(dv_t), _ptr(mu_k_t), _ptr(mu_v_t),
                             float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out, lse


def lla_decode_attn(q, zk, zv, dk_t, dv_t, N=None, mu_k_t=None, mu_v_t=None, scale=None,
                    out=None, lse=None, workspace=None, stream=None, want_lse=True):
    """Per-head absorbed decode for one (layer, loop) step.

    q [B,H,d_h] fp32; zk [B,H,n_cap,r_k], zv [B,H,n_cap,r_v] bf16 or fp32;
    dk_t [H,d_h,r_k], dv_t [H,d_h,r_v] fp32; mu_k_t, mu_v_t [H,d_h] or None.
    Returns (out [B,H,d_h], lse [B,H] or None)."""
    return _decode("lla_decode_attn", "lla_decode_attn_workspace", q, zk, zv, dk_t, dv_t, N,
                   mu_k_t, mu_v_t, scale, out, lse, workspace, stream, want_lse, two_d=False)


def lla_decode_attn_noalloc(q, zk, zv, dk_t, dv_t, N=None, mu_k_t=None, mu_v_t=None, scale=None,
                            out=None, lse=None, stream=None, want_lse=True):
    """Per-head decode like lla_decode_attn, for callers that cannot allocate
    device memory: the library uses its own fixed scratch array instead of a
    workspace (see include/lla.h for the size limit and the ordering rule).
    Only `out` and `lse` are allocated here when not given."""
    _check_decode(q, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, two_d=False)
    _need_cuda(q, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse)
    B, H, d_h = q.shape
    n_cap, r_k = zk.shape[2], zk.shape[3]
    r_v = zv.shape[3]
    N = n_cap if N is None else N
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    if out is None:
        out = torch.empty((B, H, d_h), device=q.device, dtype=torch.float32)
    if lse is None and want_lse:
        lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    st = lib().lla_decode_attn_noalloc(_ptr(q), _ptr(zk), _ptr(zv), _dtype_code(zk), B, H, d_h,
                                       N, n_cap, r_k, r_v, _ptr(dk_t), _ptr(dv_t), _ptr(mu_k_t),
                                       _ptr(mu_v_t), float(scale), _ptr(out), _ptr(lse),
                                       _stream(stream))
    _check(st)
    return out, lse


def lla_decode_attn_rope(q, q_rope, zk, zv, dk_t, dv_t, N=None, mu_k_t=None, mu_v_t=None,
                         scale=None, out=None, lse=None, workspace=None, stream=None,
                         want_lse=True):
    """Per-head decode with the decoupled rotary branch: zk [B,H,n_cap,r_k+d_r]
    holds each token's latent followed by its rotated rotary key; q_rope
    [B,H,d_r] fp32 is this loop's rotated rotary query; dk_t [H,d_h,r_k].
    Returns (out [B,H,d_h], lse [B,H] or None)."""
    _expect(q.dim() == 3 and q_rope.dim() == 3, "q and q_rope must be [B, H, d_h] and [B, H, d_r]")
    B, H, d_h = q.shape
    d_r = q_rope.shape[2]
    n_cap, rq = zk.shape[2], zk.shape[3]
    r_k, r_v = dk_t.shape[2], zv.shape[3]
    if rq != r_k + d_r:
        raise LLAError(LLA_ERR_INVALID_ARG, "zk rows must hold r_k + d_r values")
    _check_decode(q, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, two_d=False, r_k=r_k,
                  q_rope=q_rope)
    _need_cuda(q, q_rope, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, workspace)
    N = n_cap if N is None else N
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    if out is None:
        out = torch.empty((B, H, d_h), device=q.device, dtype=torch.float32)
    if lse is None and want_lse:
        lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    h = lib()
    need = int(h.lla_decode_attn_workspace(B, H, N, rq, r_v))
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    st = h.lla_decode_attn_rope(_ptr(q), _ptr(q_rope), _ptr(zk), _ptr(zv), _dtype_code(zk), B, H,
                                d_h, d_r, N, n_cap, r_k, r_v, _ptr(dk_t), _ptr(dv_t),
                                _ptr(mu_k_t), _ptr(mu_v_t), float(scale), _ptr(out), _ptr(lse),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check(st)
    return out, lse


def lla_decode_attn_paged_workspace(B, H, r_k, r_v):
    return int(lib().lla_decode_attn_paged_workspace(B, H, r_k, r_v))


def lla_decode_attn_paged(q, zk_pages, zv_pages, block_table, seq_lens, dk_t, dv_t, mu_k_t=None,
                          mu_v_t=None, scale=None, sink=0, window=0, out=None, lse=None,
                          workspace=None, stream=None, want_lse=True, planned=False):
    """Per-head absorbed decode over a paged store with per-sequence lengths.

    q [B,H,d_h] fp32; zk_pages [P,H,page_size,r_k], zv_pages [P,H,page_size,r_v]
    bf16 or fp32; block_table [B,max_blocks] int32 and seq_lens [B] int32 on
    the device; sink, window: the eviction set (window 0 keeps every token).
    With planned=True this is lla_decode_attn_paged_planned: it reuses the
    plan that lla_decode_attn_paged_plan left in `workspace` (required).
    Returns (out [B,H,d_h], lse [B,H] or None)."""
    _check_paged(q, zk_pages, zv_pages, block_table, seq_lens, two_d=False)
    _check_query_side(q, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, zk_pages.shape[-1],
                      zv_pages.shape[-1])
    _need_cuda(q, zk_pages, zv_pages, block_table, seq_lens, dk_t, dv_t, mu_k_t, mu_v_t, out,
               lse, workspace)
    B, H, d_h = q.shape
    num_pages, page_size, r_k = zk_pages.shape[0], zk_pages.shape[2], zk_pages.shape[3]
    r_v = zv_pages.shape[3]
    max_blocks = block_table.shape[1]
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    if out is None:
        out = torch.empty((B, H, d_h), device=q.device, dtype=torch.float32)
    if lse is None and want_lse:
        lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    h = lib()
    need = int(h.lla_decode_attn_paged_workspace(B, H, r_k, r_v))
    _expect(workspace is not None or not planned, "a planned call needs the plan's workspace")
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    fn = h.lla_decode_attn_paged_planned if planned else h.lla_decode_attn_paged
    st = fn(_ptr(q), _ptr(zk_pages), _ptr(zv_pages), _dtype_code(zk_pages),
                                 B, H, d_h, r_k, r_v, page_size, num_pages, _ptr(block_table),
                                 max_blocks, _ptr(seq_lens), int(sink), int(window), _ptr(dk_t),
                                 _ptr(dv_t), _ptr(mu_k_t), _ptr(mu_v_t), float(scale), _ptr(out),
                                 _ptr(lse), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out, lse


def _paged_plan(two_d, zk_pages, zv_pages, block_table, seq_lens, H, workspace, sink, window,
                stream):
    _same_latent_type(zk_pages, zv_pages)
    lead = 2 if two_d else 3
    _expect(zk_pages.dim() == lead + 1 and zv_pages.dim() == lead + 1 and
            tuple(zk_pages.shape[:lead]) == tuple(zv_pages.shape[:lead]),
            "page pools must be [P, page_size, r]" if two_d else "page pools must be [P, H, page_size, r]")
    _expect(block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32,
            "block_table and seq_lens must be int32")
    _expect(block_table.dim() == 2, "block_table must be [B, max_blocks]")
    B = block_table.shape[0]
    _shape("seq_lens", seq_lens, (B,))
    _expect(workspace is not None, "the plan is written into `workspace`; pass the one the "
                                   "planned calls will use")
    _need_cuda(zk_pages, zv_pages, block_table, seq_lens, workspace)
    P, ps = zk_pages.shape[0], zk_pages.shape[-2]
    r_k, r_v = zk_pages.shape[-1], zv_pages.shape[-1]
    ws_bytes = workspace.numel() * workspace.element_size()
    h = lib()
    if two_d:
        st = h.lla2d_decode_attn_paged_plan(B, H, r_k, r_v, ps, P, _ptr(block_table),
                                            block_table.shape[1], _ptr(seq_lens), int(sink),
                                            int(window), _ptr(workspace), ws_bytes,
                                            _stream(stream))
    else:
        st = h.lla_decode_attn_paged_plan(_dtype_code(zk_pages), B, zk_pages.shape[1], r_k, r_v,
                                          ps, P, _ptr(block_table), block_table.shape[1],
                                          _ptr(seq_lens), int(sink), int(window), _ptr(workspace),
                                          ws_bytes, _stream(stream))
    _check(st)
    return workspace


def lla_decode_attn_paged_plan(zk_pages, zv_pages, block_table, seq_lens, workspace, sink=0,
                               window=0, stream=None):
    """Plans a per-head paged decode step once: writes the plan of the
    lengths and table into `workspace` (sized by
    lla_decode_attn_paged_workspace) for later
    lla_decode_attn_paged(..., planned=True) calls. Returns workspace."""
    return _paged_plan(False, zk_pages, zv_pages, block_table, seq_lens, None, workspace, sink,
                       window, stream)


def lla_decode_attn_paged_planned(*args, **kw):
    """lla_decode_attn_paged on the plan already in `workspace`."""
    return lla_decode_attn_paged(*args, planned=True, **kw)


def lla2d_decode_attn_paged_plan(zk_pages, zv_pages, block_table, seq_lens, H, workspace, sink=0,
                                 window=0, stream=None):
    """The LLA-2D counterpart of lla_decode_attn_paged_plan (H heads)."""
    return _paged_plan(True, zk_pages, zv_pages, block_table, seq_lens, H, workspace, sink,
                       window, stream)


def lla2d_decode_attn_paged_planned(*args, **kw):
    """lla2d_decode_attn_paged on the plan already in `workspace`."""
    return lla2d_decode_attn_paged(*args, planned=True, **kw)


def lla2d_decode_attn_rope(q, q_rope, zk, zv, dk_t, dv_t, N=None, mu_k_t=None, mu_v_t=None,
                           scale=None, out=None, lse=None, workspace=None, stream=None,
                           want_lse=True):
    """LLA-2D decode with the decoupled rotary branch: zk [B,n_cap,r_k+d_r]
    holds each token's latent followed by its rotated rotary key (shared by
    every head); q_rope [B,H,d_r]; dk_t [H,d_h,r_k]. Returns (out, lse)."""
    _expect(q.dim() == 3 and q_rope.dim() == 3, "q and q_rope must be [B, H, d_h] and [B, H, d_r]")
    B, H, d_h = q.shape
    d_r = q_rope.shape[2]
    n_cap, rq = zk.shape[1], zk.shape[2]
    r_k, r_v = dk_t.shape[2], zv.shape[2]
    if rq != r_k + d_r:
        raise LLAError(LLA_ERR_INVALID_ARG, "zk rows must hold r_k + d_r values")
    _check_decode(q, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, two_d=True, r_k=r_k,
                  q_rope=q_rope)
    _need_cuda(q, q_rope, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, workspace)
    N = n_cap if N is None else N
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    if out is None:
        out = torch.empty((B, H, d_h), device=q.device, dtype=torch.float32)
    if lse is None and want_lse:
        lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    h = lib()
    need = int(h.lla2d_decode_attn_workspace(B, H, N, rq, r_v))
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    st = h.lla2d_decode_attn_rope(_ptr(q), _ptr(q_rope), _ptr(zk), _ptr(zv), _dtype_code(zk), B,
                                  H, d_h, d_r, N, n_cap, r_k, r_v, _ptr(dk_t), _ptr(dv_t),
                                  _ptr(mu_k_t), _ptr(mu_v_t), float(scale), _ptr(out), _ptr(lse),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream))
    _check(st)
    return out, lse


def lla2d_decode_attn_paged_workspace(B, H, r_k, r_v):
    return int(lib().lla2d_decode_attn_paged_workspace(B, H, r_k, r_v))


def lla2d_decode_attn_paged(q, zk_pages, zv_pages, block_table, seq_lens, dk_t, dv_t,
                            mu_k_t=None, mu_v_t=None, scale=None, sink=0, window=0, out=None,
                            lse=None, workspace=None, stream=None, want_lse=True, planned=False):
    """LLA-2D absorbed decode over a paged store: zk_pages [P,page_size,r_k],
    zv_pages [P,page_size,r_v] bf16 shared by every head, page_size a
    multiple of 64; block_table [B,max_blocks] and seq_lens [B] int32 on
    the device. planned=True: lla2d_decode_attn_paged_planned on the plan in
    `workspace`. Returns (out [B,H,d_h], lse [B,H] or None)."""
    _check_paged(q, zk_pages, zv_pages, block_table, seq_lens, two_d=True)
    _check_query_side(q, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, zk_pages.shape[-1],
                      zv_pages.shape[-1])
    _need_cuda(q, zk_pages, zv_pages, block_table, seq_lens, dk_t, dv_t, mu_k_t, mu_v_t, out,
               lse, workspace)
    B, H, d_h = q.shape
    num_pages, page_size, r_k = zk_pages.shape
    r_v = zv_pages.shape[2]
    max_blocks = block_table.shape[1]
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    if out is None:
        out = torch.empty((B, H, d_h), device=q.device, dtype=torch.float32)
    if lse is None and want_lse:
        lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    h = lib()
    need = int(h.lla2d_decode_attn_paged_workspace(B, H, r_k, r_v))
    _expect(workspace is not None or not planned, "a planned call needs the plan's workspace")
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    fn = h.lla2d_decode_attn_paged_planned if planned else h.lla2d_decode_attn_paged
    st = fn(_ptr(q), _ptr(zk_pages), _ptr(zv_pages),
                                   _dtype_code(zk_pages), B, H, d_h, r_k, r_v, page_size,
                                   num_pages, _ptr(block_table), max_blocks, _ptr(seq_lens),
                                   int(sink), int(window), _ptr(dk_t), _ptr(dv_t), _ptr(mu_k_t),
                                   _ptr(mu_v_t),
                                   float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out, lse


def lla2d_decode_attn(q, zk, zv, dk_t, dv_t, N=None, mu_k_t=None, mu_v_t=None, scale=None,
                      out=None, lse=None, workspace=None, stream=None, want_lse=True):
    """LLA-2D absorbed decode for one (layer, loop) step: zk [B,n_cap,r_k],
    zv [B,n_cap,r_v] bf16, shared by every head."""
    return _decode("lla2d_decode_attn", "lla2d_decode_attn_workspace", q, zk, zv, dk_t, dv_t,
                   N, mu_k_t, mu_v_t, scale, out, lse, workspace, stream, want_lse, two_d=True)


def _check_encode(x, w_down_t, mu=None, muw=None):
    """x [T,N,G,d_loop] bf16, w_down_t [G,r,T*d_loop] bf16, mu [G,T*d_loop]
    fp32, muw [G,r] fp32."""
    _expect(x.dtype == torch.bfloat16, f"x must be bfloat16, got {x.dtype}")
    _expect(x.dim() == 4, f"x must be [T, N, G, d_loop], got {tuple(x.shape)}")
    T, N, G, d_loop = x.shape
    _expect(w_down_t.dtype == torch.bfloat16, f"w_down_t must be bfloat16, got {w_down_t.dtype}")
    _expect(w_down_t.dim() == 3 and w_down_t.shape[0] == G and w_down_t.shape[2] == T * d_loop,
            f"w_down_t must be [G, r, T*d_loop] = [{G}, r, {T * d_loop}], "
            f"got {tuple(w_down_t.shape)}")
    r = w_down_t.shape[1]
    _f32("mu", mu, (G, T * d_loop))
    _f32("muw", muw, (G, r))


def _check_z(z, x, G, N, r, z_row_stride, z_group_stride):
    """z is a bfloat16 CUDA tensor on x's device whose storage holds every
    row the strides address (z may be a strided view into a larger store;
    the library writes through its data pointer)."""
    _expect(z.dtype == torch.bfloat16, f"z must be bfloat16, got {z.dtype}")
    _expect(z.is_cuda and z.device == x.device, f"z must be on {x.device}")
    last = (G - 1) * int(z_group_stride) + (N - 1) * int(z_row_stride) + r
    have = z.untyped_storage().nbytes() // 2 - z.storage_offset()
    _expect(last <= have, f"z strides address {last} elements past z's start; its storage "
                          f"holds {have}")


def lla_encode(x, w_down_t, mu=None, z=None, z_row_stride=None, z_group_stride=None,
               stream=None):
    """Latent write: x [T,N,G,d_loop] bf16, w_down_t [G,r,T*d_loop] bf16 (W_down transposed),
    mu [G,T*d_loop] fp32 or None. Writes z (default a new [G,N,r] bf16
    tensor; pass z plus strides in elements to write into a larger store).
    Returns z."""
    _check_encode(x, w_down_t, mu=mu)
    _need_cuda(x, w_down_t, mu)
    T, N, G, d_loop = x.shape
    r = w_down_t.shape[1]
    if z is None:
        z = torch.empty((G, N, r), device=x.device, dtype=torch.bfloat16)
        z_row_stride, z_group_stride = r, N * r
    if z_row_stride is None or z_group_stride is None:
        raise LLAError(LLA_ERR_INVALID_ARG, "pass z_row_stride and z_group_stride with z")
    _check_z(z, x, G, N, r, z_row_stride, z_group_stride)
    st = lib().lla_encode(_ptr(x), _dtype_code(x), T, N, G, d_loop, r, _ptr(w_down_t), _ptr(mu),
                          _ptr(z), int(z_row_stride), int(z_group_stride), _stream(stream))
    _check(st)
    return z


def lla_encode_bias(w_down_t, mu, muw=None, stream=None):
    """mu W_down of a codec, once: w_down_t [G,r,K] bf16, mu [G,K] fp32.
    Returns muw [G,r] fp32."""
    _expect(w_down_t.dtype == torch.bfloat16 and w_down_t.dim() == 3,
            "w_down_t must be a bfloat16 [G, r, K] tensor")
    G, r, K = w_down_t.shape
    _f32("mu", mu, (G, K))
    _f32("muw", muw, (G, r))
    _need_cuda(w_down_t, mu, muw)
    if muw is None:
        muw = torch.empty((G, r), device=w_down_t.device, dtype=torch.float32)
    _check(lib().lla_encode_bias(_ptr(w_down_t), _ptr(mu), G, K, r, _ptr(muw), _stream(stream)))
    return muw


def lla_encode_with_bias_workspace_bytes(T, N, G, d_loop, r):
    """Workspace bytes lla_encode_with_bias can use to split over K (0: none)."""
    return int(lib().lla_encode_with_bias_workspace(T, N, G, d_loop, r))


def lla_encode_with_bias(x, w_down_t, muw=None, z=None, z_row_stride=None, z_group_stride=None,
                         workspace=None, stream=None, split=True):
    """lla_encode with the mean term precomputed by lla_encode_bias (muw
    [G,r] fp32, or None for a zero mean). With split (default) a workspace
    is allocated when the shape benefits from a split over K (or pass one).
    Returns z."""
    _check_encode(x, w_down_t, muw=muw)
    _need_cuda(x, w_down_t, muw, workspace)
    T, N, G, d_loop = x.shape
    r = w_down_t.shape[1]
    if workspace is None and split:
        need = int(lib().lla_encode_with_bias_workspace(T, N, G, d_loop, r))
        if need:
            workspace = torch.empty(need, device=x.device, dtype=torch.uint8)
    if z is None:
        z = torch.empty((G, N, r), device=x.device, dtype=torch.bfloat16)
        z_row_stride, z_group_stride = r, N * r
    if z_row_stride is None or z_group_stride is None:
        raise LLAError(LLA_ERR_INVALID_ARG, "pass z_row_stride and z_group_stride with z")
    _check_z(z, x, G, N, r, z_row_stride, z_group_stride)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().lla_encode_with_bias(_ptr(x), _dtype_code(x), T, N, G, d_loop, r, _ptr(w_down_t),
                                    _ptr(muw), _ptr(z), int(z_row_stride), int(z_group_stride),
                                    _ptr(workspace), ws_bytes, _stream(stream))
    _check(st)
    return z


def lla_encode_paged(x, w_down_t, muw, z_pages, block_table, positions, seq_idx=None,
                     workspace=None, stream=None, split=True):
    """Latent write into a paged store: token n's latent (lla_encode_with_bias
    of x [T,N,G,d_loop] bf16 with w_down_t [G,r,T*d_loop] and muw [G,r] or
    None) goes to position positions[n] of sequence seq_idx[n] (n when
    seq_idx is None) through block_table [n_seq,max_blocks] int32.
    z_pages is the pool, contiguous bf16: [P,G,page_size,r_row] per head, or
    [P,page_size,r_row] for LLA-2D (G = 1); each row's first r values are
    written (r_row > r keeps a rotary tail). Returns z_pages."""
    _check_encode(x, w_down_t, muw=muw)
    T, N, G, d_loop = x.shape
    r = w_down_t.shape[1]
    _expect(z_pages.dtype == torch.bfloat16, f"z_pages must be bfloat16, got {z_pages.dtype}")
    if z_pages.dim() == 3:
        _expect(G == 1, "an LLA-2D pool [P, page_size, r] takes G = 1")
        P, ps, rr = z_pages.shape
        strides = (ps * rr, 0, rr)
    else:
        _expect(z_pages.dim() == 4 and z_pages.shape[1] == G,
                f"z_pages must be [P, G={G}, page_size, r] or [P, page_size, r], "
                f"got {tuple(z_pages.shape)}")
        P, _, ps, rr = z_pages.shape
        strides = (G * ps * rr, ps * rr, rr)
    _expect(rr >= r, f"pool rows hold {rr} values, fewer than r = {r}")
    _expect(block_table.dtype == torch.int32 and positions.dtype == torch.int32 and
            (seq_idx is None or seq_idx.dtype == torch.int32),
            "block_table, positions and seq_idx must be int32")
    _expect(block_table.dim() == 2, "block_table must be [n_seq, max_blocks]")
    _shape("positions", positions, (N,))
    _shape("seq_idx", seq_idx, (N,))
    _need_cuda(x, w_down_t, muw, z_pages, block_table, positions, seq_idx, workspace)
    if workspace is None and split:
        need = int(lib().lla_encode_with_bias_workspace(T, N, G, d_loop, r))
        if need:
            workspace = torch.empty(need, device=x.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().lla_encode_paged(_ptr(x), _dtype_code(x), T, N, G, d_loop, r, _ptr(w_down_t),
                                _ptr(muw), _ptr(z_pages), *strides, ps, P, _ptr(block_table),
                                block_table.shape[0], block_table.shape[1], _ptr(seq_idx),
                                _ptr(positions), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st)
    return z_pages


def lla_merge_attn(out_parts, lse_parts, out=None, lse=None, stream=None):
    """Log-sum-exp merge of attention over disjoint context parts:
    out_parts [R, ..., d], lse_parts [R, ...] fp32 on the device (each part
    a decode call's (out, lse)). Returns (out [..., d], lse [...])."""
    _f32("out_parts", out_parts)
    _f32("lse_parts", lse_parts)
    _expect(out_parts.dim() >= 2 and tuple(lse_parts.shape) == tuple(out_parts.shape[:-1]),
            f"lse_parts {tuple(lse_parts.shape)} must be out_parts {tuple(out_parts.shape)} "
            "without its last axis")
    _f32("out", out, out_parts.shape[1:])
    _f32("lse", lse, lse_parts.shape[1:])
    _need_cuda(out_parts, lse_parts, out, lse)
    R, d = out_parts.shape[0], out_parts.shape[-1]
    U = lse_parts[0].numel()
    if out is None:
        out = torch.empty(out_parts.shape[1:], device=out_parts.device, dtype=torch.float32)
    if lse is None:
        lse = torch.empty(lse_parts.shape[1:], device=out_parts.device, dtype=torch.float32)
    _check(lib().lla_merge_attn(_ptr(out_parts), _ptr(lse_parts), R, U, d, _ptr(out), _ptr(lse),
                                _stream(stream)))
    return out, lse

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

# Every symbol include/lla.h declares.
EXPORTS = (
    "lla_status_string", "lla_last_error", "lla_version", "lla_device_status",
    "lla_selftest_wait_timeout", "lla_set_timing_events", "lla_merge_attn",
    "lla_decode_attn_workspace", "lla_decode_attn", "lla_decode_attn_noalloc",
    "lla_decode_attn_rope",
    "lla_decode_attn_paged_workspace", "lla_decode_attn_paged",
    "lla2d_decode_attn_workspace", "lla2d_decode_attn", "lla2d_decode_attn_rope",
    "lla2d_decode_attn_paged_workspace", "lla2d_decode_attn_paged",
    "lla_encode", "lla_encode_bias", "lla_encode_with_bias_workspace", "lla_encode_with_bias",
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
    "lla2d_decode_attn_workspace": ([_c_int] * 5, _c_size),
    "lla2d_decode_attn_rope": ([_vp, _vp, _vp, _vp, _c_int] + [_c_int] * 8 + [_vp] * 4 +
                               [_c_float, _vp, _vp, _vp, _c_size, _vp], _c_int),
    "lla2d_decode_attn_paged_workspace": ([_c_int] * 4, _c_size),
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
}


def library_path() -> str:
    return _build.LIB


def lib(build_if_missing: bool = True):
    """Loads liblla.so (building it with nvcc if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build() if build_if_missing else _build.LIB
            if not os.path.exists(path):
                raise LLAError(LLA_ERR_CUDA, f"liblla.so not found at {path}")
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
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise LLAError(LLA_ERR_INVALID_ARG, "tensors must be contiguous CUDA tensors")


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


def lla_decode_attn_workspace(B, H, N, r_k, r_v) -> int:
    return int(lib().lla_decode_attn_workspace(B, H, N, r_k, r_v))


def lla2d_decode_attn_workspace(B, H, N, r_k, r_v) -> int:
    return int(lib().lla2d_decode_attn_workspace(B, H, N, r_k, r_v))


def _decode(fn_name, ws_name, q, zk, zv, dk_t, dv_t, N, mu_k_t, mu_v_t, scale, out, lse,
            workspace, stream, want_lse, two_d):
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
    _need_cuda(q, q_rope, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, workspace)
    B, H, d_h = q.shape
    d_r = q_rope.shape[2]
    n_cap, rq = zk.shape[2], zk.shape[3]
    r_k, r_v = dk_t.shape[2], zv.shape[3]
    if rq != r_k + d_r:
        raise LLAError(LLA_ERR_INVALID_ARG, "zk rows must hold r_k + d_r values")
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
                          workspace=None, stream=None, want_lse=True):
    """Per-head absorbed decode over a paged store with per-sequence lengths.

    q [B,H,d_h] fp32; zk_pages [P,H,page_size,r_k], zv_pages [P,H,page_size,r_v]
    bf16 or fp32; block_table [B,max_blocks] int32 and seq_lens [B] int32 on
    the device; sink, window: the eviction set (window 0 keeps every token).
    Returns (out [B,H,d_h], lse [B,H] or None)."""
    _need_cuda(q, zk_pages, zv_pages, block_table, seq_lens, dk_t, dv_t, mu_k_t, mu_v_t, out,
               lse, workspace)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise LLAError(LLA_ERR_INVALID_ARG, "block_table and seq_lens must be int32")
    if not (block_table.is_contiguous() and seq_lens.is_contiguous()):
        raise LLAError(LLA_ERR_INVALID_ARG, "block_table and seq_lens must be contiguous")
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
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    st = h.lla_decode_attn_paged(_ptr(q), _ptr(zk_pages), _ptr(zv_pages), _dtype_code(zk_pages),
                                 B, H, d_h, r_k, r_v, page_size, num_pages, _ptr(block_table),
                                 max_blocks, _ptr(seq_lens), int(sink), int(window), _ptr(dk_t),
                                 _ptr(dv_t), _ptr(mu_k_t), _ptr(mu_v_t), float(scale), _ptr(out),
                                 _ptr(lse), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out, lse


def lla2d_decode_attn_rope(q, q_rope, zk, zv, dk_t, dv_t, N=None, mu_k_t=None, mu_v_t=None,
                           scale=None, out=None, lse=None, workspace=None, stream=None,
                           want_lse=True):
    """LLA-2D decode with the decoupled rotary branch: zk [B,n_cap,r_k+d_r]
    holds each token's latent followed by its rotated rotary key (shared by
    every head); q_rope [B,H,d_r]; dk_t [H,d_h,r_k]. Returns (out, lse)."""
    _need_cuda(q, q_rope, zk, zv, dk_t, dv_t, mu_k_t, mu_v_t, out, lse, workspace)
    B, H, d_h = q.shape
    d_r = q_rope.shape[2]
    n_cap, rq = zk.shape[1], zk.shape[2]
    r_k, r_v = dk_t.shape[2], zv.shape[2]
    if rq != r_k + d_r:
        raise LLAError(LLA_ERR_INVALID_ARG, "zk rows must hold r_k + d_r values")
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
                            lse=None, workspace=None, stream=None, want_lse=True):
    """LLA-2D absorbed decode over a paged store: zk_pages [P,page_size,r_k],
    zv_pages [P,page_size,r_v] bf16 shared by every head, page_size a
    multiple of 64; block_table [B,max_blocks] and seq_lens [B] int32 on
    the device. Returns (out [B,H,d_h], lse [B,H] or None)."""
    _need_cuda(q, zk_pages, zv_pages, block_table, seq_lens, dk_t, dv_t, mu_k_t, mu_v_t, out,
               lse, workspace)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise LLAError(LLA_ERR_INVALID_ARG, "block_table and seq_lens must be int32")
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
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    st = h.lla2d_decode_attn_paged(_ptr(q), _ptr(zk_pages), _ptr(zv_pages),
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


def lla_encode(x, w_down_t, mu=None, z=None, z_row_stride=None, z_group_stride=None,
               stream=None):
    """Latent write: x [T,N,G,d_loop] bf16, w_down_t [G,r,T*d_loop] bf16 (W_down transposed),
    mu [G,T*d_loop] fp32 or None. Writes z (default a new [G,N,r] bf16
    tensor; pass z plus strides in elements to write into a larger store).
    Returns z."""
    _need_cuda(x, w_down_t, mu)
    T, N, G, d_loop = x.shape
    r = w_down_t.shape[1]
    if z is None:
        z = torch.empty((G, N, r), device=x.device, dtype=torch.bfloat16)
        z_row_stride, z_group_stride = r, N * r
    if z_row_stride is None or z_group_stride is None:
        raise LLAError(LLA_ERR_INVALID_ARG, "pass z_row_stride and z_group_stride with z")
    st = lib().lla_encode(_ptr(x), _dtype_code(x), T, N, G, d_loop, r, _ptr(w_down_t), _ptr(mu),
                          _ptr(z), int(z_row_stride), int(z_group_stride), _stream(stream))
    _check(st)
    return z


def lla_encode_bias(w_down_t, mu, muw=None, stream=None):
    """mu W_down of a codec, once: w_down_t [G,r,K] bf16, mu [G,K] fp32.
    Returns muw [G,r] fp32."""
    _need_cuda(w_down_t, mu, muw)
    G, r, K = w_down_t.shape
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
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().lla_encode_with_bias(_ptr(x), _dtype_code(x), T, N, G, d_loop, r, _ptr(w_down_t),
                                    _ptr(muw), _ptr(z), int(z_row_stride), int(z_group_stride),
                                    _ptr(workspace), ws_bytes, _stream(stream))
    _check(st)
    return z


def lla_merge_attn(out_parts, lse_parts, out=None, lse=None, stream=None):
    """Log-sum-exp merge of attention over disjoint context parts:
    out_parts [R, ..., d], lse_parts [R, ...] fp32 on the device (each part
    a decode call's (out, lse)). Returns (out [..., d], lse [...])."""
    _need_cuda(out_parts, lse_parts, out, lse)
    R, d = out_parts.shape[0], out_parts.shape[-1]
    U = lse_parts[0].numel()
    if out_parts[0].numel() != U * d:
        raise LLAError(LLA_ERR_INVALID_ARG, "out_parts and lse_parts disagree on the units")
    if out is None:
        out = torch.empty(out_parts.shape[1:], device=out_parts.device, dtype=torch.float32)
    if lse is None:
        lse = torch.empty(lse_parts.shape[1:], device=out_parts.device, dtype=torch.float32)
    _check(lib().lla_merge_attn(_ptr(out_parts), _ptr(lse_parts), R, U, d, _ptr(out), _ptr(lse),
                                _stream(stream)))
    return out, lse

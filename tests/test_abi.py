"""Host-side checks of the C ABI: the library builds, loads, exports every
symbol include/lla.h declares, and rejects bad arguments before touching a
device. Nothing here launches a kernel."""

import ctypes
import os
import re

import pytest

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "lla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lla\w*)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    h = lla.lib()
    declared = header_functions()
    assert declared, "no declarations parsed"
    for name in declared:
        assert hasattr(h, name), f"{name} declared in lla.h but not exported"
    assert sorted(_lib.EXPORTS) == declared


def test_status_strings_and_version():
    h = lla.lib()
    for code, name in [(0, b"LLA_OK"), (1, b"LLA_ERR_INVALID_ARG"), (2, b"LLA_ERR_UNSUPPORTED"),
                       (3, b"LLA_ERR_WORKSPACE"), (4, b"LLA_ERR_CUDA"), (99, b"LLA_ERR_UNKNOWN")]:
        assert h.lla_status_string(code) == name
    assert h.lla_version() >= 100


def _call_decode(**over):
    h = lla.lib()
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: arguments fail first
    args = dict(q=fake, zk=fake, zv=fake, zdt=1, B=2, H=2, d_h=16, N=8, n_cap=8, r_k=8, r_v=8,
                dk=fake, dv=fake, mu_k=None, mu_v=None, scale=0.25, out=fake, lse=None,
                ws=fake, ws_bytes=0, stream=None)
    args.update(over)
    return h.lla_decode_attn(*args.values())


@pytest.mark.parametrize("over, why", [
    (dict(zdt=7), "zdt"),
    (dict(q=None), "non-NULL"),
    (dict(B=0), "B and H"),
    (dict(d_h=0), "d_h"),
    (dict(d_h=300), "d_h"),
    (dict(N=0), "N must be >= 1"),
    (dict(N=9), "n_cap"),
    (dict(r_k=12), "multiples of 8"),
    (dict(r_v=264), "multiples of 8"),
    (dict(zdt=0, r_k=136), "multiples of 8"),
    (dict(zk=ctypes.c_void_p(0x100008)), "16-byte"),
    (dict(ws=ctypes.c_void_p(0x100004)), "workspace must be 16-byte"),
])
def test_decode_rejects_bad_arguments_on_the_host(over, why):
    st = _call_decode(**over)
    assert st == _lib.LLA_ERR_INVALID_ARG
    assert why in lla.lib().lla_last_error().decode()


def test_decode_reports_small_workspace_before_launch():
    need = lla.lla_decode_attn_workspace(2, 2, 8, 8, 8)
    assert need > 0
    st = _call_decode(ws_bytes=need - 16)
    assert st == _lib.LLA_ERR_WORKSPACE


def test_workspace_sizes_are_consistent():
    assert lla.lla_decode_attn_workspace(0, 1, 1, 8, 8) == 0
    assert lla.lla_decode_attn_workspace(1, 1, 1, 12, 8) == 0
    small = lla.lla_decode_attn_workspace(1, 2, 64, 8, 8)
    big = lla.lla_decode_attn_workspace(64, 16, 4096, 128, 128)
    assert 0 < small < big
    # q' alone is B*H*r_k floats: the workspace must hold at least that
    assert big >= 64 * 16 * 128 * 4
    # and it stays small next to the latent store it scans (2 GiB here)
    assert big < 16 << 20


def test_device_status_needs_a_pointer():
    assert lla.lib().lla_device_status(None, 0) == _lib.LLA_ERR_INVALID_ARG


def test_lla2d_rejects_unsupported_shapes_on_the_host():
    h = lla.lib()
    fake = ctypes.c_void_p(0x100000)

    def call(**over):
        args = dict(q=fake, zk=fake, zv=fake, zdt=1, B=2, H=16, d_h=128, N=8, n_cap=8, r_k=256,
                    r_v=256, dk=fake, dv=fake, mu_k=None, mu_v=None, scale=0.1, out=fake,
                    lse=None, ws=fake, ws_bytes=0, stream=None)
        args.update(over)
        return h.lla2d_decode_attn(*args.values())

    assert call(zdt=0, r_k=128, r_v=128) == _lib.LLA_ERR_UNSUPPORTED
    assert call(H=33) == _lib.LLA_ERR_UNSUPPORTED
    assert call(r_k=96) == _lib.LLA_ERR_UNSUPPORTED
    assert call(r_v=64) == _lib.LLA_ERR_UNSUPPORTED
    assert call(ws_bytes=16) == _lib.LLA_ERR_WORKSPACE
    assert lla.lla2d_decode_attn_workspace(2, 33, 8, 256, 256) == 0
    assert lla.lla2d_decode_attn_workspace(2, 16, 8, 256, 192) == 0
    assert lla.lla2d_decode_attn_workspace(256, 16, 8192, 256, 256) > 256 * 16 * 256 * 4


def test_encode_rejects_bad_arguments_on_the_host():
    h = lla.lib()
    fake = ctypes.c_void_p(0x100000)

    def call(**over):
        args = dict(x=fake, xdt=1, T=4, N=10, G=2, d_loop=128, r=16, w=fake, mu=None, z=fake,
                    zrs=16, zgs=160, stream=None)
        args.update(over)
        return h.lla_encode(*args.values())

    assert call(xdt=0) == _lib.LLA_ERR_INVALID_ARG
    assert call(d_loop=96) == _lib.LLA_ERR_INVALID_ARG
    assert call(r=12) == _lib.LLA_ERR_INVALID_ARG
    assert call(r=264) == _lib.LLA_ERR_INVALID_ARG
    assert call(zrs=8) == _lib.LLA_ERR_INVALID_ARG         # rows narrower than r
    assert call(zgs=16) == _lib.LLA_ERR_INVALID_ARG        # groups overlap rows
    assert call(x=ctypes.c_void_p(0x100008)) == _lib.LLA_ERR_INVALID_ARG
    assert call(N=0) == _lib.LLA_ERR_INVALID_ARG

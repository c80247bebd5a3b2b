"""Host-side checks of the C ABI: the library builds, loads, exports every
symbol include/lla.h declares, and rejects bad arguments before touching a
device. Nothing here launches a kernel.

Many calls below pass placeholder pointers that are never valid device
addresses; each is meant to fail a host-side check first. So that a case
which wrongly passed those checks could never reach a kernel, this file
runs only where no CUDA device is visible (the CPU test pass)."""

import ctypes
import os
import re

import pytest
import torch

import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.skipif(
    torch.cuda.is_available(),
    reason="placeholder-pointer calls run only where no CUDA device is visible")


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
    assert call(r_k=12) == _lib.LLA_ERR_INVALID_ARG          # ranks are multiples of 8
    assert call(r_v=264) == _lib.LLA_ERR_INVALID_ARG
    # ranks that are not whole boxes or tiles are accepted (zero-padded
    # inside): these stop at the workspace check
    assert call(r_k=96, r_v=160) == _lib.LLA_ERR_WORKSPACE
    assert call(r_k=8, r_v=72) == _lib.LLA_ERR_WORKSPACE
    assert call(ws_bytes=16) == _lib.LLA_ERR_WORKSPACE
    assert lla.lla2d_decode_attn_workspace(2, 33, 8, 256, 256) == 0
    assert lla.lla2d_decode_attn_workspace(2, 16, 8, 256, 196) == 0
    assert lla.lla2d_decode_attn_workspace(2, 16, 8, 96, 160) > 0
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


FAKE = ctypes.c_void_p(0x100000)  # never dereferenced: every call below fails on the host


@pytest.mark.parametrize("fn", ["lla_decode_attn_paged_plan", "lla2d_decode_attn_paged_plan"])
def test_paged_plan_rejects_bad_arguments_on_the_host(fn):
    h = lla.lib()
    two_d = fn.startswith("lla2d")

    def call(**over):
        args = dict(zdt=1, B=2, H=16, r_k=128, r_v=128, ps=64, P=9, bt=FAKE, mb=3, sl=FAKE,
                    sink=0, window=0, ws=FAKE, ws_bytes=0, stream=None)
        args.update(over)
        if two_d:
            del args["zdt"]
        return getattr(h, fn)(*args.values())

    cases = [
        (dict(bt=None), _lib.LLA_ERR_INVALID_ARG, b"non-NULL"),
        (dict(sl=ctypes.c_void_p(0x100002)), _lib.LLA_ERR_INVALID_ARG, b"4-byte"),
        (dict(B=0), _lib.LLA_ERR_INVALID_ARG, b"B and H"),
        (dict(r_k=12), _lib.LLA_ERR_INVALID_ARG, b"multiples of 8"),
        (dict(P=0), _lib.LLA_ERR_INVALID_ARG, b"num_pages"),
        (dict(mb=1 << 28), _lib.LLA_ERR_INVALID_ARG, b"31 bits"),
        (dict(window=-1), _lib.LLA_ERR_INVALID_ARG, b"sink and window"),
        (dict(ws=ctypes.c_void_p(0x100008)), _lib.LLA_ERR_INVALID_ARG, b"16-byte"),
        (dict(ws_bytes=16), _lib.LLA_ERR_WORKSPACE, b"workspace"),
    ]
    if two_d:
        cases += [(dict(H=33), _lib.LLA_ERR_UNSUPPORTED, b"H <= 32"),
                  (dict(ps=96), _lib.LLA_ERR_UNSUPPORTED, b"multiple of 64")]
    else:
        cases += [(dict(zdt=3), _lib.LLA_ERR_INVALID_ARG, b"zdt"),
                  (dict(zdt=0, r_k=136), _lib.LLA_ERR_INVALID_ARG, b"multiples of 8")]
    for over, code, why in cases:
        assert call(**over) == code, over
        assert why in h.lla_last_error(), (over, h.lla_last_error())


def test_paged_encode_rejects_bad_arguments_on_the_host():
    h = lla.lib()

    def call(**over):
        # a per-head pool [P=9][G=2][page_size=4][r_row=24] written at r = 16:
        # one page spans (G-1)*96 + (4-1)*24 + 16 = 184 elements
        args = dict(x=FAKE, xdt=1, T=4, N=10, G=2, d_loop=128, r=16, w=FAKE, muw=None, z=FAKE,
                    zps=2 * 4 * 24, zgs=4 * 24, zrs=24, ps=4, P=9, bt=FAKE, n_seq=10, mb=3,
                    seq=None, pos=FAKE, ws=None, ws_bytes=0, stream=None)
        args.update(over)
        return h.lla_encode_paged(*args.values())

    # every case must fail on the host for its own reason (the message says
    # which), so no placeholder pointer can reach a launch
    for over, why in [
        (dict(ps=0), b"page_size, num_pages"),
        (dict(n_seq=0), b"page_size, num_pages"),
        (dict(mb=1 << 30), b"31 bits"),
        (dict(zrs=8), b"z_row_stride >= r"),
        (dict(zgs=24), b"overlap"),
        (dict(zps=176), b"z_page_stride"),
        (dict(zps=188), b"z_page_stride"),
        (dict(bt=None), b"non-NULL"),
        (dict(pos=None), b"non-NULL"),
        (dict(pos=ctypes.c_void_p(0x100002)), b"4-byte aligned"),
        (dict(seq=ctypes.c_void_p(0x100002)), b"4-byte aligned"),
        (dict(z=ctypes.c_void_p(0x100008)), b"16-byte aligned"),
        (dict(muw=ctypes.c_void_p(0x100004)), b"muw must be 16-byte"),
        (dict(xdt=0), b"xdt"),
    ]:
        assert call(**over) == _lib.LLA_ERR_INVALID_ARG, over
        assert why in h.lla_last_error(), (over, h.lla_last_error())


def test_paged_decode_rejects_bad_arguments_on_the_host():
    h = lla.lib()

    def call(**over):
        args = dict(q=FAKE, zk=FAKE, zv=FAKE, zdt=1, B=2, H=2, d_h=16, r_k=8, r_v=8, ps=16,
                    npages=4, bt=FAKE, maxb=2, sl=FAKE, sink=0, window=0, dk=FAKE, dv=FAKE,
                    mu_k=None, mu_v=None, scale=0.25, out=FAKE, lse=None, ws=FAKE, ws_bytes=0,
                    stream=None)
        args.update(over)
        return h.lla_decode_attn_paged(*args.values())

    assert call(bt=None) == _lib.LLA_ERR_INVALID_ARG
    assert call(sl=ctypes.c_void_p(0x100002)) == _lib.LLA_ERR_INVALID_ARG
    assert call(ps=0) == _lib.LLA_ERR_INVALID_ARG
    assert call(npages=0) == _lib.LLA_ERR_INVALID_ARG
    assert call(maxb=0) == _lib.LLA_ERR_INVALID_ARG
    assert call(ps=1 << 20, maxb=1 << 12) == _lib.LLA_ERR_INVALID_ARG  # 2^32 tokens
    assert call(sink=-1) == _lib.LLA_ERR_INVALID_ARG
    assert call(window=-1) == _lib.LLA_ERR_INVALID_ARG
    assert call(r_k=12) == _lib.LLA_ERR_INVALID_ARG
    need = lla.lla_decode_attn_paged_workspace(2, 2, 8, 8)
    assert need > 0
    assert call(ws_bytes=need - 16) == _lib.LLA_ERR_WORKSPACE
    assert lla.lla_decode_attn_paged_workspace(0, 2, 8, 8) == 0


def test_rope_decode_rejects_bad_arguments_on_the_host():
    h = lla.lib()

    def call(fn, **over):
        args = dict(q=FAKE, qr=FAKE, zk=FAKE, zv=FAKE, zdt=1, B=2, H=16, d_h=128, d_r=64, N=8,
                    n_cap=8, r_k=192, r_v=256, dk=FAKE, dv=FAKE, mu_k=None, mu_v=None,
                    scale=0.1, out=FAKE, lse=None, ws=FAKE, ws_bytes=0, stream=None)
        args.update(over)
        return getattr(h, fn)(*args.values())

    for fn in ("lla_decode_attn_rope", "lla2d_decode_attn_rope"):
        assert call(fn, qr=None) == _lib.LLA_ERR_INVALID_ARG
        assert call(fn, d_r=12) == _lib.LLA_ERR_INVALID_ARG
        assert call(fn, d_r=0) == _lib.LLA_ERR_INVALID_ARG
        assert call(fn, ws_bytes=16) == _lib.LLA_ERR_WORKSPACE
    # per-head: latent + rotary rows at most 256 bf16 wide
    assert call("lla_decode_attn_rope", r_k=224) == _lib.LLA_ERR_INVALID_ARG
    # LLA-2D: rows up to 384 wide (200 + 64 is accepted and zero-padded;
    # it stops at the workspace check)
    assert call("lla2d_decode_attn_rope", r_k=200) == _lib.LLA_ERR_WORKSPACE
    assert call("lla2d_decode_attn_rope", r_k=384) == _lib.LLA_ERR_UNSUPPORTED
    assert call("lla2d_decode_attn_rope", r_k=320, ws_bytes=16) == _lib.LLA_ERR_WORKSPACE
    assert lla.lla2d_decode_attn_workspace(2, 16, 8, 384, 256) > 0
    assert lla.lla2d_decode_attn_workspace(2, 16, 8, 448, 256) == 0


def test_paged_lla2d_rejects_bad_arguments_on_the_host():
    h = lla.lib()

    def call(**over):
        args = dict(q=FAKE, zk=FAKE, zv=FAKE, zdt=1, B=2, H=16, d_h=128, r_k=256, r_v=256,
                    ps=256, npages=4, bt=FAKE, maxb=2, sl=FAKE, sink=0, window=0, dk=FAKE,
                    dv=FAKE, mu_k=None, mu_v=None, scale=0.1, out=FAKE, lse=None, ws=FAKE,
                    ws_bytes=0, stream=None)
        args.update(over)
        return h.lla2d_decode_attn_paged(*args.values())

    assert call(ps=32) == _lib.LLA_ERR_UNSUPPORTED       # pages hold whole 64-token boxes
    assert call(ps=200) == _lib.LLA_ERR_UNSUPPORTED
    assert call(H=40) == _lib.LLA_ERR_UNSUPPORTED
    assert call(zdt=0, r_k=128, r_v=128) == _lib.LLA_ERR_UNSUPPORTED
    assert call(bt=None) == _lib.LLA_ERR_INVALID_ARG
    assert call(npages=0) == _lib.LLA_ERR_INVALID_ARG
    assert call(window=-1) == _lib.LLA_ERR_INVALID_ARG
    assert call(ws_bytes=16) == _lib.LLA_ERR_WORKSPACE
    assert lla.lla2d_decode_attn_paged_workspace(2, 16, 256, 256) > 0
    assert lla.lla2d_decode_attn_paged_workspace(2, 16, 100, 256) == 0


def test_encode_bias_entry_points_reject_bad_arguments_on_the_host():
    h = lla.lib()
    assert h.lla_encode_bias(None, FAKE, 2, 512, 16, FAKE, None) == _lib.LLA_ERR_INVALID_ARG
    assert h.lla_encode_bias(FAKE, ctypes.c_void_p(0x100004), 2, 512, 16, FAKE, None) == \
        _lib.LLA_ERR_INVALID_ARG                                     # mu not 16-byte aligned
    assert h.lla_encode_bias(FAKE, FAKE, 2, 12, 16, FAKE, None) == _lib.LLA_ERR_INVALID_ARG

    def call(**over):
        args = dict(x=FAKE, xdt=1, T=4, N=10, G=2, d_loop=128, r=16, w=FAKE, muw=None, z=FAKE,
                    zrs=16, zgs=160, ws=None, ws_bytes=0, stream=None)
        args.update(over)
        return h.lla_encode_with_bias(*args.values())

    assert call(muw=ctypes.c_void_p(0x100004)) == _lib.LLA_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(0x100008)) == _lib.LLA_ERR_INVALID_ARG
    assert call(d_loop=96) == _lib.LLA_ERR_INVALID_ARG
    assert call(zgs=16) == _lib.LLA_ERR_INVALID_ARG
    # split over K only where few tiles meet a long contraction
    assert h.lla_encode_with_bias_workspace(4, 256, 1, 2048, 256) > 0
    assert h.lla_encode_with_bias_workspace(4, 32768, 16, 128, 16) == 0


def test_selftest_rejects_bad_timeouts_on_the_host():
    h = lla.lib()
    assert h.lla_selftest_wait_timeout(0, None) == _lib.LLA_ERR_INVALID_ARG
    assert h.lla_selftest_wait_timeout(2000000, None) == _lib.LLA_ERR_INVALID_ARG


_NOALLOC_REJECT = r"""
import ctypes, sys
sys.path.insert(0, sys.argv[1])
import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import _lib
# 512 sequences x 16 heads with r = 128 need over 4 MiB for the absorbed
# queries alone
need = lla.lla_decode_attn_workspace(512, 16, 1, 128, 128)
assert need > 4 << 20, need
fake = ctypes.c_void_p(0x100000)
st = lla.lib().lla_decode_attn_noalloc(fake, fake, fake, 1, 512, 16, 128, 1, 1, 128, 128,
                                       fake, fake, None, None, 0.1, fake, None, None)
assert st == _lib.LLA_ERR_WORKSPACE, st
assert b"scratch" in lla.lib().lla_last_error()
print("rejected")
"""


def test_noalloc_rejects_shapes_beyond_its_scratch_before_launching():
    # Runs in a child process with no visible CUDA device, so the fake
    # pointers can never reach a kernel whatever the machine: the call must
    # return LLA_ERR_WORKSPACE from its host-side size check.
    import subprocess
    import sys
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", _NOALLOC_REJECT, ROOT], env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "rejected" in res.stdout

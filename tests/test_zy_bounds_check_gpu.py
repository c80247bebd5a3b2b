"""The bounds-check build (liblla_check.so, LLA_BOUNDS_CHECK) on the GPU.

In that build every computed global access of the kernels is tested against
the extent of the buffer it belongs to, and a miss sets
LLA_DEVICE_OUT_OF_BOUNDS instead of touching memory. This file runs the
library's paths through it on the small and ragged cases where an indexing
slip would show (contexts of 1, 7, 64, 65 and 127 tokens, splits that do not
divide N, ragged pages, eviction, padded ranks, split-K writes) and checks
that no access is flagged and that every result still matches the fp64
oracle. The checked library runs in a child process (one library per
process); pytest collects this file just before the no-alloc file."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np
import torch
import decode_attention_encode_b200 as lla
from decode_attention_encode_b200 import _lib, synth
import oracle
from lla_cases import (compare, compare_paged, make_decode_inputs, make_paged_inputs,
                       oracle_paged_reference, oracle_reference, check_encoded, to_f64)

assert _lib.library_path().endswith("liblla_check.so"), _lib.library_path()
BF16, F32 = torch.bfloat16, torch.float32

def clean(what):
    st = lla.device_status(clear=True)
    assert st == 0, f"{what}: device status {st:#x}"

# per-head dense: tiny fp32 and short, odd contexts with ranks of 1..5 segments
inp = make_decode_inputs(1, 2, 16, 64, 8, 8, F32, seed=0)
units = [(0, 0), (0, 1)]
out, lse = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"])
compare(out, lse, units, *oracle_reference(inp, units), F32); clean("tiny fp32")
for N in (1, 7, 64, 65, 127):
    for r_k, r_v in ((24, 40), (96, 160)):
        inp = make_decode_inputs(3, 5, 64, N, r_k, r_v, BF16, n_cap=N + 5, mu=True, seed=N + r_k)
        out, lse = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N,
                                       mu_k_t=inp["mu_k"], mu_v_t=inp["mu_v"])
        u = [(b, h) for b in range(3) for h in range(5)]
        compare(out, lse, u, *oracle_reference(inp, u), BF16); clean(f"per-head N={N}")
# many units over the one-wave grid (pieces spanning units), and the tensor-core forms
inp = make_decode_inputs(300, 4, 64, 77, 192, 256, BF16, seed=3)
out, lse = lla.lla_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=77)
u = [(0, 0), (150, 2), (299, 3)]
compare(out, lse, u, *oracle_reference(inp, u), BF16); clean("per-head tc forms")

# paged per-head: ragged lengths, pages that do not divide the tile, eviction
for ps, sink, window in ((7, 0, 0), (64, 4, 100)):
    lens = [0, 1, 7, 64, 65, 127, 500]
    inp = make_paged_inputs(lens, 3, 64, 24, 24, BF16, ps, mu=True, seed=ps)
    out, lse = lla.lla_decode_attn_paged(inp["q"], inp["zk"], inp["zv"], inp["block_table"],
                                         inp["seq_lens"], inp["dk"], inp["dv"], inp["mu_k"],
                                         inp["mu_v"], sink=sink, window=window)
    compare_paged(out, lse, *oracle_paged_reference(inp, sink, window), lens, BF16)
    clean(f"paged ps={ps}")

# LLA-2D dense and paged (64-token pages), padded ranks
for N, r_k, r_v in ((1, 256, 256), (127, 96, 160), (129, 64, 72)):
    inp = make_decode_inputs(3, 16, 128, N, r_k, r_v, BF16, two_d=True, n_cap=N + 3, seed=N)
    out, lse = lla.lla2d_decode_attn(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"], N=N)
    u = [(b, h) for b in range(3) for h in range(16)]
    compare(out, lse, u, *oracle_reference(inp, u, two_d=True), BF16); clean(f"2d N={N}")
lens = np.array([1, 64, 65, 300, 0], dtype=np.int32)
bt, P = synth.page_table(lens, 64, seed=5, spare=1)
zk = synth.latents((P, 64, 256), 1, "cuda", dtype=BF16)
zv = synth.latents((P, 64, 256), 2, "cuda", dtype=BF16)
q = synth.queries((5, 16, 128), 128, 3, "cuda")
dk, dv = synth.orthonormal(16, 128, 256, 4, "cuda"), synth.orthonormal(16, 128, 256, 5, "cuda")
bt_d, sl = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
out, lse = lla.lla2d_decode_attn_paged(q, zk, zv, bt_d, sl, dk, dv)
ref_o, ref_l = oracle.paged2d_decode(to_f64(q), to_f64(zk), to_f64(zv), bt.astype(np.int64), lens,
                                     to_f64(dk), to_f64(dv))
full = lens > 0
err = np.abs(to_f64(out)[full] - ref_o[full]).max() / np.abs(ref_o[full]).max()
assert err < 2e-2, err
clean("2d paged 64-token pages")

# latent writes: unsplit, split over K, wide stack, paged
for T, N, G, d_loop, r, split in ((4, 130, 3, 64, 16, False), (4, 7, 2, 128, 24, True),
                                  (4, 200, 1, 2048, 256, False)):
    x = synth.normal((T, N, G, d_loop), 21, "cuda", dtype=BF16)
    w = synth.orthonormal(G, T * d_loop, r, 22, "cuda").to(BF16)
    w_t = w.transpose(1, 2).contiguous()
    mu = synth.normal((G, T * d_loop), 23, "cuda", std=0.5)
    z = lla.lla_encode_with_bias(x, w_t, lla.lla_encode_bias(w_t, mu), split=split)
    check_encoded(z, oracle.encode(to_f64(x), to_f64(w), to_f64(mu))); clean(f"encode r={r}")
pool = synth.latents((9, 3, 16, 24), 7, "cuda", dtype=BF16)
bt2 = torch.tensor([[0, 1], [2, 3], [4, 5]], dtype=torch.int32, device="cuda")
pos = torch.tensor([0, 17, 31], dtype=torch.int32, device="cuda")
x = synth.normal((4, 3, 3, 64), 8, "cuda", dtype=BF16)
w_t = synth.orthonormal(3, 256, 24, 9, "cuda").to(BF16).transpose(1, 2).contiguous()
lla.lla_encode_paged(x, w_t, None, pool, bt2, pos)
torch.cuda.synchronize(); clean("paged write")

# context merge and the no-alloc entry point
inp = make_decode_inputs(2, 3, 64, 100, 24, 24, BF16, seed=6)
o1, l1 = lla.lla_decode_attn(inp["q"], inp["zk"][:, :, :60].contiguous(),
                             inp["zv"][:, :, :60].contiguous(), inp["dk"], inp["dv"])
o2, l2 = lla.lla_decode_attn(inp["q"], inp["zk"][:, :, 60:].contiguous(),
                             inp["zv"][:, :, 60:].contiguous(), inp["dk"], inp["dv"])
om, lm = lla.lla_merge_attn(torch.stack([o1, o2]), torch.stack([l1, l2]))
u = [(b, h) for b in range(2) for h in range(3)]
compare(om, lm, u, *oracle_reference(inp, u), BF16); clean("merge")
out, lse = lla.lla_decode_attn_noalloc(inp["q"], inp["zk"], inp["zv"], inp["dk"], inp["dv"])
compare(out, lse, u, *oracle_reference(inp, u), BF16); clean("noalloc")
print("bounds-check build: all paths clean")
"""


def test_every_path_runs_clean_in_the_bounds_check_build():
    from decode_attention_encode_b200 import build
    build.build(variant="check")
    env = dict(os.environ, LLA_LIBRARY_VARIANT="check")
    res = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True,
                         text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    assert "all paths clean" in res.stdout

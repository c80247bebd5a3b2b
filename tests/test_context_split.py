"""Context split across ranks on CPU: two gloo ranks each hold half of every
sequence's cached tokens, decode their half with the oracle, and exchange
(out, lse) through context_split.gather_and_merge; the merged result must
equal the oracle's decode over the whole context. The merge used here is the
oracle's; the GPU merge kernel is checked against it in
test_context_split_gpu.py."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def inputs():
    r = np.random.default_rng(5)
    B, H, d, N, rk, rv = 2, 3, 8, 21, 8, 16
    return dict(q=r.standard_normal((B, H, d)), zk=r.standard_normal((B, H, N, rk)),
                zv=r.standard_normal((B, H, N, rv)), dk=r.standard_normal((H, d, rk)),
                dv=r.standard_normal((H, d, rv)), mk=r.standard_normal((H, d)),
                mv=r.standard_normal((H, d)), N=N)


def worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    from decode_attention_encode_b200.context_split import gather_and_merge, shard_range
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x = inputs()
    a, b = shard_range(x["N"], world, rank)
    o, l = oracle.lla_decode(x["q"], x["zk"][:, :, a:b], x["zv"][:, :, a:b], x["dk"], x["dv"],
                             x["mk"], x["mv"])

    def merge(outs, lses):
        mo, ml = oracle.merge_attn(outs.numpy(), lses.numpy())
        return torch.from_numpy(mo), torch.from_numpy(ml)

    mo, ml = gather_and_merge(torch.from_numpy(o), torch.from_numpy(l), merge=merge)
    out.put((rank, mo.numpy(), ml.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def test_shard_range_covers_the_context_once():
    from decode_attention_encode_b200.context_split import shard_range
    for N in (0, 1, 7, 8, 1000):
        for world in (1, 2, 3, 8):
            parts = [shard_range(N, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == N
            assert all(p[1] == q[0] for p, q in zip(parts, parts[1:]))
            sizes = [p[1] - p[0] for p in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(5, 2, 2)


def test_two_gloo_ranks_merge_to_the_whole_context():
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    x = inputs()
    ref_o, ref_l = oracle.lla_decode(x["q"], x["zk"], x["zv"], x["dk"], x["dv"], x["mk"], x["mv"])
    for _ in range(world):
        rank, mo, ml = q.get(timeout=5)
        np.testing.assert_allclose(mo, ref_o, atol=1e-12)
        np.testing.assert_allclose(ml, ref_l, atol=1e-12)

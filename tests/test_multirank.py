"""The multi-process path of bench.py on CPU: two gloo ranks, as torchrun
would start them. The data path has no collective (each rank decodes its own
sequences); this checks the plumbing around it: rendezvous, barrier, the
max-over-ranks step time, the whole-job rate, and that ranks draw different
sequences."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from decode_attention_encode_b200 import synth
    w, r, _ = bench.dist_setup("gloo")
    assert (w, r) == (world, rank)
    bench.barrier(w)
    step_ms = 10.0 + 5.0 * rank               # rank 1 is the slow one
    slowest = bench.max_over_ranks(step_ms, w)
    rate = bench.aggregate_rate(1000.0, slowest, w)
    # each rank's sequences come from its own seed offset
    z = synth.latents((2, 3, 8), seed=1 + 1000 * rank, decay=True)
    gathered = [torch.zeros_like(z.float()) for _ in range(w)]
    dist.all_gather(gathered, z.float())
    out.put((rank, slowest, rate, bool(torch.equal(gathered[0], gathered[1]))))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_and_shard_sequences():
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
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, slowest, rate, same in res:
        assert slowest == pytest.approx(15.0)
        assert rate == pytest.approx(2 * 1000.0 / 15e-3)
        assert not same

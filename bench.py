#!/usr/bin/env python
"""Benchmark of the LLA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl lla|reference]

One step is a full looped decode step of the chosen workload: for every loop
t and layer d, one absorbed per-head decode call (query absorb, latent
stream with online softmax, split merge with the V decoder) over every
cached token of layer d, i.e. L*T calls. Prints one JSON line on rank 0.

Metric: cached tokens attended per second per (layer, loop) step, i.e.
B * N * L * T / step time. Inputs are resident in HBM when timing starts and
each layer's latent store is larger than L2, so no flush is needed.

Multi-GPU: every rank decodes its own batch of sequences (weak scaling, no
collective on the data path); the step time is the max over ranks.

--impl reference times the fp64 CPU oracle (explicit reconstruction then
textbook attention) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from decode_attention_encode_b200 import synth  # noqa: E402

METRIC = "LLA decode: cached tokens attended/sec per loop step; HBM GB/s vs B200 peak"
UNIT = "tokens/s"
DEFAULT_CONFIG = "perhead_21x"
CSRC = os.path.join(ROOT, "decode_attention_encode_b200", "csrc")
PROFILE_DIR = os.path.join(ROOT, "profiles")
ENCODE_CONFIGS = synth.ENCODE_CONFIGS


def main_kernel(config_name: str):
    """(kernel name, source file) of the kernel that dominates a workload."""
    if config_name in ENCODE_CONFIGS:
        return "k_encode", os.path.join(CSRC, "encode.cu")
    if synth.DECODE_CONFIGS[config_name].two_d:
        return "k_lla2d", os.path.join(CSRC, "lla2d.cu")
    if synth.DECODE_CONFIGS[config_name].page_size:
        return "k_stream_paged", os.path.join(CSRC, "stream.cu")
    return "k_stream", os.path.join(CSRC, "stream.cu")


def step_runner(step, eager: bool):
    """What the device-timed region runs per step: the workload's step
    replayed from a CUDA graph captured once (the same kernels on the same
    buffers, launched without per-call host work), or the eager calls.
    Returns (run, description)."""
    if eager:
        return step, "eager library calls"
    try:
        stream = torch.cuda.current_stream()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
    except Exception as e:  # a capture the runtime refuses: time the eager calls
        torch.cuda.synchronize()
        return step, f"eager library calls (graph capture failed: {type(e).__name__})"
    return graph.replay, "one step captured as a CUDA graph, replayed"


def with_layers(cfg, layers: int):
    """The workload with `layers` layers (0: its own count)."""
    import dataclasses
    return dataclasses.replace(cfg, L=layers) if layers > 0 else cfg


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=int(os.environ.get("WORLD_SIZE", "1")))
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--config", default=DEFAULT_CONFIG,
                   choices=sorted(synth.DECODE_CONFIGS) + sorted(ENCODE_CONFIGS))
    p.add_argument("--impl", default="lla", choices=["lla", "reference"])
    p.add_argument("--layers", type=int, default=0,
                   help="run the workload with this many layers instead of its own (a smaller "
                        "case for profiler captures; the JSON line names the layer count)")
    p.add_argument("--eager", action="store_true",
                   help="time the steps as eager library calls instead of replaying one "
                        "captured step graph")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(backend: str = "nccl"):
    """One process per GPU: reads RANK / LOCAL_RANK / WORLD_SIZE / MASTER_*
    from the environment. Sequences are sharded by rank (each rank decodes
    its own batch), so the data path has no collective; the process group
    only carries the barrier and the max-over-ranks timing."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's value (step times are taken as the max over ranks)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, ms_per_step: float, world: int) -> float:
    """Whole-job throughput: every rank processes `units_per_rank` units per
    step (weak scaling) and the step takes the slowest rank's time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        sm = sorted(r[0] for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2])
                          if v.lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

class DecodeWorkload:
    """All layers' latent stores, decoders and queries of one config on the
    device. The 2-D config keeps one latent per token and layer.

    The step also carries the latent write of each sequence's newest
    token: after the T x L attention calls, the token's stacked per-loop K
    and V of every layer are encoded into the slot after the attended range
    (position N_b), so every step measures the same context.

    A paged config keeps each layer's store as a pool of pages with one
    shared block table and seeded ragged lengths; the table covers position
    N_b too, and the newest token goes there through lla_encode_paged (its
    page looked up on the device). A rotary config stores [latent | rotated
    rotary key] key rows and takes one rotary query per (layer, loop) call;
    its step is the attention calls alone."""

    def __init__(self, cfg: synth.DecodeConfig, device: str, seed_offset: int = 0):
        self.cfg = cfg
        c = cfg
        s = c.seed + seed_offset
        self.paged = c.page_size > 0
        self.rope = c.d_r > 0
        self.write_latents = not self.rope and c.dtype == "bf16" and c.d_h % 64 == 0
        n_cap = c.N + 1 if self.write_latents else c.N
        zk_shape = (c.B, n_cap, c.r_k + c.d_r) if c.two_d else (c.B, c.H, n_cap, c.r_k + c.d_r)
        zv_shape = (c.B, n_cap, c.r_v) if c.two_d else (c.B, c.H, n_cap, c.r_v)
        if self.paged:
            lens = c.lengths()
            # the table also covers position N_b, where the newest token goes
            bt, num_pages = synth.page_table(lens + 1 if self.write_latents else lens,
                                             c.page_size, s + 12)
            self.block_table = torch.from_numpy(bt).to(device)
            self.seq_lens = torch.from_numpy(lens).to(device)
            zk_shape = ((num_pages, c.page_size, c.r_k) if c.two_d
                        else (num_pages, c.H, c.page_size, c.r_k))
            zv_shape = ((num_pages, c.page_size, c.r_v) if c.two_d
                        else (num_pages, c.H, c.page_size, c.r_v))
        self.zk = [synth.latents(zk_shape, s + 1000 * l + 1, device, decay=c.decay,
                                 dtype=c.torch_dtype) for l in range(c.L)]
        self.zv = [synth.latents(zv_shape, s + 1000 * l + 2, device, decay=c.decay,
                                 dtype=c.torch_dtype) for l in range(c.L)]
        self.dk = synth.orthonormal(c.L * c.T * c.H, c.d_h, c.r_k, s + 3, device).view(
            c.L, c.T, c.H, c.d_h, c.r_k)
        self.dv = synth.orthonormal(c.L * c.T * c.H, c.d_h, c.r_v, s + 4, device).view(
            c.L, c.T, c.H, c.d_h, c.r_v)
        self.q = synth.queries((c.L, c.T, c.B, c.H, c.d_h), c.d_h, s + 5, device)
        if self.rope:
            self.q_rope = synth.queries((c.L, c.T, c.B, c.H, c.d_r), c.d_r, s + 13, device)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((c.L, c.T, c.B, c.H), device=device, dtype=torch.float32)
        import decode_attention_encode_b200 as lla
        self.lla = lla
        if self.paged:
            wsfn = (lla.lla2d_decode_attn_paged_workspace if c.two_d
                    else lla.lla_decode_attn_paged_workspace)
            need = wsfn(c.B, c.H, c.r_k, c.r_v)
        elif self.rope:
            wsfn = lla.lla2d_decode_attn_workspace if c.two_d else lla.lla_decode_attn_workspace
            need = wsfn(c.B, c.H, c.N, c.r_k + c.d_r, c.r_v)
        else:
            wsfn = lla.lla2d_decode_attn_workspace if c.two_d else lla.lla_decode_attn_workspace
            need = wsfn(c.B, c.H, c.N, c.r_k, c.r_v)
        self.ws = torch.empty(max(16, need), dtype=torch.uint8, device=device)
        self.fn = lla.lla2d_decode_attn if c.two_d else lla.lla_decode_attn
        self.scale = 1.0 / math.sqrt(c.d_h)
        if self.write_latents:
            # Encoders W_down^T [G][r][K] per (layer, axis), means, and the
            # newest token's stacked per-loop K and V [T][B][H][d_h]. Per-head
            # LLA encodes each head (G = H, K = T d_h); LLA-2D encodes the
            # whole stack of a token (G = 1, K = T H d_h). The mean term
            # mu W_down is a codec constant, formed once here.
            G, K = (1, c.T * c.H * c.d_h) if c.two_d else (c.H, c.T * c.d_h)
            self.enc_g, self.enc_k = G, K
            self.wk = synth.orthonormal(c.L * G, K, c.r_k, s + 6, device).transpose(1, 2) \
                .contiguous().to(torch.bfloat16).view(c.L, G, c.r_k, K)
            self.wv = synth.orthonormal(c.L * G, K, c.r_v, s + 7, device).transpose(1, 2) \
                .contiguous().to(torch.bfloat16).view(c.L, G, c.r_v, K)
            self.muk = synth.normal((c.L, G, K), s + 8, device, std=0.1)
            self.muv = synth.normal((c.L, G, K), s + 9, device, std=0.1)
            self.muwk = torch.stack([lla.lla_encode_bias(self.wk[l], self.muk[l]) for l in range(c.L)])
            self.muwv = torch.stack([lla.lla_encode_bias(self.wv[l], self.muv[l]) for l in range(c.L)])
            self.xk = synth.normal((c.L, c.T, c.B, c.H, c.d_h), s + 10, device, dtype=torch.bfloat16)
            self.xv = synth.normal((c.L, c.T, c.B, c.H, c.d_h), s + 11, device, dtype=torch.bfloat16)
            self.n_cap = n_cap
            d_loop = K // c.T
            need = max(lla.lla_encode_with_bias_workspace_bytes(c.T, c.B, G, d_loop, r)
                       for r in (c.r_k, c.r_v))
            self.enc_split = need > 0
            self.enc_ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)

    def step(self, q=None, out=None, lse=None, xk=None, xv=None, timers=None):
        """One looped decode step: loops outer, layers inner (each loop's
        query depends on the previous loop's output in a real model), then
        the newest token's latent write. With `timers` (launch_timers) the
        main kernel of every decode call is bracketed by its own events."""
        c = self.cfg
        q = self.q if q is None else q
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        self.plan()
        for t in range(c.T):
            for l in range(c.L):
                if timers is not None:
                    timers.next()
                self.call(l, t, q, out, lse)
        if timers is not None:
            timers.pause()
        if self.write_latents:
            self.write_newest(self.xk if xk is None else xk, self.xv if xv is None else xv)

    def plan(self):
        """A paged store's step plan, made once: every (layer, loop) call of
        the step attends the same lengths through the same table."""
        if not self.paged:
            return
        c = self.cfg
        if c.two_d:
            self.lla.lla2d_decode_attn_paged_plan(self.zk[0], self.zv[0], self.block_table,
                                                  self.seq_lens, c.H, self.ws)
        else:
            self.lla.lla_decode_attn_paged_plan(self.zk[0], self.zv[0], self.block_table,
                                                self.seq_lens, self.ws)

    def call(self, l, t, q=None, out=None, lse=None, q_rope=None):
        """The (layer l, loop t) decode call through the public API."""
        c = self.cfg
        q = self.q if q is None else q
        q_rope = getattr(self, "q_rope", None) if q_rope is None else q_rope
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        if self.paged:  # on the step's plan (plan())
            fn = self.lla.lla2d_decode_attn_paged if c.two_d else self.lla.lla_decode_attn_paged
            fn(q[l, t], self.zk[l], self.zv[l], self.block_table, self.seq_lens, self.dk[l, t],
               self.dv[l, t], scale=self.scale, out=out[l, t], lse=lse[l, t], workspace=self.ws,
               planned=True)
        elif self.rope:
            fn = self.lla.lla2d_decode_attn_rope if c.two_d else self.lla.lla_decode_attn_rope
            fn(q[l, t], q_rope[l, t], self.zk[l], self.zv[l], self.dk[l, t], self.dv[l, t], N=c.N,
               scale=self.scale, out=out[l, t], lse=lse[l, t], workspace=self.ws)
        else:
            self.fn(q[l, t], self.zk[l], self.zv[l], self.dk[l, t], self.dv[l, t], N=c.N,
                    scale=self.scale, out=out[l, t], lse=lse[l, t], workspace=self.ws)

    def write_newest(self, xk, xv):
        """Each sequence's newest token into position N_b of every layer's
        store (slot N of a dense store; through the block table of a paged
        one)."""
        c = self.cfg
        for l in range(c.L):
            for x, w, muw, z, r in ((xk, self.wk, self.muwk, self.zk, c.r_k),
                                    (xv, self.wv, self.muwv, self.zv, c.r_v)):
                xs = x[l].view(c.T, c.B, 1, c.H * c.d_h) if c.two_d else x[l]
                if self.paged:
                    self.lla.lla_encode_paged(xs, w[l], muw[l], z[l], self.block_table,
                                              self.seq_lens, workspace=self.enc_ws)
                elif c.two_d:  # x [T][B][H][d_h] read as [T][B][1][H d_h]
                    self.lla.lla_encode_with_bias(
                        x[l].view(c.T, c.B, 1, c.H * c.d_h), w[l], muw[l], z=z[l][:, c.N],
                        z_row_stride=self.n_cap * r, z_group_stride=0, workspace=self.enc_ws)
                else:
                    self.lla.lla_encode_with_bias(
                        x[l], w[l], muw[l], z=z[l][:, :, c.N], z_row_stride=c.H * self.n_cap * r,
                        z_group_stride=self.n_cap * r, workspace=self.enc_ws)

    def launches_per_step(self) -> int:
        n = 3 * self.cfg.L * self.cfg.T + (1 if self.paged else 0)
        if self.write_latents:
            n += (4 if self.enc_split else 2) * self.cfg.L
        return n


class EncodeWorkload:
    """Prefill latent write of one sequence: for every layer and both axes,
    the N tokens' stacked per-loop K (or V) vectors x [T][N][G][d_loop] are
    encoded into the [G][N][r] latent store (48 calls at 24 layers). All
    inputs are resident on the device; the encoders come from an SVD of a
    seeded N(0, 1) calibration set per (layer, axis, head)."""

    def __init__(self, cfg: synth.EncodeConfig, device: str, seed_offset: int = 0):
        import decode_attention_encode_b200 as lla
        self.lla = lla
        c = self.cfg = cfg
        s = c.seed + seed_offset
        K = c.T * c.d_loop
        self.x = [synth.normal((c.T, c.N, c.G, c.d_loop), s + 10 + i, device, dtype=torch.bfloat16)
                  for i in range(2 * c.L)]
        # codec fit: top-r right singular vectors of the centred calibration
        # matrix, per (layer, axis, head); done once, outside the timed region
        w_t, mu = [], []
        for i in range(2 * c.L):
            cal = synth.normal((c.G, c.n_cal, K), s + 1000 + i, device)
            m = cal.mean(dim=1, keepdim=True)
            _, _, vh = torch.linalg.svd(cal - m, full_matrices=False)
            w_t.append(vh[:, :c.r, :].contiguous().to(torch.bfloat16))   # [G][r][K]
            mu.append(m[:, 0, :].contiguous())                             # [G][K]
        self.w_t, self.mu = w_t, mu
        # the mean term mu W_down is a codec constant: formed once
        self.muw = [lla.lla_encode_bias(w_t[i], mu[i]) for i in range(2 * c.L)]
        self.z = [torch.empty((c.G, c.N, c.r), device=device, dtype=torch.bfloat16)
                  for _ in range(2 * c.L)]

    def step(self, x=None, timers=None):
        x = self.x if x is None else x
        for i in range(2 * self.cfg.L):
            if timers is not None:
                timers.next()
            self.lla.lla_encode_with_bias(x[i], self.w_t[i], self.muw[i], z=self.z[i],
                                          z_row_stride=self.cfg.r,
                                          z_group_stride=self.cfg.N * self.cfg.r, split=False)

    def launches_per_step(self) -> int:
        return 2 * self.cfg.L


def run_encode_bench(args, world, rank, local):
    cfg = with_layers(ENCODE_CONFIGS[args.config], args.layers)
    dev = f"cuda:{local}"
    wl = EncodeWorkload(cfg, dev, seed_offset=rank)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()
    run_step, execution = step_runner(wl.step, args.eager)
    run_step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_per_step = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    # every encode kernel of a second pass of the steps, bracketed by its own
    # pair of CUDA events that the library records on the call's stream
    timers = wl.lla.launch_timers(args.steps * wl.launches_per_step())
    with timers:
        for _ in range(args.steps):
            wl.step(timers=timers)
    kern_ms = sum(timers.ms) / len(timers.ms)
    call_bytes = (cfg.T * cfg.N * cfg.G * cfg.d_loop + cfg.G * cfg.N * cfg.r) * 2
    hbm_peak, peak_src = peaks()
    tc_peak, tc_src = tensor_peak()
    achieved = call_bytes / (kern_ms * 1e-3) / 1e9
    flops = 2 * cfg.N * cfg.G * cfg.T * cfg.d_loop * cfg.r
    tflops = flops / (kern_ms * 1e-3) / 1e12
    # which roof binds: the arithmetic intensity against the ridge point
    tensor_bound = flops / call_bytes > tc_peak * 1e12 / (hbm_peak * 1e9)
    line = {
        "metric": "LLA encode: prefill tokens encoded/sec (every layer, K and V)",
        "value": aggregate_rate(cfg.N, ms_per_step, world), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{cfg.name}: lla_encode of N={cfg.N} tokens x G={cfg.G} heads x "
                               f"{cfg.L} layers x 2 axes, stack {cfg.T}x{cfg.d_loop}, r={cfg.r}",
                   "step": f"{2 * cfg.L} encode calls", "execution": execution,
                   "accumulation": "fp32",
                   "l2": "no flush: each call reads 0.54 GB of fresh input",
                   "parallelism": f"dp{world} (independent sequences per GPU)"},
        "roofline": ({"bound": "tensor", "achieved": tflops, "peak": tc_peak, "unit": "TFLOP/s",
                      "frac": tflops / tc_peak, "hbm_gbs": achieved, "hbm_frac": achieved / hbm_peak,
                      "peak_source": tc_src}
                     if tensor_bound else
                     {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                      "frac": achieved / hbm_peak, "tensor_tflops": tflops,
                      "tensor_frac": tflops / tc_peak,
                      "peak_source": "measured: MEASURED_PEAKS.json hbm_gbs (copy, burst)"
                      if peak_src == "measured" else "fallback 6.65 TB/s"}),
        "gpu_launches": wl.launches_per_step() * args.steps,
        "clocks": clk,
        "e2e": None,
    }
    line["roofline"].update({"traffic": profiled_traffic(cfg.name), "kernel": "k_encode",
                             "kernel_ms_mean": kern_ms,
                             "kernel_timing": f"every k_encode launch of a second pass of the "
                                              f"{args.steps} timed steps, CUDA events on the "
                                              "call's stream",
                             "algorithmic_bytes_per_launch": call_bytes,
                             "algorithmic_flops_per_launch": flops})
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        n = 512
        x = wl.x[0][:, :n].double().cpu().numpy()
        w = wl.w_t[0].transpose(1, 2).double().cpu().numpy()
        mu = wl.mu[0].double().cpu().numpy()
        threads = max(1, oracle.max_threads())
        rates = {}
        for nt, budget in ((1, 6.0), (threads, 6.0)):
            t0, reps = time.perf_counter(), 0
            while True:
                oracle.encode(x, w, mu, nthreads=nt)
                reps += 1
                if time.perf_counter() - t0 >= budget:
                    break
            rates[nt] = reps * n / (2 * cfg.L) / (time.perf_counter() - t0)
        line["cpu_baseline"] = {
            "value": rates[threads], "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} tokens of one (layer, axis) call in fp64, repeated; tokens/s "
                      f"divides by the {2 * cfg.L} calls of a step",
            "single_thread": {"value": rates[1], "threads": 1},
            "all_cores": {"value": rates[threads], "threads": threads,
                          "parallel": "OpenMP over (group, token)"},
            **host_cores()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def profiled_traffic(config_name: str):
    """DRAM bytes per launch of the workload's main kernel from the committed
    ncu summary, if that summary was taken on the current kernel source."""
    kernel, src = main_kernel(config_name)
    path = os.path.join(PROFILE_DIR, f"{kernel}_{config_name}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    cur = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if not h or not t or h.group(1) != cur:
        return None
    return float(t.group(1))


def tensor_peak():
    """Dense bf16 tensor-core peak (TFLOP/s): the measured burst figure,
    since one encode launch is timed alone."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured: MEASURED_PEAKS.json bf16_tflops (burst)"
    return 1590.0, "fallback 1.59 PFLOP/s (burst)"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a fixed sample of decode units
# ---------------------------------------------------------------------------

def host_cores():
    """os.cpu_count(), the CPUs this process may run on, and nproc's answer."""
    try:
        nproc = int(subprocess.run(["nproc"], capture_output=True, text=True,
                                   timeout=10).stdout.strip())
    except Exception:
        nproc = None
    try:
        usable = len(os.sched_getaffinity(0))
    except Exception:
        usable = None
    return {"os_cpu_count": os.cpu_count(), "usable": usable, "nproc": nproc}


def unit_tokens(cfg: synth.DecodeConfig, units) -> float:
    """Cached tokens a sample of (b, layer, loop, h) units stands for: a
    (layer, loop) step attends each sequence's tokens once over all H heads,
    so a unit is N_b / H of them."""
    lens = cfg.lengths()
    return float(sum(int(lens[b]) for b, _, _, _ in units)) / cfg.H


def draw_unit_inputs(cfg: synth.DecodeConfig, units, seed: int = 0):
    """Host fp64 inputs of each sampled unit drawn with the workload's
    recipes (the reference arm has no device store to read from)."""
    lens = cfg.lengths()
    out = []
    for i, (b, l, t, h) in enumerate(units):
        n, s = int(lens[b]), seed + 10 * i
        f = lambda x: x.double().numpy()
        u = dict(q=f(synth.queries((cfg.d_h,), cfg.d_h, s)),
                 zk=f(synth.latents((n, cfg.r_k), s + 1, decay=cfg.decay, dtype=cfg.torch_dtype)),
                 zv=f(synth.latents((n, cfg.r_v), s + 2, decay=cfg.decay, dtype=cfg.torch_dtype)),
                 dk=f(synth.orthonormal(1, cfg.d_h, cfg.r_k, s + 3)[0]),
                 dv=f(synth.orthonormal(1, cfg.d_h, cfg.r_v, s + 4)[0]))
        if cfg.d_r:
            u["q_rope"] = f(synth.queries((cfg.d_r,), cfg.d_r, s + 5))
            u["k_rope"] = f(synth.latents((n, cfg.d_r), s + 6, dtype=cfg.torch_dtype))
        out.append(u)
    return out


def gather_unit_inputs(wl, units):
    """Host fp64 copies of each sampled unit's device inputs (its query, its
    own latent rows, this loop's decoders), read from the benchmark's store."""
    c = wl.cfg
    lens = c.lengths()
    f = lambda x: x.double().cpu().numpy()
    out = []
    for b, l, t, h in units:
        n = int(lens[b])
        if wl.paged:
            pos = torch.arange(n, device=wl.block_table.device)
            pages = wl.block_table[b, pos // c.page_size].long()
            rows = pos % c.page_size
            zk = wl.zk[l][pages, rows] if c.two_d else wl.zk[l][pages, h, rows]
            zv = wl.zv[l][pages, rows] if c.two_d else wl.zv[l][pages, h, rows]
        elif c.two_d:
            zk, zv = wl.zk[l][b, :n], wl.zv[l][b, :n]
        else:
            zk, zv = wl.zk[l][b, h, :n], wl.zv[l][b, h, :n]
        u = dict(q=f(wl.q[l, t, b, h]), zk=f(zk[:, :c.r_k]), zv=f(zv), dk=f(wl.dk[l, t, h]),
                 dv=f(wl.dv[l, t, h]))
        if c.d_r:
            u["q_rope"] = f(wl.q_rope[l, t, b, h])
            u["k_rope"] = f(zk[:, c.r_k:])
        out.append(u)
    return out


def run_oracle_units(cfg: synth.DecodeConfig, inputs, threads: int):
    """The oracle, as it stands, on every unit of the sample with `threads`
    host threads. Units of one length go through the oracle's batched call
    (OpenMP over units); ragged or rotary samples take one oracle call per
    unit, spread over a pool of `threads` Python threads (ctypes releases the
    interpreter lock inside the C code). Returns (out [U, d_h], lse [U])."""
    import numpy as np

    import oracle
    scale = 1.0 / math.sqrt(cfg.d_h)
    uniform = not cfg.page_size and not cfg.d_r
    if uniform:
        st = lambda k: np.stack([u[k] for u in inputs])
        return oracle.decode_units(st("q"), st("zk"), st("zv"), st("dk"), st("dv"), scale=scale,
                                   nthreads=threads)

    def one(u):
        if cfg.d_r:
            return oracle.decode_unit_rope(u["q"], u["q_rope"], u["zk"], u["k_rope"], u["zv"],
                                           u["dk"], u["dv"], scale=scale)
        o, l = oracle.decode_units(u["q"][None], u["zk"][None], u["zv"][None], u["dk"][None],
                                   u["dv"][None], scale=scale, nthreads=1)
        return o[0], float(l[0])

    if threads <= 1:
        res = [one(u) for u in inputs]
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=threads) as ex:
            res = list(ex.map(one, inputs))
    return np.stack([r[0] for r in res]), np.array([r[1] for r in res])


def oracle_rates(cfg: synth.DecodeConfig, units, inputs, single_budget_s: float = 8.0,
                 all_budget_s: float = 5.0):
    """Times the oracle on the fixed sample: single-threaded on the longest
    prefix of the sample that fits the budget (at least one unit), and on all
    host threads over the whole sample, repeated for about `all_budget_s`.
    Returns (all-core rate, record, all-core outputs)."""
    import oracle
    threads = max(1, oracle.max_threads())  # read before any call changes it
    t0 = time.perf_counter()
    run_oracle_units(cfg, inputs[:1], 1)
    t1 = time.perf_counter() - t0
    k = max(1, min(len(units), int(single_budget_s / max(t1, 1e-6))))
    if k > 1:
        t0 = time.perf_counter()
        run_oracle_units(cfg, inputs[:k], 1)
        t1 = time.perf_counter() - t0
    single = unit_tokens(cfg, units[:k]) / t1
    # whole passes over the sample until about `all_budget_s` have passed
    passes, t0 = 0, time.perf_counter()
    while True:
        res = run_oracle_units(cfg, inputs, threads)
        passes += 1
        if time.perf_counter() - t0 >= all_budget_s:
            break
    tall = (time.perf_counter() - t0) / passes
    rate = unit_tokens(cfg, units) / tall
    cores = host_cores()
    rec = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
           "sample": f"{len(units)} (b, layer, loop, h) units of this workload (32 seeded-random "
                     f"units plus the 16 corners, repeats removed), "
                     f"{'ragged lengths, ' if cfg.page_size else ''}"
                     f"explicit K/V reconstruction then textbook softmax in fp64; tokens/s "
                     f"counts N_b/H cached tokens per unit",
           "all_cores": {"value": rate, "threads": threads, "units_timed": len(units),
                         "seconds_per_pass": tall, "passes": passes,
                         "parallel": "OpenMP over units" if not cfg.page_size and not cfg.d_r
                         else "one oracle call per unit on a thread pool"},
           "single_thread": {"value": single, "threads": 1, "units_timed": k, "seconds": t1},
           **cores}
    return rate, rec, res


def cpu_baseline(wl):
    """The oracle timed on the fixed sample of the benchmark's own store, and
    that sample's GPU outputs checked against it."""
    import numpy as np
    c = wl.cfg
    units = synth.sample_units(c.B, c.L, c.T, c.H)
    inputs = gather_unit_inputs(wl, units)
    rate, rec, (ref_o, ref_l) = oracle_rates(c, units, inputs)
    idx = [list(x) for x in zip(*[(l, t, b, h) for b, l, t, h in units])]
    got = wl.out[idx[0], idx[1], idx[2], idx[3]].double().cpu().numpy()
    got_l = wl.lse[idx[0], idx[1], idx[2], idx[3]].double().cpu().numpy()
    err = float(np.abs(got - ref_o).max() / np.abs(ref_o).max())
    rec["parity"] = {"units": len(units), "max_rel_err": err,
                     "lse_max_abs_err": float(np.abs(got_l - ref_l).max()),
                     "tolerance": "max|o_gpu - o_ref| / max|o_ref| <= 2e-2"}
    return rate, rec


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, world, rank):
    """The oracle arm: each step is one all-core pass of the oracle over the
    fixed 48-unit sample of the workload (inputs drawn on the host with the
    workload's recipes); ms_per_step is that pass's measured wall time."""
    if rank != 0:
        return
    if args.config in ENCODE_CONFIGS:
        print(json.dumps({"impl": "reference", "unavailable":
                          "the reference arm times the decode workloads only"}), flush=True)
        return
    import oracle
    cfg = with_layers(synth.DECODE_CONFIGS[args.config], args.layers)
    units = synth.sample_units(cfg.B, cfg.L, cfg.T, cfg.H)
    inputs = draw_unit_inputs(cfg, units)
    threads = max(1, oracle.max_threads())
    _, rec, _ = oracle_rates(cfg, units, inputs)
    for _ in range(args.warmup):
        run_oracle_units(cfg, inputs, threads)
    step_s = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run_oracle_units(cfg, inputs, threads)
        step_s.append(time.perf_counter() - t0)
    mean_s = sum(step_s) / len(step_s)
    value = unit_tokens(cfg, units) / mean_s
    rec.update({"value": value, "all_cores": dict(rec["all_cores"], value=value,
                                                  seconds_per_pass=mean_s, passes=args.steps)})
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * mean_s, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(cfg), "parallelism": f"cpu ({threads} threads)",
                   "step": f"one all-core oracle pass over the fixed sample of {len(units)} "
                           "(b, layer, loop, h) units (a bounded sample of the decode step)"},
        "cpu_baseline": rec,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def describe(cfg: synth.DecodeConfig) -> str:
    kind = "LLA-2D" if cfg.two_d else "per-head LLA"
    n = (f"N={cfg.N} mean (ragged +-{int(cfg.spread * 100)}%, {cfg.tokens()} tokens), "
         f"{cfg.page_size}-token pages" if cfg.page_size else f"N={cfg.N}")
    rope = f" d_r={cfg.d_r} (rotary branch)" if cfg.d_r else ""
    return (f"{cfg.name}: {kind} decode, L={cfg.L} T={cfg.T} H={cfg.H} d_h={cfg.d_h} "
            f"r_k={cfg.r_k}{rope} r_v={cfg.r_v} B={cfg.B} {n} {cfg.dtype} latents")


def run_lla(args, world, rank, local):
    cfg = with_layers(synth.DECODE_CONFIGS[args.config], args.layers)
    dev = f"cuda:{local}"
    wl = DecodeWorkload(cfg, dev, seed_offset=rank)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()
    run_step, execution = step_runner(wl.step, args.eager)
    run_step()
    torch.cuda.synchronize()

    # device-timed region
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for _ in range(args.steps):
        run_step()
    ev[1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed_ms = ev[0].elapsed_time(ev[1])
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    ms_per_step = elapsed_ms / args.steps

    # each whole call of one eager step's first loop, timed on its own
    call_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(cfg.L)]
    wl.plan()
    for t in range(cfg.T):
        for l in range(cfg.L):
            if t == 0:
                call_ev[l][0].record(stream)
            wl.call(l, t)
            if t == 0:
                call_ev[l][1].record(stream)
    if wl.write_latents:
        wl.write_newest(wl.xk, wl.xv)
    torch.cuda.synchronize()
    call_ms = sorted(a.elapsed_time(b) for a, b in call_ev)
    call_ms_mean = sum(call_ms) / len(call_ms)

    # the main kernel alone: a second pass over the same steps in which the
    # library brackets every main-kernel launch with its own pair of CUDA
    # events on the call's stream (kept out of the first pass, which gives
    # value and ms_per_step: an event between two programmatically launched
    # kernels would order them fully)
    timers = wl.lla.launch_timers(args.steps * cfg.L * cfg.T)
    with timers:
        for _ in range(args.steps):
            wl.step(timers=timers)
    kern_ms_mean = sum(timers.ms) / len(timers.ms)

    tokens_per_step = cfg.tokens() * cfg.L * cfg.T
    value = aggregate_rate(tokens_per_step, ms_per_step, world)
    step_bytes = cfg.step_bytes()
    hbm_peak, peak_src = peaks()
    achieved = step_bytes / (kern_ms_mean * 1e-3) / 1e9
    kname, _ = main_kernel(cfg.name)

    # End to end through the public API: every step copies its inputs (the
    # queries of every (layer, loop) call and the newest token's per-loop K/V)
    # from pinned host memory and reads every output back into pinned host
    # memory. Copies run on their own streams, chunked per call, so they
    # overlap the decode calls; the timed region ends when the last output
    # has landed on the host.
    e2e = None
    if not args.no_e2e:
        c = cfg
        h2d = torch.cuda.Stream()
        d2h = torch.cuda.Stream()
        q_host = wl.q.to("cpu").pin_memory()
        q_dev = torch.empty_like(wl.q)
        qr_host = wl.q_rope.to("cpu").pin_memory() if wl.rope else None
        qr_dev = torch.empty_like(wl.q_rope) if wl.rope else None
        # a paged store's per-step inputs: lengths and block table (a serving
        # loop grows them every step); the decode calls read the device copies
        pg_hosts = [wl.seq_lens.to("cpu").pin_memory(), wl.block_table.to("cpu").pin_memory()] \
            if wl.paged else []
        pg_devs = [wl.seq_lens, wl.block_table] if wl.paged else []
        x_hosts = [wl.xk.to("cpu").pin_memory(), wl.xv.to("cpu").pin_memory()] \
            if wl.write_latents else []
        x_devs = [torch.empty_like(wl.xk), torch.empty_like(wl.xv)] if wl.write_latents else []
        out_host = torch.empty(wl.out.shape, dtype=torch.float32).pin_memory()
        lse_host = torch.empty(wl.lse.shape, dtype=torch.float32).pin_memory()
        # Each buffer waits only for its own last use: call (l, t)'s query
        # copy for the next step waits for this step's call (l, t), its
        # output for this step's read-back of (l, t), so one step's copies
        # run under the neighbouring steps' calls.
        ev = lambda: [[torch.cuda.Event() for _ in range(c.L)] for _ in range(c.T)]
        in_ev, done_ev, back_ev = ev(), ev(), ev()
        x_ev, wrote_ev, pg_ev = (torch.cuda.Event() for _ in range(3))
        state = {"first": True}

        def e2e_step():
            first = state["first"]
            state["first"] = False
            with torch.cuda.stream(h2d):
                if first or wl.paged:
                    # a paged step's lengths and table are free once the
                    # whole previous step is done (a separate copy stream
                    # waiting on the step's end measured 4-6% slower)
                    h2d.wait_stream(stream)
                for d_, h_ in zip(pg_devs, pg_hosts):
                    d_.copy_(h_, non_blocking=True)
                pg_ev.record(h2d)
                for t in range(c.T):
                    for l in range(c.L):
                        if not first:
                            h2d.wait_event(done_ev[t][l])  # the previous step's call (l, t)
                        q_dev[l, t].copy_(q_host[l, t], non_blocking=True)
                        if wl.rope:
                            qr_dev[l, t].copy_(qr_host[l, t], non_blocking=True)
                        in_ev[t][l].record(h2d)
                if not first:
                    h2d.wait_event(wrote_ev)  # the previous step's latent write
                for d_, h_ in zip(x_devs, x_hosts):
                    d_.copy_(h_, non_blocking=True)
                x_ev.record(h2d)
            if wl.paged:  # the step's plan reads the lengths and table just copied
                stream.wait_event(pg_ev)
                wl.plan()
            for t in range(c.T):
                for l in range(c.L):
                    stream.wait_event(in_ev[t][l])
                    if not first:
                        stream.wait_event(back_ev[t][l])  # out[l, t] has been read back
                    wl.call(l, t, q=q_dev, q_rope=qr_dev)
                    done_ev[t][l].record(stream)
                    with torch.cuda.stream(d2h):
                        d2h.wait_event(done_ev[t][l])
                        out_host[l, t].copy_(wl.out[l, t], non_blocking=True)
                        lse_host[l, t].copy_(wl.lse[l, t], non_blocking=True)
                        back_ev[t][l].record(d2h)
            if wl.write_latents:
                stream.wait_event(x_ev)
                wl.write_newest(*x_devs)
            wrote_ev.record(stream)

        for _ in range(2):
            e2e_step()
        stream.wait_stream(d2h)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        stream.wait_stream(d2h)  # the last outputs have landed on the host
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
        e2e = {"value": aggregate_rate(tokens_per_step, e2e_ms, world), "unit": UNIT,
               "h2d_bytes_per_step": (q_host.numel() + (qr_host.numel() if wl.rope else 0)) * 4
                                     + sum(h_.numel() * 2 for h_ in x_hosts)
                                     + sum(h_.numel() * 4 for h_ in pg_hosts),
               "d2h_bytes_per_step": (out_host.numel() + lse_host.numel()) * 4,
               "copies": "pinned host memory, per-call chunks on separate copy streams"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": describe(cfg),
            "execution": execution,
            "step": (f"one plan kernel, then " if wl.paged else "")
                    + f"{cfg.L * cfg.T} decode calls (T loops x L layers), 3 kernels each"
                    + (f", then {2 * cfg.L} latent writes of the newest token" if wl.write_latents else ""),
            "accumulation": "fp32",
            "l2": "no flush: each layer's latent store "
                  f"({step_bytes / 1e9:.2f} GB) is larger than L2 (126 MB)",
            "parallelism": f"dp{world} (independent sequences per GPU)",
            "global_batch": cfg.B * world, "seq_len": cfg.N,
        },
        "hbm_gbs_per_call": step_bytes / (call_ms_mean * 1e-3) / 1e9,
        # per-head decode reads each cached token once per head
        "token_head_reads_per_s": None if cfg.two_d else value * cfg.H,
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "traffic": profiled_traffic(cfg.name),
            "kernel": kname, "kernel_ms_mean": kern_ms_mean,
            "kernel_timing": f"every {kname} launch of a second pass of the {args.steps} timed "
                             "steps, CUDA events on the call's stream",
            "algorithmic_bytes_per_launch": step_bytes,
            "peak_source": "measured: MEASURED_PEAKS.json hbm_gbs (copy, burst)"
            if peak_src == "measured" else "fallback 6.65 TB/s",
        },
        "call_ms": {"mean": call_ms_mean, "min": call_ms[0], "max": call_ms[-1]},
        "gpu_launches": wl.launches_per_step() * args.steps,
        "clocks": clk,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        _, line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup("nccl")
    try:
        if args.config in ENCODE_CONFIGS:
            run_encode_bench(args, world, rank, local)
        else:
            run_lla(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

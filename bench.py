#!/usr/bin/env python3
"""Benchmark of the scaled-FP8 cast path on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch of synthetic inputs
that are resident in HBM before the timed region starts:

  per-token group quant   bf16 x[4096, 7168], group 128, e4m3fn   (+ its round trip
                          back to bf16 through cast_from_fp8, group granularity)
  block dequant           e4m3fn W[7168, 18432], 128 x 128 scales -> bf16
  per-channel cast        bf16 X[8192, 8192] -> e4m3fn, one scale per row
  per-tensor cast         fp32 v[64 Mi] -> e5m2; fp16 [1 Mi] zeros -> e4m3fn
  grouped block dequant   64 x [2048, 7168] + 8 x [7000, 1000] e4m3fn -> bf16

`value` is the step's algorithmic bytes (each input read once per pass the
method needs, each output written once) divided by the device time of the
step, in GB/s, summed over ranks.  The step streams ~4.4 GB, far more than
the 126 MB L2, so no operation finds its inputs in L2 from the previous step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Beside the step, rank 0 reports measurements that are not part of `value`:
"isolated" times per-token quant, block dequant, the round trip, the
per-channel and the fp32 per-tensor casts each alone, over rotating buffer
sets at least 4x the L2 size (each launch reads cold inputs and pays for the
write-back of one launch of its own outputs), as the median and p10 / p90 of
blocks of back-to-back launches; "matmul" times the two fp8 products on the
tensor cores (TFLOP/s against the fp8 peak) beside the library products on
the same operands (torch._scaled_mm / cuBLASLt for per-tensor scales; torch's
blockwise scaled_mm and vLLM's CUTLASS blockwise product for the per-token x
128 x 128-block scales), then each product back to back for two seconds
under the board's power cap (--no-matmul skips the section).

With N > 1 it runs under torchrun, one rank per GPU, each rank doing the full
step on its own copy of the inputs (independent problems, weak scaling, no
data-path collective); the time is the max over ranks.  Beside it, every
rank then runs the method's two exchange steps ("sharded": the per-tensor
cast of a tensor split over the ranks with its 4-byte int32 MAX all-reduce,
and the fp8 all-gather beside a bf16 NCCL all-gather); --sharded runs them
at N = 1 too.  `--marginal` prints each op's marginal cost inside the live
step instead.  `--impl reference` times the CPU oracle on a bounded sample
of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "achieved HBM GB/s and % of B200 peak for per-token quant and block dequant"
UNIT = "GB/s"
WORKLOAD = ("scaled-fp8 cast pass: per-token quant bf16[4096,7168] g128 e4m3fn + round trip to bf16; "
            "block dequant e4m3fn[7168,18432] B128 -> bf16; per-channel bf16[8192,8192] -> e4m3fn; "
            "per-tensor f32[64Mi] -> e5m2 and f16[1Mi] zeros -> e4m3fn; "
            "grouped block dequant 64x[2048,7168] + 8x[7000,1000] -> bf16")
E4M3FN, E5M2 = 0, 1
GRAN_GROUP = 2


# ---------------------------------------------------------------------------
# the workload: inputs, outputs, algorithmic bytes, and the step
# ---------------------------------------------------------------------------
class Op:
    """One call of the step: `ins` are the tensors it reads that come from the
    host in an end-to-end run, `outs` the tensors it writes."""

    def __init__(self, name, fn, bytes_, launches, kernel, ins=(), outs=(), elems=0):
        self.name, self.fn, self.bytes, self.launches, self.kernel = name, fn, bytes_, launches, kernel
        self.ins, self.outs = list(ins), list(outs)
        self.elems = elems          # elements the op converts


class Workload:
    """All inputs of one step on `device`, outputs preallocated, plus the op list."""

    def __init__(self, device, fp8q, host_inputs=None):
        self.device = device
        self.fp8q = fp8q
        h = host_inputs if host_inputs is not None else make_host_inputs()
        self.host = h
        d = device
        bf16 = torch.bfloat16
        to = lambda a, dt=None: _to_dev(a, d, dt)  # noqa: E731

        m, n = workloads.C2_SHAPE
        self.c2_x = to(h["c2_x"], bf16)
        self.c2_q = torch.empty((m, n), dtype=torch.uint8, device=d)
        self.c2_s = torch.empty((m, n // 128), dtype=torch.float32, device=d)
        self.c2_y = torch.empty((m, n), dtype=bf16, device=d)

        M, N = workloads.C3_SHAPE
        self.c3_w = to(h["c3_w"])
        self.c3_s = to(h["c3_s"])
        self.c3_y = torch.empty((M, N), dtype=bf16, device=d)

        R, C = workloads.C4A_SHAPE
        self.c4a_x = to(h["c4a_x"], bf16)
        self.c4a_q = torch.empty((R, C), dtype=torch.uint8, device=d)
        self.c4a_s = torch.empty((R,), dtype=torch.float32, device=d)

        self.c4b_x = to(h["c4b_v"])
        self.c4b_q = torch.empty((workloads.C4B_NUMEL,), dtype=torch.uint8, device=d)
        self.c4b_s = torch.empty((1,), dtype=torch.float32, device=d)
        self.c4c_x = to(h["c4c_v"], torch.float16)
        self.c4c_q = torch.empty((workloads.C4C_NUMEL,), dtype=torch.uint8, device=d)
        self.c4c_s = torch.empty((1,), dtype=torch.float32, device=d)
        self.ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device=d)

        self.c5_w = [to(w) for w, _ in h["c5"]]
        self.c5_s = [to(s) for _, s in h["c5"]]
        self.c5_y = [torch.empty(w.shape, dtype=bf16, device=d) for w in self.c5_w]

        c2_el = m * n
        c2_bytes = c2_el * 2 + c2_el + c2_el // 128 * 4
        c3_el = M * N
        c3_bytes = c3_el + c3_el * 2 + self.c3_s.numel() * 4
        c4a_bytes = R * C * 2 + R * C + R * 4
        c4b_bytes = 2 * workloads.C4B_NUMEL * 4 + workloads.C4B_NUMEL + 4
        c4c_bytes = 2 * workloads.C4C_NUMEL * 2 + workloads.C4C_NUMEL + 4
        c5_el = sum(w.numel() for w in self.c5_w)
        c5_bytes = c5_el * 3 + sum(s.numel() for s in self.c5_s) * 4
        f = fp8q
        # Each op pays for the dirty L2 lines (up to ~60 MB) the op before it
        # left; the tiny fp16 zero-tensor cast follows the 3 GB grouped dequant
        # of the previous step, so that write-back lands on it rather than on
        # the per-token quant.  The step total does not depend on the order.
        self.ops = [
            Op("cast_per_tensor_f16_zero", lambda: f.fp8q_cast_per_tensor(self.c4c_x, self.c4c_q, self.c4c_s, self.ws, E4M3FN),
               c4c_bytes, 2, "tensor_amax_kernel+tensor_cast_kernel", [self.c4c_x], [self.c4c_q, self.c4c_s],
               workloads.C4C_NUMEL),
            Op("per_token_group_quant", lambda: f.fp8q_per_token_group_quant(self.c2_x, self.c2_q, self.c2_s, 128, E4M3FN),
               c2_bytes, 1, "per_token_vec_kernel", [self.c2_x], [self.c2_q, self.c2_s], c2_el),
            Op("block_dequant", lambda: f.fp8q_block_dequant(self.c3_w, self.c3_s, self.c3_y, 128, E4M3FN),
               c3_bytes, 1, "dequant_kernel", [self.c3_w, self.c3_s], [self.c3_y], c3_el),
            # the round trip reads q after the block dequant has streamed ~400 MB
            # through L2, so it finds no q bytes left in L2
            Op("cast_from_fp8_group", lambda: f.fp8q_cast_from_fp8(self.c2_q, self.c2_s, self.c2_y, GRAN_GROUP, 128, E4M3FN),
               c2_bytes, 1, "dequant_kernel", [], [self.c2_y], c2_el),
            Op("cast_per_channel", lambda: f.fp8q_cast_per_channel(self.c4a_x, self.c4a_q, self.c4a_s, E4M3FN),
               c4a_bytes, 1, "per_channel_vec_kernel", [self.c4a_x], [self.c4a_q, self.c4a_s], R * C),
            Op("cast_per_tensor_f32_e5m2", lambda: f.fp8q_cast_per_tensor(self.c4b_x, self.c4b_q, self.c4b_s, self.ws, E5M2),
               c4b_bytes, 2, "tensor_amax_kernel+tensor_cast_kernel", [self.c4b_x], [self.c4b_q, self.c4b_s],
               workloads.C4B_NUMEL),
            Op("block_dequant_grouped", lambda: f.fp8q_block_dequant_grouped(self.c5_w, self.c5_s, self.c5_y, 128, E4M3FN),
               c5_bytes, 1, "dequant_kernel", [*self.c5_w, *self.c5_s], self.c5_y, c5_el),
        ]
        self.step_bytes = sum(o.bytes for o in self.ops)
        self.launches_per_step = sum(o.launches for o in self.ops)

    def step(self, events=None, only=None):
        """One pass over every op.  events: a (start, end) pair per op, or, with
        only = i, one pair recorded around op i alone."""
        for i, op in enumerate(self.ops):
            ev = None if events is None else (events if only is not None else events[i])
            if ev is not None and (only is None or only == i):
                ev[0].record()
            op.fn()
            if ev is not None and (only is None or only == i):
                ev[1].record()

    # host<->device traffic of one end-to-end step
    def inputs(self):
        return [t for op in self.ops for t in op.ins]

    def outputs(self):
        return [t for op in self.ops for t in op.outs]


class EndToEnd:
    """The step from pinned host memory to pinned host memory.  The step's ops
    are cut into units -- rows or weights of an op whose rows (weights) are
    independent, the whole op otherwise (the per-tensor casts need their
    whole tensor) -- and each unit's inputs go host->device on a copy-in
    stream, the unit runs on the compute stream, its outputs go device->host
    on a copy-out stream.  Events order each unit's three parts and keep the
    next step from overwriting a buffer still in use, so the upload of one
    unit overlaps the compute and download of the ones before it (PCIe
    carries both directions at once) and a large op starts downloading
    after its first unit rather than after its last."""

    def __init__(self, wl: Workload, chunks: int = 4, weight_chunks: int = 8):
        self.wl = wl
        f = wl.fp8q
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)  # noqa: E731
        self.h = {}
        for t in wl.inputs():
            self.h[id(t)] = pin(t)
            self.h[id(t)].copy_(t)
        for t in wl.outputs():
            self.h[id(t)] = pin(t)
        H = lambda t: self.h[id(t)]  # noqa: E731

        def rows(n, k):
            step = -(-n // k)
            step = -(-step // 128) * 128              # whole 128-row blocks (block-scale rows)
            return [(r, min(n, r + step)) for r in range(0, n, step)]

        units = []
        for op in wl.ops:
            if op.name == "per_token_group_quant":
                x, q, sc = wl.c2_x, wl.c2_q, wl.c2_s
                for r0, r1 in rows(x.shape[0], chunks):
                    units.append(((lambda a=x[r0:r1], b=q[r0:r1], c=sc[r0:r1]:
                                   f.fp8q_per_token_group_quant(a, b, c, 128, E4M3FN)),
                                  [(x[r0:r1], H(x)[r0:r1])], [(q[r0:r1], H(q)[r0:r1]), (sc[r0:r1], H(sc)[r0:r1])]))
            elif op.name == "block_dequant":
                w, sc, y = wl.c3_w, wl.c3_s, wl.c3_y
                for r0, r1 in rows(w.shape[0], chunks):
                    b0, b1 = r0 // 128, -(-r1 // 128)
                    units.append(((lambda a=w[r0:r1], b=sc[b0:b1], c=y[r0:r1]:
                                   f.fp8q_block_dequant(a, b, c, 128, E4M3FN)),
                                  [(w[r0:r1], H(w)[r0:r1]), (sc[b0:b1], H(sc)[b0:b1])], [(y[r0:r1], H(y)[r0:r1])]))
            elif op.name == "cast_from_fp8_group":
                q, sc, y = wl.c2_q, wl.c2_s, wl.c2_y
                for r0, r1 in rows(q.shape[0], chunks):
                    units.append(((lambda a=q[r0:r1], b=sc[r0:r1], c=y[r0:r1]:
                                   f.fp8q_cast_from_fp8(a, b, c, GRAN_GROUP, 128, E4M3FN)),
                                  [], [(y[r0:r1], H(y)[r0:r1])]))
            elif op.name == "cast_per_channel":
                x, q, sc = wl.c4a_x, wl.c4a_q, wl.c4a_s
                for r0, r1 in rows(x.shape[0], chunks):
                    units.append(((lambda a=x[r0:r1], b=q[r0:r1], c=sc[r0:r1]:
                                   f.fp8q_cast_per_channel(a, b, c, E4M3FN)),
                                  [(x[r0:r1], H(x)[r0:r1])], [(q[r0:r1], H(q)[r0:r1]), (sc[r0:r1], H(sc)[r0:r1])]))
            elif op.name == "block_dequant_grouped":
                n = len(wl.c5_w)
                step = -(-n // weight_chunks)
                for i in range(0, n, step):
                    ws, ss, ys = wl.c5_w[i:i + step], wl.c5_s[i:i + step], wl.c5_y[i:i + step]
                    units.append(((lambda a=ws, b=ss, c=ys: f.fp8q_block_dequant_grouped(a, b, c, 128, E4M3FN)),
                                  [(t, H(t)) for t in ws + ss], [(t, H(t)) for t in ys]))
            else:
                units.append((op.fn, [(t, H(t)) for t in op.ins], [(t, H(t)) for t in op.outs]))
        self.units = units
        self.s_in, self.s_comp, self.s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        self.done_comp = [None] * len(units)
        self.done_out = [None] * len(units)
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in wl.inputs())
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in wl.outputs())
        assert self.h2d_bytes == sum(d.numel() * d.element_size() for _, ins, _ in units for d, _ in ins)
        assert self.d2h_bytes == sum(d.numel() * d.element_size() for _, _, outs in units for d, _ in outs)

    def step(self):
        for i, (fn, ins, outs) in enumerate(self.units):
            with torch.cuda.stream(self.s_in):
                if self.done_comp[i] is not None:
                    self.s_in.wait_event(self.done_comp[i])      # previous step's unit i has read its inputs
                for d, hst in ins:
                    d.copy_(hst, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(self.s_in)
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(ev_in)
                if self.done_out[i] is not None:
                    self.s_comp.wait_event(self.done_out[i])     # previous step's outputs are on the host
                fn()
                ev_c = torch.cuda.Event()
                ev_c.record(self.s_comp)
                self.done_comp[i] = ev_c
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(ev_c)
                for d, hst in outs:
                    hst.copy_(d, non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(self.s_out)
                self.done_out[i] = ev_o

    def time(self, steps: int) -> float:
        """Milliseconds per step on the device clock (first upload to last download)."""
        self.step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.s_in)
        for _ in range(steps):
            self.step()
        self.s_out.wait_stream(self.s_comp)
        self.s_out.wait_stream(self.s_in)
        e1.record(self.s_out)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps


def shard_range(numel: int, world: int, rank: int, align: int = 8):
    """[start, stop) of `rank`'s shard of a flat tensor: equal shards, each a multiple of
    `align` elements (32-byte aligned for fp32), the last one shorter or empty."""
    per = -(-numel // world)
    per = -(-per // align) * align
    start = min(numel, rank * per)
    return start, min(numel, start + per)


class LegKernels:
    """The device work of the sharded leg, through libfp8q's binding."""

    def __init__(self, fp8q):
        self.f = fp8q

    def tensor_amax(self, x, amax_bits, ws):
        self.f.fp8q_tensor_amax(x, amax_bits, ws)

    def cast_with_amax(self, x, amax_bits, q, scale_inv):
        self.f.fp8q_cast_per_tensor_with_amax(x, amax_bits, q, scale_inv, E5M2)

    def all_gather_fp8(self, out, x, group):
        self.f.all_gather_fp8(out, x, group, "e5m2")


class ShardedLeg:
    """The method's two exchange steps across the ranks of a torchrun job, timed beside the
    replicas headline (they are not part of `value`):

      cast_to_fp8_sharded  the per-tensor e5m2 cast of the fp32 v[64 Mi] tensor split over the
                           ranks: each rank's amax pass over its shard, an int32 MAX all-reduce
                           of the 4-byte amax bits, then each rank's cast pass with the global
                           amax (ColossalAI fp8_compress_fsdp_params_comm_hook's all_reduce(MAX))
      all_gather_fp8       each rank's bf16 shard of `gather_elems` elements cast with its own
                           scale into a record, one NCCL all-gather of the records, every record
                           dequantised (ColossalAI all_gather_fp8), beside a plain bf16 NCCL
                           all_gather_into_tensor of the same shards

    Times are per call, CUDA events on the current stream, the max over ranks.  `kernels` and
    `timer` are the device work and the clock; tests pass host stand-ins to run the rest of
    the leg (sharding, buffers, exchanges, byte counts) on gloo ranks."""

    def __init__(self, device, rank, world, v_host, gather_elems=1 << 24, group=None, kernels=None,
                 timer=None, ws_bytes=8192, seed=20261208):
        self.device, self.rank, self.world, self.group = device, rank, world, group
        self.k = kernels
        self.timer = timer or _device_timer
        self.numel = int(v_host.size)
        s0, s1 = shard_range(self.numel, world, rank)
        self.shard = (s0, s1)
        self.x = _to_dev(np.ascontiguousarray(v_host[s0:s1]), device)
        self.q = torch.empty((s1 - s0,), dtype=torch.uint8, device=device)
        self.sinv = torch.empty((1,), dtype=torch.float32, device=device)
        self.amax = torch.zeros((1,), dtype=torch.int32, device=device)
        self.ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=device)
        g = np.random.default_rng(seed + rank)
        self.gather_elems = int(gather_elems)
        self.g = _to_dev(workloads.to_bf16_bits(g.standard_normal(self.gather_elems, dtype=np.float32)),
                         device, torch.bfloat16)
        self.out = torch.empty((world * self.gather_elems,), dtype=torch.bfloat16, device=device)

    def cast_sharded(self):
        import dequantisation_fp8q_token_b200 as fp8q
        self.k.tensor_amax(self.x, self.amax, self.ws)
        fp8q.allreduce_amax_bits(self.amax, self.group)
        self.k.cast_with_amax(self.x, self.amax, self.q, self.sinv)

    def gather_fp8(self):
        self.k.all_gather_fp8(self.out, self.g, self.group)

    def gather_bf16(self):
        import torch.distributed as dist
        dist.all_gather_into_tensor(self.out, self.g, group=self.group)

    def _time(self, fn, reps, warmup):
        for _ in range(warmup):
            fn()
        barrier(self.world)
        return max_over_ranks(self.timer(fn, reps, self.device), self.world, self.device)

    def run(self, reps: int = 20, warmup: int = 3):
        import dequantisation_fp8q_token_b200 as fp8q
        import torch.distributed as dist
        res = {}
        ms = self._time(self.cast_sharded, reps, warmup)
        # every rank must hold the one scale_inv that the global amax gives
        same = True
        if self.world > 1:
            allsinv = torch.empty((self.world,), dtype=torch.float32, device=self.device)
            dist.all_gather_into_tensor(allsinv, self.sinv, group=self.group)
            bits = allsinv.view(torch.int32).cpu()
            same = bool((bits == bits[0]).all())
        nbytes = 2 * self.numel * 4 + self.numel + 4
        res["cast_to_fp8_sharded"] = {
            "what": "per-tensor e5m2 cast of fp32 v[64 Mi] split over the ranks: amax pass, int32 MAX "
                    "all-reduce of 4 bytes, cast pass",
            "elements_total": self.numel, "elements_this_rank": self.shard[1] - self.shard[0],
            "us": round(ms * 1e3, 2), "bytes_total": nbytes, "gb_s_total": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "allreduce_bytes": 4, "scale_inv_identical_on_all_ranks": same}
        R = fp8q.record_bytes(self.gather_elems)
        ms8 = self._time(self.gather_fp8, reps, warmup)
        gathered = self.world * self.gather_elems * 2          # bf16 bytes every rank ends up with
        e = {"what": "each rank's bf16 shard cast into a [scale | e5m2 codes] record, one NCCL all-gather "
                     "of the records, every record dequantised to bf16",
             "elements_per_rank": self.gather_elems, "record_bytes": R,
             "wire_bytes_received_per_rank": (self.world - 1) * R,
             "bf16_wire_bytes_received_per_rank": (self.world - 1) * 2 * self.gather_elems,
             "us": round(ms8 * 1e3, 2), "bf16_gb_s_gathered": round(gathered / (ms8 * 1e-3) / 1e9, 1)}
        if self.world > 1:
            ms16 = self._time(self.gather_bf16, reps, warmup)
            e["nccl_bf16_all_gather_us"] = round(ms16 * 1e3, 2)
            e["nccl_bf16_gb_s_gathered"] = round(gathered / (ms16 * 1e-3) / 1e9, 1)
            e["speedup_vs_bf16"] = round(ms16 / ms8, 3)
        res["all_gather_fp8"] = e
        res["ranks"] = self.world
        return res


def _device_timer(fn, reps, device):
    """Milliseconds per call of fn: CUDA events around `reps` calls on the current stream."""
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / reps


def pcie_bound(h2d_bytes: int, d2h_bytes: int, device, n: int = 1 << 30):
    """The fastest the end-to-end step's transfers can go on this machine: pinned copies of n bytes
    each way, alone and both at once (CUDA events), then the step's bytes moved both ways at the
    shared rate and the remainder of the larger direction at its own rate."""
    h1 = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    h2 = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    d1 = torch.empty(n, dtype=torch.uint8, device=device)
    d2 = torch.empty(n, dtype=torch.uint8, device=device)
    s1, s2 = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def timed(fn, reps=4):
        fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / reps

    def both():
        cur = torch.cuda.current_stream(device)
        s1.wait_stream(cur)
        s2.wait_stream(cur)
        with torch.cuda.stream(s1):
            d1.copy_(h1, non_blocking=True)
        with torch.cuda.stream(s2):
            h2.copy_(d2, non_blocking=True)
        cur.wait_stream(s1)
        cur.wait_stream(s2)
    up = n / timed(lambda: d1.copy_(h1, non_blocking=True)) / 1e6        # GB/s
    down = n / timed(lambda: h2.copy_(d2, non_blocking=True)) / 1e6
    shared = n / timed(both) / 1e6
    common = min(h2d_bytes, d2h_bytes)
    rest_up, rest_down = h2d_bytes - common, d2h_bytes - common
    ms = common / shared / 1e6 + rest_up / up / 1e6 + rest_down / down / 1e6
    del h1, h2, d1, d2
    torch.cuda.empty_cache()
    return {"h2d_gb_s": round(up, 1), "d2h_gb_s": round(down, 1), "both_gb_s_each": round(shared, 1),
            "bound_ms_per_step": round(ms, 3)}


def _quantile(v, q):
    """The q-quantile of a sorted list (nearest rank)."""
    return v[min(len(v) - 1, int(round(q * (len(v) - 1))))]


def isolated_timing(wl: Workload, launches: int = 60, min_footprint: int = 0):
    """Each op the metric names, timed alone in a steady state: the op runs
    over `sets` copies of its buffers, rotating, with the sets together at
    least 4x the L2 size, so every launch reads cold inputs and pays for the
    write-back of exactly one launch's outputs (its own kind).

    `us` and its p10 / p50 / p90: the op's launches over every set, captured
    once in a CUDA graph (the same kernels with the same arguments; the
    launches keep their programmatic-dependent-launch attribute) and replayed
    `blocks` times, one event pair per replay (the per-launch mean of each
    replay is one sample).  Launched one by one from Python instead, a short
    op is bound by the binding's host cost (~10-12 us a call, `host_us_per_call`):
    the 89 MB per-token quant reads 14.4-14.9 us that way against 13.2 us from
    the graph on B200, so that figure (`us_stream`, blocks of back-to-back
    launches) is reported beside it, not as the op's time.  An event pair
    around every single launch (`us_event_per_launch`) overstates a short
    kernel further: an event between two kernels serialises them and exposes
    the launch latency that back-to-back launches hide."""
    f = wl.fp8q
    d = wl.device
    l2 = torch.cuda.get_device_properties(d).L2_cache_size
    need = max(4 * l2, min_footprint)
    blocks = 10
    per_block = max(1, launches // blocks)
    out = {}

    def run(name, make_set, footprint, nbytes, elems):
        sets = [make_set(i) for i in range(max(1, -(-need // footprint)))]
        # warm up for at least 10 ms of launches, so the clocks have settled before timing
        t0 = time.perf_counter()
        k = 0
        while k < len(sets) or time.perf_counter() - t0 < 0.01:
            sets[k % len(sets)]()
            k += 1
            if k % 32 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        # the binding's host cost per call (no synchronisation inside)
        t0 = time.perf_counter()
        for j in range(4 * len(sets)):
            sets[j % len(sets)]()
        host_us = (time.perf_counter() - t0) / (4 * len(sets)) * 1e6
        torch.cuda.synchronize()
        # launched one by one from Python: blocks of back-to-back launches
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(blocks)]
        k = 0
        for b in range(blocks):
            evs[b][0].record()
            for _ in range(per_block):
                sets[k % len(sets)]()
                k += 1
            evs[b][1].record()
        torch.cuda.synchronize()
        blk = sorted(a.elapsed_time(e) * 1e3 / per_block for a, e in evs)
        # the same launches replayed from a CUDA graph: per_block launches of every set
        nl = per_block * len(sets)
        side = torch.cuda.Stream(d)
        side.wait_stream(torch.cuda.current_stream(d))
        with torch.cuda.stream(side):
            for j in range(nl):
                sets[j % len(sets)]()
        torch.cuda.current_stream(d).wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        # thread-local capture: other threads (a process group's watchdog under torchrun) keep
        # making CUDA calls while this thread captures
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            for j in range(nl):
                sets[j % len(sets)]()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(blocks)]
        for b in range(blocks):
            gev[b][0].record()
            graph.replay()
            gev[b][1].record()
        torch.cuda.synchronize()
        rep = sorted(a.elapsed_time(e) * 1e3 / nl for a, e in gev)
        del graph
        one = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
        for j in range(launches):
            one[j][0].record()
            sets[j % len(sets)]()
            one[j][1].record()
        torch.cuda.synchronize()
        durs = sorted(a.elapsed_time(e) * 1e3 for a, e in one)
        us = statistics.median(rep)
        us_stream = statistics.median(blk)
        out[name] = {"us": round(us, 2), "gb_s": round(nbytes / (us * 1e-6) / 1e9, 1),
                     "gelem_s": round(elems / (us * 1e-6) / 1e9, 2),
                     "us_p10_p50_p90": [round(_quantile(rep, q), 2) for q in (0.1, 0.5, 0.9)],
                     "launches": blocks * nl, "replays": blocks, "timing": "cuda_graph_replay",
                     "us_stream": round(us_stream, 2), "gb_s_stream": round(nbytes / (us_stream * 1e-6) / 1e9, 1),
                     "us_stream_p10_p50_p90": [round(_quantile(blk, q), 2) for q in (0.1, 0.5, 0.9)],
                     "host_us_per_call": round(host_us, 1),
                     "us_event_per_launch": round(statistics.median(durs), 2),
                     "us_event_per_launch_p10_p50_p90": [round(_quantile(durs, q), 2) for q in (0.1, 0.5, 0.9)],
                     "sets": len(sets)}
        del sets
        torch.cuda.empty_cache()

    m, n = wl.c2_x.shape
    c2_bytes = m * n * 3 + m * (n // 128) * 4

    def per_token_set(i):
        x = wl.c2_x if i == 0 else wl.c2_x.clone()
        q = torch.empty((m, n), dtype=torch.uint8, device=d)
        s = torch.empty((m, n // 128), dtype=torch.float32, device=d)
        return lambda: f.fp8q_per_token_group_quant(x, q, s, 128, E4M3FN)
    run("per_token_group_quant", per_token_set, c2_bytes, c2_bytes, m * n)

    M, N = wl.c3_w.shape
    c3_bytes = M * N * 3 + wl.c3_s.numel() * 4

    def dequant_set(i):
        w = wl.c3_w if i == 0 else wl.c3_w.clone()
        y = torch.empty((M, N), dtype=torch.bfloat16, device=d)
        return lambda: f.fp8q_block_dequant(w, wl.c3_s, y, 128, E4M3FN)
    run("block_dequant", dequant_set, c3_bytes, c3_bytes, M * N)

    def round_trip_set(i):
        q = wl.c2_q if i == 0 else wl.c2_q.clone()
        s = wl.c2_s if i == 0 else wl.c2_s.clone()
        y = torch.empty((m, n), dtype=torch.bfloat16, device=d)
        return lambda: f.fp8q_cast_from_fp8(q, s, y, GRAN_GROUP, 128, E4M3FN)
    run("cast_from_fp8_group", round_trip_set, c2_bytes, c2_bytes, m * n)

    R, C = wl.c4a_x.shape
    c4a_bytes = R * C * 3 + R * 4

    def per_channel_set(i):
        x = wl.c4a_x if i == 0 else wl.c4a_x.clone()
        q = torch.empty((R, C), dtype=torch.uint8, device=d)
        s = torch.empty((R,), dtype=torch.float32, device=d)
        return lambda: f.fp8q_cast_per_channel(x, q, s, E4M3FN)
    run("cast_per_channel", per_channel_set, c4a_bytes, c4a_bytes, R * C)

    n4 = wl.c4b_x.numel()
    c4b_bytes = 2 * n4 * 4 + n4 + 4

    def per_tensor_set(i):
        x = wl.c4b_x if i == 0 else wl.c4b_x.clone()
        q = torch.empty((n4,), dtype=torch.uint8, device=d)
        s = torch.empty((1,), dtype=torch.float32, device=d)
        return lambda: f.fp8q_cast_per_tensor(x, q, s, wl.ws, E5M2)
    run("cast_per_tensor_f32_e5m2", per_tensor_set, n4 * 5 + 4, c4b_bytes, n4)
    return out


def _raiser(msg: str):
    """A stand-in for a library call that is unavailable here: raises with the reason."""
    def fn():
        raise RuntimeError(msg)
    return fn


class MatmulWorkload:
    """The two fp8 products on the tensor cores: c2's activations x[4096, 7168]
    quantised per token by the library (codes and 1 x 128 scales, made once,
    before timing) times the e4m3fn weight W[18432, 7168] with 128 x 128 block
    scales; bf16 out [4096, 18432].  Per-tensor: the same codes with one scale
    each (ColossalAI linear_fp8's torch._scaled_mm)."""

    def __init__(self, wl: Workload):
        f, d = wl.fp8q, wl.device
        m, k = wl.c2_x.shape
        self.q = torch.empty((m, k), dtype=torch.uint8, device=d)
        self.sa = torch.empty((m, k // 128), dtype=torch.float32, device=d)
        f.fp8q_per_token_group_quant(wl.c2_x, self.q, self.sa, 128, E4M3FN)
        w, sb = workloads.mm_w_s()
        self.w, self.sb = _to_dev(w, d), _to_dev(sb, d)
        self.n = self.w.shape[0]
        self.out = torch.empty((m, self.n), dtype=torch.bfloat16, device=d)
        self.s1 = self.sa[:1, :1].reshape(1).clone()
        self.s2 = self.sb[:1, :1].reshape(1).clone()
        self.status = torch.zeros(1, dtype=torch.int32, device=d)
        self.flops = 2.0 * m * self.n * k
        self.shape = (m, self.n, k)
        self.fp8q = f
        self.ops = {
            "scaled_mm_blockwise": lambda: f.fp8q_scaled_mm_blockwise(self.q, self.sa, self.w, self.sb, self.out,
                                                                      status=self.status),
            "scaled_mm_per_tensor": lambda: f.fp8q_scaled_mm(self.q, self.w, self.s1, self.s2, self.out,
                                                             status=self.status),
        }

    @staticmethod
    def _timed(fn, steps: int, warmup: int, device, min_ms: float = 20.0, rest_s: float = 0.0):
        """ms per call of fn (CUDA events around at least `steps` back-to-back calls, and enough
        calls to span `min_ms`, after `warmup`), with the SM clocks sampled while it runs.
        rest_s: an idle pause first, so that products timed one after another each start from
        the same power state (a dense product drives the board to its power cap within tens of
        milliseconds, and the clocks it leaves lowered would otherwise fall on the next entry)."""
        if rest_s > 0:
            torch.cuda.synchronize(device)
            time.sleep(rest_s)
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize(device)
        steps = max(steps, int(min_ms / max(e0.elapsed_time(e1), 1e-3)) + 1)
        with ClockSampler(device.index or 0) as clk:
            e0.record()
            for _ in range(steps):
                fn()
            e1.record()
            torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / steps, clk.summary()

    @staticmethod
    def _timed_graph(fn, per_graph: int, replays: int, device):
        """ms per call of fn replayed from a CUDA graph of `per_graph` back-to-back calls (the same
        kernels and arguments, without the host's launch path between them): the median over
        `replays` replays, with the SM clocks sampled while they run."""
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(side):
            for _ in range(per_graph):
                fn()
        torch.cuda.current_stream(device).wait_stream(side)
        torch.cuda.synchronize(device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            for _ in range(per_graph):
                fn()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize(device)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
        with ClockSampler(device.index or 0) as clk:
            for a, e in evs:
                a.record()
                graph.replay()
                e.record()
            torch.cuda.synchronize(device)
        del graph
        return statistics.median(a.elapsed_time(e) / per_graph for a, e in evs), clk.summary()

    def time(self, steps: int, warmup: int, device):
        """Every entry of the section, memory-bound ones first (a long run of tensor-core work
        leaves the SM clocks lowered by the power cap for a while)."""
        res = self.time_decode(steps, warmup, device)
        res.update(self.time_products(steps, warmup, device))
        res.update(self.time_linear(steps, warmup, device))
        res["sustained 2 s"] = self.time_sustained(device)
        if int(self.status.item()) != 0:
            raise RuntimeError("a bounded wait of the fp8 product ran out")
        return res

    def library_ops(self):
        """Library products on the same operands, for context: torch._scaled_mm (cuBLASLt) with
        per-tensor scales; for the fine-grained scales, torch's blockwise scaled_mm (1 x 128 and
        128 x 128, which this torch build serves on sm_90 only) and vLLM's CUTLASS blockwise
        product (cutlass_scaled_mm: activation scales M-major, the weight and its block scales
        passed transposed, as vLLM's own block-fp8 linear passes them)."""
        a8 = self.q.view(torch.float8_e4m3fn)
        b8 = self.w.view(torch.float8_e4m3fn)
        ops = {"torch_scaled_mm (cuBLASLt)": lambda: torch._scaled_mm(a8, b8.t(), scale_a=self.s1, scale_b=self.s2,
                                                                      out_dtype=torch.bfloat16)}

        def torch_blockwise():
            import torch.nn.functional as F
            st = F.ScalingType
            return F.scaled_mm(a8, b8.t(), self.sa, st.BlockWise1x128, self.sb, st.BlockWise128x128,
                               output_dtype=torch.bfloat16)
        ops["torch scaled_mm blockwise (1x128, 128x128)"] = torch_blockwise
        try:
            import vllm._custom_ops as vops
            sa_mn = self.sa.t().contiguous().t()
            sb_t = self.sb.t()
            out = torch.empty_like(self.out)
            ops["vllm cutlass_scaled_mm blockwise (CUTLASS sm100)"] = (
                lambda: torch.ops._C.cutlass_scaled_mm(out, a8, b8.t(), sa_mn, sb_t, None) or out)
            major, minor = torch.cuda.get_device_capability()
            if not vops.cutlass_scaled_mm_supports_block_fp8(major * 10 + minor):
                raise RuntimeError("vLLM reports no block-fp8 CUTLASS product for this device")
        except Exception as ex:     # vLLM or its compiled ops missing on this machine
            msg = str(ex).splitlines()[0][:200] if str(ex) else type(ex).__name__
            ops["vllm cutlass_scaled_mm blockwise (CUTLASS sm100)"] = _raiser(msg)
        return ops

    def time_products(self, steps: int, warmup: int, device):
        """The two products on the full workload, and the library products (library_ops) on the
        same operands for context; each library output is compared with libfp8q's once."""
        ops = dict(self.ops)
        lib_ops = self.library_ops()
        ops.update(lib_ops)
        ref = {}
        for name, fn in self.ops.items():
            fn()
            ref[name] = self.out.float().clone()
        res = {}
        for name, fn in ops.items():
            try:
                ms, clk = self._timed(fn, steps, warmup, device, rest_s=1.0)
                res[name] = {"ms": round(ms, 4), "tflops": round(self.flops / (ms * 1e-3) / 1e12, 1), "clocks": clk,
                             "rest_before_s": 1.0}
                if name in lib_ops:
                    y = fn().float()
                    r = ref["scaled_mm_blockwise" if "blockwise" in name else "scaled_mm_per_tensor"]
                    res[name]["max_abs_diff_over_max_abs_vs_libfp8q"] = float((y - r).abs().max() / r.abs().max())
            except Exception as ex:      # the library baseline may be missing on some builds
                res[name] = {"unavailable": str(ex).splitlines()[0][:200] if str(ex) else type(ex).__name__}
        del ref
        return res

    def time_sustained(self, device, seconds: float = 2.0):
        """Each product back to back for `seconds` (CUDA events around the run, NVML clocks and
        power sampled during it): under the board's 1000 W cap a dense product settles at lowered
        SM clocks after the first tens of milliseconds, which the short timings above precede."""
        ops = dict(self.ops)
        lib = self.library_ops()
        for k in ("torch_scaled_mm (cuBLASLt)", "vllm cutlass_scaled_mm blockwise (CUTLASS sm100)"):
            ops[k] = lib[k]
        res = {}
        for name, fn in ops.items():
            try:
                fn()
                torch.cuda.synchronize(device)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                n = 0
                with ClockSampler(device.index or 0, period_s=0.02, power=True) as clk:
                    t0 = time.perf_counter()
                    e0.record()
                    while time.perf_counter() - t0 < seconds:
                        for _ in range(10):
                            fn()
                        n += 10
                        torch.cuda.synchronize(device)
                    e1.record()
                    torch.cuda.synchronize(device)
                ms = e0.elapsed_time(e1) / n
                res[name] = {"ms": round(ms, 4), "tflops": round(self.flops / (ms * 1e-3) / 1e12, 1), "launches": n,
                             "clocks": clk.summary()}
            except Exception as ex:
                res[name] = {"unavailable": str(ex).splitlines()[0][:200] if str(ex) else type(ex).__name__}
        return res

    def time_decode(self, steps: int, warmup: int, device):
        """The two products at decode-sized activations (M = 1 and 64 rows of the same per-token
        codes) against the same weight: weight streaming, so GB/s of N*K + M*K + 2*M*N bytes;
        and the weight transpose of the backward (GB/s of its 2 bytes per element)."""
        f = self.fp8q
        res = {}
        for m in (1, 64):
            q, sa = self.q[:m], self.sa[:m]
            out = torch.empty((m, self.n), dtype=torch.bfloat16, device=device)
            nbytes = self.w.numel() + q.numel() + 2 * out.numel()
            for name, fn in [(f"scaled_mm_blockwise M={m}",
                              lambda: f.fp8q_scaled_mm_blockwise(q, sa, self.w, self.sb, out, status=self.status)),
                             (f"scaled_mm_per_tensor M={m}",
                              lambda: f.fp8q_scaled_mm(q, self.w, self.s1, self.s2, out, status=self.status))]:
                # launched one by one from Python, then the same calls replayed from a CUDA
                # graph (a ~25 us product is close enough to the launch path's cost for it to show)
                ms_stream, _ = self._timed(fn, steps, warmup, device)
                ms, clk = self._timed_graph(fn, 40, 10, device)
                res[name] = {"ms": round(ms, 4), "gb_s": round(nbytes / (ms * 1e-3) / 1e9, 1), "clocks": clk,
                             "timing": "cuda_graph_replay", "ms_stream": round(ms_stream, 4),
                             "gb_s_stream": round(nbytes / (ms_stream * 1e-3) / 1e9, 1)}
        k = self.q.shape[1]
        wt = torch.empty((k, self.n), dtype=torch.uint8, device=device)
        ms, clk = self._timed(lambda: f.fp8q_transpose_fp8(self.w, wt, self.n), steps, warmup, device)
        res["transpose_fp8 (weight)"] = {"ms": round(ms, 4), "gb_s": round(2.0 * self.w.numel() / (ms * 1e-3) / 1e9, 1),
                                         "clocks": clk}
        return res

    def time_linear(self, steps: int, warmup: int, device):
        """ColossalAI linear_fp8 forward + backward on bf16 x[4096, 7168], w[18432, 7168] and a bias
        (three fp8 products of 2*M*N*K each, the three per-tensor casts and the bias gradient).
        The gradients are cleared before each backward, as a training step's zero_grad does, so
        no accumulation into .grad runs in the timed region."""
        f = self.fp8q
        g = torch.Generator(device=device).manual_seed(20261207)
        m, k = self.q.shape
        x = torch.randn((m, k), generator=g, device=device).to(torch.bfloat16).requires_grad_(True)
        w = (torch.randn((self.n, k), generator=g, device=device) * 0.02).to(torch.bfloat16).requires_grad_(True)
        b = torch.randn((self.n,), generator=g, device=device).to(torch.bfloat16).requires_grad_(True)
        go = (torch.randn((m, self.n), generator=g, device=device) * 1e-3).to(torch.bfloat16)

        def step():
            x.grad = w.grad = b.grad = None
            y = f.linear_fp8(x, w, b)
            y.backward(go)
        ms, clk = self._timed(step, steps, warmup, device)
        return {"linear_fp8 forward+backward": {"ms": round(ms, 4), "tflops": round(3 * self.flops / (ms * 1e-3) / 1e12, 1),
                                                "clocks": clk}}


def fp8_tensor_peak(sustained: bool = False):
    """Dense fp8 tensor-core peak: the measured cuBLAS bf16 figure (burst, or the seconds-long
    loop under the power cap) times the nominal fp8 : bf16 ratio of 2."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    kind = "sustained" if sustained else "burst"
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if key in d:
            return 2.0 * float(d[key]), f"2 x measured bf16 {kind} (nominal fp8:bf16 ratio)"
    return 2.0 * (1400.0 if sustained else 1590.0), f"2 x fallback bf16 {kind} (nominal fp8:bf16 ratio)"


def _to_dev(a, device, dt=None):
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    if dt is not None:
        t = t.view(dt)
    return t.to(device)


def make_host_inputs():
    c3_w, c3_s = workloads.c3_w_s()
    return {
        "c2_x": workloads.c2_x(),
        "c3_w": c3_w, "c3_s": c3_s,
        "c4a_x": workloads.c4a_x(),
        "c4b_v": workloads.c4b_v(),
        "c4c_v": workloads.c4c_v(),
        "c5": [workloads.c5_weight(i) for i in range(len(workloads.C5_SHAPES))],
    }


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int, period_s: float = 0.005, power: bool = False):
        self.index, self.period, self.power = index, period_s, power
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        self.watts = []
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        if self.power:
            self.watts.append(nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for k, bit in self.REASONS.items():
            if r & bit:
                self.reasons.add(k)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()
            if not self.samples:
                try:
                    self._sample()
                except Exception:
                    pass

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        d = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
             "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}
        if self.power and self.watts:
            d["power_w_median"] = round(statistics.median(self.watts), 1)
        return d


# ---------------------------------------------------------------------------
# roofline helpers
# ---------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# kernel sources each op's device code depends on (the launch wrappers are host code)
OP_SOURCES = {
    "per_token_group_quant": ["quant_per_token.cu", "fp8q_device.cuh"],
    "block_dequant": ["dequant.cu", "fp8q_device.cuh"],
    "cast_from_fp8_group": ["dequant.cu", "fp8q_device.cuh"],
    "block_dequant_grouped": ["dequant.cu", "fp8q_device.cuh"],
    "cast_per_channel": ["quant_scaled.cu", "fp8q_device.cuh"],
    "cast_per_tensor_f32_e5m2": ["quant_scaled.cu", "fp8q_device.cuh"],
    "cast_per_tensor_f16_zero": ["quant_scaled.cu", "fp8q_device.cuh"],
}


def source_fingerprint(files) -> str:
    """Hash of the kernel sources' code: comments and whitespace are removed first, so an edit
    to a comment keeps a capture's record valid and any change to the code voids it."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dequantisation_fp8q_token_b200", "csrc")
    for fn in sorted(files):
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            code = f.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        code = re.sub(r"\s+", " ", code).strip()
        h.update(fn.encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


def recorded_traffic(op_name: str):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on
    the kernel sources the op runs now (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get("ops", {}).get(op_name)
    if e is None or e.get("source_fingerprint") != source_fingerprint(OP_SOURCES[op_name]):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline; never on the product path)
# ---------------------------------------------------------------------------
def oracle_sample_pass(orc, h, frac: float, threads: int):
    """Run every op of the step on the oracle over a `frac` sample of its rows /
    elements; returns the algorithmic bytes of the sample."""
    nbytes = 0
    m, n = workloads.C2_SHAPE
    r = max(1, int(m * frac))
    q, s = orc.per_token_group_quant(h["c2_x"][:r], orc.BF16, 128, orc.E4M3FN, threads=threads)
    nbytes += r * n * 3 + r * (n // 128) * 4
    orc.cast_from_fp8(q, s, orc.GRAN_GROUP, orc.E4M3FN, 128, orc.BF16, threads=threads)
    nbytes += r * n * 3 + r * (n // 128) * 4
    M, N = workloads.C3_SHAPE
    r = max(1, int(M * frac))
    orc.block_dequant(h["c3_w"], h["c3_s"], orc.E4M3FN, 128, orc.BF16, rows=(0, r), threads=threads)
    nbytes += r * N * 3
    R, C = workloads.C4A_SHAPE
    r = max(1, int(R * frac))
    orc.cast_per_channel(h["c4a_x"][:r], orc.BF16, orc.E4M3FN, threads=threads)
    nbytes += r * C * 3 + r * 4
    k = max(1, int(workloads.C4B_NUMEL * frac))
    orc.cast_per_tensor(h["c4b_v"][:k], orc.F32, orc.E5M2, threads=threads)
    nbytes += k * 9
    k = max(1, int(workloads.C4C_NUMEL * frac))
    orc.cast_per_tensor(h["c4c_v"][:k], orc.F16, orc.E4M3FN, threads=threads)
    nbytes += k * 5
    for w, sc in h["c5"]:
        M, N = w.shape
        r = max(1, int(M * frac))
        orc.block_dequant(w, sc, orc.E4M3FN, 128, orc.BF16, rows=(0, r), threads=threads)
        nbytes += r * N * 3
    return nbytes


def cpu_baseline(h, budget_s: float = 15.0):
    import oracle as orc
    orc.build()
    threads = os.cpu_count() or 1
    frac = 1.0 / 4096
    # grow the sample until one pass takes about `budget_s` (small samples are
    # dominated by thread start-up, so grow by at most 8x per probe)
    while True:
        t0 = time.perf_counter()
        b = oracle_sample_pass(orc, h, frac, threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 2 or frac >= 1.0:
            break
        frac = min(1.0, frac * min(8.0, max(1.5, budget_s / max(dt, 1e-3))))
    reps = 1
    if dt < budget_s / 2:
        # the whole step is faster than the budget: time several full passes
        reps = max(1, int(budget_s / max(dt, 1e-3)))
        t0 = time.perf_counter()
        b = sum(oracle_sample_pass(orc, h, frac, threads) for _ in range(reps))
        dt = time.perf_counter() - t0
    what = (f"{reps} passes over the whole step" if reps > 1 else
            f"the first {frac:.5f} of the rows / elements of every op of the step")
    # one thread, on a sample grown until one pass takes an eighth of the budget or more
    f1 = 1.0 / 4096
    while True:
        t0 = time.perf_counter()
        b1 = oracle_sample_pass(orc, h, f1, 1)
        d1 = time.perf_counter() - t0
        if d1 >= budget_s / 8 or f1 >= 1.0:
            break
        f1 = min(1.0, f1 * min(8.0, max(1.5, (budget_s / 4) / max(d1, 1e-3))))
    return {"value": round(b / dt / 1e9, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{what} ({b / 1e6:.1f} MB algorithmic), plain C oracle on {threads} threads",
            "seconds": round(dt, 2), "cpu_model": cpu_model(),
            "one_thread": {"value": round(b1 / d1 / 1e9, 4), "unit": UNIT, "seconds": round(d1, 2),
                           "sample": f"the first {f1:.5f} of every op of the step ({b1 / 1e6:.1f} MB algorithmic)"}}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def dist_setup(ngpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dominant_sample_steps(steps: int, samples: int = 5):
    """The timed steps that carry the dominant op's event pair: the last step of each of about
    `samples` equal groups, never step 0 unless it is the only one."""
    every = max(1, steps // samples)
    return list(range(max(every - 1, 1) if steps > 1 else 0, steps, every))


def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import dequantisation_fp8q_token_b200 as fp8q
    fp8q.lib()
    h = make_host_inputs()
    wl = Workload(device, fp8q, h)
    torch.cuda.synchronize()

    # NVML is set up before the warm-up: its initialisation takes milliseconds, and a GPU left
    # idle that long just before the timed steps ran the first of them measurably slower
    clk = ClockSampler(local)
    nops = len(wl.ops)
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()
    # The per-op split comes from an instrumented pass before the timed steps:
    # an event recorded between two kernels keeps the second from starting
    # before the first has ended (no programmatic dependent launch across
    # it), so the timed steps carry events around the dominant op alone.
    split_steps = max(3, min(args.steps, 20))
    events = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nops)]
              for _ in range(split_steps)]
    for k in range(split_steps):
        wl.step(events[k])
    torch.cuda.synchronize()
    per_op_samples = [sorted(events[k][i][0].elapsed_time(events[k][i][1]) for k in range(split_steps))
                      for i in range(nops)]
    per_op_ms = [statistics.median(v) for v in per_op_samples]
    dom = max(range(nops), key=lambda i: per_op_ms[i])
    # the dominant op's event pair rides on every `every`-th timed step only (about 5
    # samples): the pair keeps the op from overlapping its neighbours under programmatic
    # dependent launch, which cost the step about 1.5% with a pair on every step on B200
    # (20 timed steps: 6439 against 6630 GB/s with 200).  The samples end each group of
    # `every` steps, so none falls on the first timed step, which starts on an idle GPU
    # (its dominant op measured up to a quarter slower there).
    dom_events = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for k in dominant_sample_steps(args.steps)}

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with clk:
        t_start.record()
        for k in range(args.steps):
            if k in dom_events:
                wl.step(dom_events[k], only=dom)
            else:
                wl.step()
        t_end.record()
        torch.cuda.synchronize()
    barrier(world)
    ms_local = t_start.elapsed_time(t_end)
    ms_total = max_over_ranks(ms_local, world, device)
    ms_step = ms_total / args.steps
    dom_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in dom_events.values())

    # end to end: pinned host inputs -> device, the step, outputs -> pinned host
    e2e = EndToEnd(wl)
    e2e_steps = max(1, min(args.steps, 5))
    barrier(world)
    e2e_ms = max_over_ranks(e2e.time(e2e_steps), world, device)
    bi, bo = e2e.h2d_bytes, e2e.d2h_bytes
    del e2e
    sharded = None
    if world > 1 or args.sharded:
        leg = ShardedLeg(device, rank, world, h["c4b_v"], kernels=LegKernels(fp8q),
                         ws_bytes=fp8q.fp8q_cast_per_tensor_workspace_bytes())
        sharded = leg.run()
        del leg
        torch.cuda.empty_cache()
    pcie = pcie_bound(bi, bo, device) if rank == 0 else None
    iso = isolated_timing(wl) if rank == 0 else {}
    mm = None
    if rank == 0 and not args.no_matmul:
        mmw = MatmulWorkload(wl)
        mm_res = mmw.time(max(5, min(args.steps, 50)), max(3, args.warmup), device)
        tpeak, tkind = fp8_tensor_peak()
        tpeak_s, tkind_s = fp8_tensor_peak(sustained=True)
        hpeak, _ = measured_peaks()
        for name, v in mm_res.items():
            if name.startswith("sustained"):
                for e in v.values():
                    if "tflops" in e:
                        e["frac_of_sustained_peak"] = round(e["tflops"] / tpeak_s, 4)
                continue
            if "tflops" in v:
                v["frac"] = round(v["tflops"] / tpeak, 4)
            if "gb_s" in v:
                v["frac"] = round(v["gb_s"] / hpeak, 4)
        mm = {"workload": "fp8 products: per-token e4m3fn codes of c2 x[4096,7168] (1x128 scales) times "
                          "e4m3fn W[18432,7168] (128x128 block scales), bf16 out; per-tensor: same codes, "
                          "one scale each",
              "shape_mnk": list(mmw.shape), "flops_per_launch": mmw.flops, "bound": "tensor",
              "peak_tflops": round(tpeak, 1), "peak_kind": tkind,
              "sustained_peak_tflops": round(tpeak_s, 1), "sustained_peak_kind": tkind_s,
              "l2": "operands 161 MB > 126 MB L2; compute-bound, no flush", "ops": mm_res}
        del mmw

    if rank != 0:
        _finish(world)
        return
    peak, peak_kind = measured_peaks()
    kernels = {}
    pct = _quantile
    for op, ms, v in zip(wl.ops, per_op_ms, per_op_samples):
        gbs = op.bytes / (ms * 1e-3) / 1e9
        kernels[op.name] = {"us": round(ms * 1e3, 2), "us_mean": round(statistics.mean(v) * 1e3, 2),
                            "bytes": op.bytes, "gb_s": round(gbs, 1),
                            "frac": round(gbs / peak, 4), "launches": op.launches, "elements": op.elems,
                            "gelem_s": round(op.elems / (ms * 1e-3) / 1e9, 2),
                            "us_p10_p50_p90": [round(pct(v, q) * 1e3, 2) for q in (0.1, 0.5, 0.9)]}
    dop = wl.ops[dom]
    dgbs = dop.bytes / (dom_ms * 1e-3) / 1e9      # CUDA events around it in sampled timed steps
    value = world * wl.step_bytes / (ms_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp32 -> fp8 (u8)",
        "data": "synthetic (seeded generators; shapes and value mixes of the pages' workloads)",
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "pct_of_nominal_8tbs": round(100.0 * value / world / 8000.0, 2),
        "config": {"workload": WORKLOAD, "step_bytes": wl.step_bytes, "parallelism": f"replicas x{world}",
                   "l2": "no flush: each step streams ~4.4 GB through the 126 MB L2, so every op's inputs are cold"},
        "roofline": {"bound": "hbm", "kernel": dop.kernel, "op": dop.name, "achieved": round(dgbs, 1),
                     "timed_launches": len(dom_events),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dgbs / peak, 4),
                     "bytes_per_launch": dop.bytes, "traffic": recorded_traffic(dop.name)},
        "kernels": kernels,
        "kernels_from": f"{split_steps} instrumented steps before the timed ones (events around every op)",
        "isolated": {k: {**v, "frac": round(v["gb_s"] / peak, 4),
                         "pct_of_nominal_8tbs": round(100.0 * v["gb_s"] / 8000.0, 2)} for k, v in iso.items()},
        "matmul": mm,
        "clocks": clk.summary(),
        "e2e": {"value": round(world * wl.step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                "steps": e2e_steps, "pcie": pcie,
                "frac_of_pcie_bound": round(pcie["bound_ms_per_step"] / e2e_ms, 4) if pcie else None},
        "gpu_launches": wl.launches_per_step * args.steps,
    }
    if sharded is not None:
        line["sharded"] = sharded
    # the two ops the metric names, each timed alone (isolated) and inside the step (marginal
    # cost is printed by --marginal; `kernels` holds the instrumented split)
    line["headline_ops"] = {k: {"us": iso[k]["us"], "gb_s": iso[k]["gb_s"], "gelem_s": iso[k]["gelem_s"],
                                "frac": round(iso[k]["gb_s"] / peak, 4),
                                "pct_of_nominal_8tbs": round(100.0 * iso[k]["gb_s"] / 8000.0, 2),
                                "us_p10_p50_p90": iso[k]["us_p10_p50_p90"], "timing": iso[k]["timing"],
                                "us_stream": iso[k]["us_stream"],
                                "frac_stream": round(iso[k]["gb_s_stream"] / peak, 4),
                                "host_us_per_call": iso[k]["host_us_per_call"]}
                            for k in ("per_token_group_quant", "block_dequant") if k in iso}
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(h)
    print(json.dumps(line), flush=True)
    _finish(world)


def run_marginal(args):
    """Each op's marginal cost inside the live step, measured by adding work, never by skipping
    it: the step with one more instance of op i appended at its end (after the 3 GB grouped
    dequant, so the extra instance's inputs are cold and the op before it leaves dirty L2
    lines, as in the step), minus the plain step.  Rounds alternate the plain step and each
    extended step; the medians over rounds are reported.  Prints one JSON line."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    import dequantisation_fp8q_token_b200 as fp8q
    fp8q.lib()
    wl = Workload(device, fp8q, make_host_inputs())
    steps, rounds = max(5, args.steps // 10), 5

    def timed(extra):
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            wl.step()
            if extra is not None:
                extra.fn()
        e1.record()
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / steps

    for _ in range(max(3, args.warmup)):
        wl.step()
    base, extra = [], {op.name: [] for op in wl.ops}
    with ClockSampler(0) as clk:
        for _ in range(rounds):
            base.append(timed(None))
            for op in wl.ops:
                extra[op.name].append(timed(op))
    peak, peak_kind = measured_peaks()
    b = statistics.median(base)
    res = {}
    for op in wl.ops:
        us = (statistics.median(extra[op.name]) - b) * 1e3
        res[op.name] = {"marginal_us": round(us, 2), "bytes": op.bytes,
                        "gb_s": round(op.bytes / (us * 1e-6) / 1e9, 1) if us > 0 else None,
                        "frac": round(op.bytes / (us * 1e-6) / 1e9 / peak, 4) if us > 0 else None}
    print(json.dumps({"marginal": res, "step_us_median": round(b * 1e3, 2), "steps_per_timing": steps,
                      "rounds": rounds, "peak_gb_s": peak, "peak_kind": peak_kind, "clocks": clk.summary(),
                      "sum_of_marginals_us": round(sum(v["marginal_us"] for v in res.values()), 2)}), flush=True)


def _finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The reference arm: the CPU oracle, timed as it stands on this host."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as orc
    orc.build()
    threads = os.cpu_count() or 1
    h = make_host_inputs()
    # size each step's sample so that warm-up plus timed steps take about a minute
    per_step_s = 60.0 / (args.steps + args.warmup)
    frac = 1.0 / 4096
    while True:
        t0 = time.perf_counter()
        oracle_sample_pass(orc, h, frac, threads)
        dt = time.perf_counter() - t0
        if dt >= per_step_s / 2 or frac >= 1.0:
            break
        frac = min(1.0, frac * min(8.0, max(1.5, per_step_s / max(dt, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample_pass(orc, h, frac, threads)
    t0 = time.perf_counter()
    b = 0
    for _ in range(args.steps):
        b += oracle_sample_pass(orc, h, frac, threads)
    dt = time.perf_counter() - t0
    value = b / dt / 1e9
    sample = (f"each step: the first {frac:.5f} of the rows / elements of every op of the GPU step "
              f"({b / args.steps / 1e6:.1f} MB algorithmic), plain C oracle on {threads} threads")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp32 -> fp8 (u8)",
            "data": "synthetic", "config": {"workload": WORKLOAD, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "kind": "oracle", "cores": threads,
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# single-op cases for profiler captures (ncu -k <kernel> -c <n>): one op, a few
# launches, inputs larger than L2 and a few GB on the device at most
# ---------------------------------------------------------------------------
def _profile_case(name, fp8q, device):
    """Returns (one call of the op, its algorithmic bytes)."""
    g = np.random.default_rng(20261299)
    bf16 = torch.bfloat16
    if name in ("per_token_4x", "cast_from_fp8_4x"):
        m, n = 4 * workloads.C2_SHAPE[0], workloads.C2_SHAPE[1]   # bf16 [16384, 7168]: 235 MB
        x = _to_dev(workloads.to_bf16_bits(g.standard_normal((m, n), dtype=np.float32)), device, bf16)
        q = torch.empty((m, n), dtype=torch.uint8, device=device)
        s = torch.empty((m, n // 128), dtype=torch.float32, device=device)
        y = torch.empty((m, n), dtype=bf16, device=device)
        fp8q.fp8q_per_token_group_quant(x, q, s, 128, E4M3FN)
        nbytes = m * n * 3 + m * (n // 128) * 4
        if name == "per_token_4x":
            return (lambda: fp8q.fp8q_per_token_group_quant(x, q, s, 128, E4M3FN)), nbytes
        return (lambda: fp8q.fp8q_cast_from_fp8(q, s, y, GRAN_GROUP, 128, E4M3FN)), nbytes
    if name == "block_dequant":
        w, sc = workloads.c3_w_s()
        w, sc = _to_dev(w, device), _to_dev(sc, device)
        y = torch.empty(w.shape, dtype=bf16, device=device)
        return (lambda: fp8q.fp8q_block_dequant(w, sc, y, 128, E4M3FN)), w.numel() * 3 + sc.numel() * 4
    if name in ("grouped_16", "grouped_72"):
        # 8 big + 8 ragged experts (174 MB in), or all 72 of the bench step (1 GB in, 2 GB out)
        idx = list(range(8)) + list(range(64, 72)) if name == "grouped_16" else list(range(72))
        ws, ss = zip(*[workloads.c5_weight(i) for i in idx])
        ws = [_to_dev(w, device) for w in ws]
        ss = [_to_dev(s_, device) for s_ in ss]
        ys = [torch.empty(w.shape, dtype=bf16, device=device) for w in ws]
        nbytes = sum(w.numel() * 3 for w in ws) + sum(s_.numel() * 4 for s_ in ss)
        return (lambda: fp8q.fp8q_block_dequant_grouped(ws, ss, ys, 128, E4M3FN)), nbytes
    if name == "per_channel":
        x = _to_dev(workloads.c4a_x(), device, bf16)
        q = torch.empty(x.shape, dtype=torch.uint8, device=device)
        s = torch.empty((x.shape[0],), dtype=torch.float32, device=device)
        return (lambda: fp8q.fp8q_cast_per_channel(x, q, s, E4M3FN)), x.numel() * 3 + x.shape[0] * 4
    if name == "per_tensor":
        x = _to_dev(workloads.c4b_v(), device)
        q = torch.empty(x.shape, dtype=torch.uint8, device=device)
        s = torch.empty((1,), dtype=torch.float32, device=device)
        ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device=device)
        return (lambda: fp8q.fp8q_cast_per_tensor(x, q, s, ws, E5M2)), x.numel() * 9 + 4
    if name in ("scaled_mm", "scaled_mm_blockwise", "scaled_mm_blockwise_m1", "transpose_weight"):
        m, k = workloads.C2_SHAPE
        x = _to_dev(workloads.c2_x(), device, bf16)
        q = torch.empty((m, k), dtype=torch.uint8, device=device)
        sa = torch.empty((m, k // 128), dtype=torch.float32, device=device)
        fp8q.fp8q_per_token_group_quant(x, q, sa, 128, E4M3FN)
        w, sb = workloads.mm_w_s()
        w, sb = _to_dev(w, device), _to_dev(sb, device)
        out = torch.empty((m, w.shape[0]), dtype=bf16, device=device)
        s1 = torch.ones(1, dtype=torch.float32, device=device)
        flops = 2.0 * m * w.shape[0] * k
        if name == "scaled_mm":
            return (lambda: fp8q.fp8q_scaled_mm(q, w, s1, s1, out)), flops
        if name == "scaled_mm_blockwise_m1":
            # one token: weight streaming, bytes moved (N*K + K + 2*N)
            o1 = out[:1]
            return (lambda: fp8q.fp8q_scaled_mm_blockwise(q[:1], sa[:1], w, sb, o1)), w.numel() + k + 2 * w.shape[0]
        if name == "transpose_weight":
            wt = torch.empty((k, w.shape[0]), dtype=torch.uint8, device=device)
            return (lambda: fp8q.fp8q_transpose_fp8(w, wt, w.shape[0])), 2 * w.numel()
        return (lambda: fp8q.fp8q_scaled_mm_blockwise(q, sa, w, sb, out)), flops
    if name == "sum_rows":
        # the bias gradient of linear_fp8's backward: column sums of bf16 g[4096, 18432] (151 MB)
        m, n = workloads.C2_SHAPE[0], workloads.MM_W_SHAPE[0]
        x = _to_dev(workloads.to_bf16_bits(g.standard_normal((m, n), dtype=np.float32)), device, bf16)
        out = torch.empty((n,), dtype=bf16, device=device)
        return (lambda: fp8q.fp8q_sum_rows(x, out)), x.numel() * 2 + n * 2
    if name in ("records_pack", "records_unpack"):
        # the fp8 all-gather's device work for 8 ranks of 16 Mi bf16 each
        # (32 MiB per rank): pack = each rank's per-tensor cast into its
        # record (amax pass + cast pass); unpack = all 8 records dequantised
        W, n = 8, 1 << 24
        R = fp8q.record_bytes(n)
        xs = [_to_dev(workloads.to_bf16_bits(g.standard_normal(n, dtype=np.float32)), device, bf16)
              for _ in range(W)]
        rec = torch.empty((W * R,), dtype=torch.uint8, device=device)
        y = torch.empty((W * n,), dtype=bf16, device=device)
        ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device=device)

        def pack():
            for r in range(W):
                fp8q.fp8q_pack_record(xs[r], rec[r * R:(r + 1) * R], ws, E5M2)
        pack()
        if name == "records_pack":
            return pack, W * (n * 2 * 2 + R)
        return (lambda: fp8q.fp8q_unpack_records(rec, W, n, y, E5M2)), W * (R + n * 2)
    raise SystemExit(f"unknown profile case {name}")


PROFILE_CASES = ["per_token_4x", "cast_from_fp8_4x", "block_dequant", "grouped_16", "grouped_72", "per_channel",
                 "per_tensor", "records_pack", "records_unpack", "scaled_mm", "scaled_mm_blockwise",
                 "scaled_mm_blockwise_m1", "transpose_weight", "sum_rows"]


def run_profile_case(name, iters):
    """Run one op `iters` times after one untimed launch and report the mean
    time per launch (CUDA events, back to back); prints no bench line."""
    device = torch.device("cuda", 0)
    import dequantisation_fp8q_token_b200 as fp8q
    fn, nbytes = _profile_case(name, fp8q, device)
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / max(iters, 1)
    if name in ("scaled_mm", "scaled_mm_blockwise"):
        print(f"profile case {name}: {iters} calls, {us:.2f} us per call, "
              f"{nbytes / (us * 1e-6) / 1e12 if iters else 0.0:.1f} TFLOP/s")
        return
    print(f"profile case {name}: {iters} calls, {us:.2f} us per call, "
          f"{nbytes / (us * 1e-6) / 1e9 if iters else 0.0:.1f} GB/s algorithmic")


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--profile", choices=PROFILE_CASES,
                    help="run one op of a fixed case --iters times for a profiler capture (no timing)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--no-matmul", action="store_true", help="skip the fp8 products section")
    ap.add_argument("--marginal", action="store_true",
                    help="print each op's marginal cost inside the live step (one JSON line) and exit")
    ap.add_argument("--sharded", action="store_true",
                    help="run the sharded exchange leg at N = 1 too (it always runs when N > 1)")
    args = ap.parse_args(argv)
    if args.profile:
        run_profile_case(args.profile, args.iters)
        return
    if args.marginal:
        run_marginal(args)
        return
    args.warmup = max(3, args.warmup)   # the timing rules want at least 3 untimed steps
    args.steps = max(1, args.steps)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

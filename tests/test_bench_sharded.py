"""bench.py's sharded exchange leg on two gloo ranks, without a GPU.

The leg's device work (the amax pass, the cast pass, the record pack / unpack
of all_gather_fp8) is replaced by host stand-ins that keep the data visible;
everything else runs as under torchrun: the shard ranges, the 4-byte int32
MAX all-reduce of the amax bits (libfp8q's allreduce_amax_bits), the record
exchange (libfp8q's exchange_records, an all_gather_into_tensor of the record
bytes), the bf16 all-gather beside it, the max over ranks of the times and
the byte counts of the result."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


NUMEL, GATHER = 1000, 100


class HostKernels:
    """Host stand-ins for the leg's device calls.  amax: the fp32 magnitude bits of the shard;
    cast: scale_inv := the amax as a float, so equal scale_inv on all ranks shows that the
    exchange delivered the global amax; all-gather: a record whose payload is the high byte of
    each bf16, moved by the library's own exchange, then widened back."""

    def tensor_amax(self, x, amax_bits, ws):
        import torch
        a = x.abs().max() if x.numel() else torch.tensor(0.0)
        amax_bits[0] = a.view(torch.int32)

    def cast_with_amax(self, x, amax_bits, q, scale_inv):
        scale_inv[0] = amax_bits.view(scale_inv.dtype)[0]
        q.zero_()

    def all_gather_fp8(self, out, x, group):
        import torch
        import torch.distributed as dist
        import dequantisation_fp8q_token_b200 as fp8q
        world, rank = dist.get_world_size(group), dist.get_rank(group)
        n = x.numel()
        R = fp8q.record_bytes(n)
        combined = torch.zeros(world * R, dtype=torch.uint8)
        hi = (x.view(torch.int16).to(torch.int32) >> 8).to(torch.uint8)
        combined[rank * R + 16: rank * R + 16 + n] = hi
        fp8q.exchange_records(combined, group)
        for r in range(world):
            b = combined[r * R + 16: r * R + 16 + n].to(torch.int32)
            out[r * n:(r + 1) * n] = (b << 8).to(torch.int16).view(torch.bfloat16)


def _cpu_timer(fn, reps, device):
    import time
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    return (time.perf_counter() - t0) * 1e3 / reps


def _worker(rank, world, port, q):
    import datetime
    import sys

    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        v = np.random.default_rng(7).standard_normal(NUMEL).astype(np.float32)
        v[613] = -40.0                       # the global amax lives on rank 1's shard
        leg = bench.ShardedLeg(torch.device("cpu"), rank, world, v, gather_elems=GATHER,
                               kernels=HostKernels(), timer=_cpu_timer)
        res = leg.run(reps=2, warmup=1)
        leg.gather_fp8()
        q.put((rank, res, leg.shard, leg.sinv.item(), leg.out.view(torch.int16).numpy().copy(),
               leg.g.view(torch.int16).numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_sharded_leg_host_logic_on_two_gloo_ranks():
    import dequantisation_fp8q_token_b200 as fp8q
    import bench
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        rank, res, shard, sinv, out, g = q.get(timeout=180)
        got[rank] = (res, shard, sinv, out, g)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    # the shards tile the tensor, 8-element aligned
    assert got[0][1] == (0, 504) and got[1][1] == (504, NUMEL)
    assert bench.shard_range(NUMEL, 2, 0) == (0, 504)
    # both ranks end with the global amax (|-40|), which only rank 1 held
    assert got[0][2] == got[1][2] == 40.0
    for r in (0, 1):
        res = got[r][0]
        c = res["cast_to_fp8_sharded"]
        assert c["scale_inv_identical_on_all_ranks"] is True
        assert c["elements_total"] == NUMEL and c["allreduce_bytes"] == 4
        assert c["bytes_total"] == 2 * NUMEL * 4 + NUMEL + 4
        a = res["all_gather_fp8"]
        R = fp8q.record_bytes(GATHER)
        assert a["record_bytes"] == R == 16 + 112
        assert a["wire_bytes_received_per_rank"] == R
        assert a["bf16_wire_bytes_received_per_rank"] == 2 * GATHER
        assert "speedup_vs_bf16" in a and res["ranks"] == 2
    # the two ranks report the same (max over ranks) times
    assert got[0][0]["all_gather_fp8"]["us"] == got[1][0]["all_gather_fp8"]["us"]
    # every rank holds every rank's shard in rank order (high byte of each bf16 here)
    for r in (0, 1):
        out = got[r][3].reshape(2, GATHER)
        for j in (0, 1):
            want = (got[j][4].astype(np.int32) >> 8 << 8).astype(np.int16)
            np.testing.assert_array_equal(out[j], want)


def test_shard_range_covers_everything():
    import bench
    for numel in (0, 1, 7, 8, 9, 1000, 67_108_864):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_range(numel, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == numel
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0 and a0 <= a1
            assert all(s0 % 8 == 0 for s0, s1 in spans if s1 > s0)   # an empty shard starts at numel

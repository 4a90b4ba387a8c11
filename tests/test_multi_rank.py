"""The N > 1 bench path on CPU: two gloo ranks run the same host-side logic
that bench.py uses under torchrun (barrier, max over ranks of the step time,
rank-0-only output).  No GPU is involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


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
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        got = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_single_rank_is_identity():
    import bench
    import torch
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def _amax_worker(rank, world, port, shards, q):
    import datetime
    import sys

    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import dequantisation_fp8q_token_b200 as fp8q
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = []
        for shard in shards:
            # this rank's amax bits (numpy stands in for the device amax pass here)
            a = np.abs(np.asarray(shard[rank], np.float32))
            bits = np.where(np.isnan(a), np.float32(np.nan), a).view(np.uint32)
            local = int(bits.max()) if bits.size else 0
            t = torch.tensor([local], dtype=torch.int32)
            fp8q.allreduce_amax_bits(t)
            res.append(int(t.item()))
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_sharded_amax_exchange_two_ranks():
    """The exchange of the sharded per-tensor cast: both ranks end with the
    amax of the whole tensor, NaN from either rank propagating, empty shards
    contributing 0."""
    import numpy as np
    g = np.random.default_rng(0)
    shards = [
        [g.standard_normal(100).astype(np.float32), (g.standard_normal(50) * 7).astype(np.float32)],
        [np.array([1.0, -3.0], np.float32), np.array([np.nan, 2.0], np.float32)],
        [np.array([np.inf], np.float32), np.array([-5.0], np.float32)],
        [np.zeros(0, np.float32), np.array([-0.0, 2.5], np.float32)],
    ]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_amax_worker, args=(r, 2, port, shards, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1]
    for got, sh in zip(res[0], shards):
        whole = np.abs(np.concatenate(sh))
        if np.isnan(whole).any():
            assert np.array([got], np.uint32).view(np.float32)[0] != np.array([got], np.uint32).view(np.float32)[0]
        else:
            assert np.array([got], np.uint32).view(np.float32)[0] == whole.max()


def _records_worker(rank, world, port, q):
    """The exchange steps of the fp8-compressed collectives on gloo ranks:
    records made by the oracle (standing in for the device pack), moved by
    the library's exchange functions, decoded by the oracle."""
    import datetime
    import sys

    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import dequantisation_fp8q_token_b200 as fp8q
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        n = 1000 + 17
        R = fp8q.record_bytes(n)
        assert R == oracle.record_size(n)

        def tensor(r, i):
            g = np.random.default_rng(1000 * r + i)
            return (g.standard_normal(n) * 10.0 ** (r - i)).astype(np.float32)

        # all-gather: this rank's record at slot `rank`, the rest arrive
        combined = torch.zeros(world * R, dtype=torch.uint8)
        combined[rank * R:(rank + 1) * R] = torch.from_numpy(oracle.record(tensor(rank, 0), 0, 1))
        fp8q.exchange_records(combined, None)
        got = [oracle.record_decode(combined[r * R:(r + 1) * R].numpy(), n, 1, 0) for r in range(world)]
        want = oracle.all_gather_fp8([tensor(r, 0) for r in range(world)], 0, 1)
        ag = all(np.array_equal(a.view(np.uint32), b.view(np.uint32)) for a, b in zip(got, want))

        # all-to-all of records: slot j of send goes to rank j
        send = torch.from_numpy(np.concatenate([oracle.record(tensor(rank, j), 0, 0) for j in range(world)]))
        recv = torch.empty_like(send)
        fp8q.exchange_records_all_to_all(recv, send, None)
        got = [oracle.record_decode(recv[j * R:(j + 1) * R].numpy(), n, 0, 0) for j in range(world)]
        want = oracle.all_to_all_fp8([[tensor(j, i) for i in range(world)] for j in range(world)], 0, 0)[rank]
        a2a = all(np.array_equal(a.view(np.uint32), b.view(np.uint32)) for a, b in zip(got, want))

        # all_to_all_single: payload chunks + all-gathered scales
        whole = [np.concatenate([tensor(j, i) for i in range(world)]) for j in range(world)]
        qm, sm = oracle.cast_per_tensor(whole[rank], 0, 0)
        qr = torch.empty(qm.size, dtype=torch.uint8)
        scales = torch.empty(world, dtype=torch.float32)
        fp8q.exchange_payload_all_to_all(qr, torch.from_numpy(qm), scales, torch.from_numpy(sm), None)
        c = qm.size // world
        parts = [oracle.cast_from_fp8(qr[j * c:(j + 1) * c].numpy().reshape(1, c), scales[j:j + 1].numpy(),
                                      oracle.GRAN_TENSOR, 0, yt=0).reshape(-1) for j in range(world)]
        want = oracle.all_to_all_single_fp8(whole, 0, 0)[rank]
        a2as = np.array_equal(np.concatenate(parts).view(np.uint32), want.view(np.uint32))
        q.put((rank, (ag, a2a, a2as)))
    finally:
        dist.destroy_process_group()


def test_fp8_collective_exchanges_two_ranks():
    """Each rank ends with every rank's record (all-gather), the records
    meant for it (all-to-all), or its chunk of every rank's payload with the
    senders' scales (all_to_all_single); decoding gives the oracle's result."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_records_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: (True, True, True), 1: (True, True, True)}

"""GPU parity: the per-tensor cast of a tensor sharded across ranks (local
amax, a 4-byte integer MAX across ranks, cast with the global amax).  The
shards are emulated on one GPU, and a one-rank NCCL process group drives
the helper end to end; every shard's bytes must equal its slice of the
one-tensor cast, bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch

import workloads
from gpu_util import dev, host
from helpers import assert_codes_equal, assert_f32_equal

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1


def _whole(fp8q, x, fmt, rule):
    q = torch.empty(x.numel(), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_cast_per_tensor_ex(x, q, s, ws, fmt, rule)
    return host(q), host(s)


def _sharded(fp8q, x, cuts, fmt, rule):
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    parts = torch.tensor_split(x, cuts)
    words = []
    for p in parts:
        a = torch.empty(1, dtype=torch.int32, device="cuda")
        fp8q.fp8q_tensor_amax(p, a, ws)
        words.append(a)
    amax = torch.stack(words).max(dim=0).values          # the exchange: an integer MAX over "ranks"
    qs, ss = [], []
    for p in parts:
        q = torch.empty(p.numel(), dtype=torch.uint8, device="cuda")
        s = torch.empty(1, dtype=torch.float32, device="cuda")
        fp8q.fp8q_cast_per_tensor_with_amax(p, amax, q, s, fmt, rule)
        qs.append(host(q))
        ss.append(host(s))
    return np.concatenate(qs), ss, host(amax)


@pytest.mark.parametrize("rule", [0, 1])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
@pytest.mark.parametrize("kind", ["normal", "nan_in_one_shard", "zero", "one_big"])
def test_sharded_equals_whole(fp8q, rule, fmt, kind):
    g = np.random.default_rng(hash((rule, fmt, kind)) & 0xFFFF)
    v = (g.standard_normal(3_000_017) * 0.01).astype(np.float32)
    if kind == "nan_in_one_shard":
        v[2_500_000] = np.nan
    elif kind == "zero":
        v[:] = 0.0
    elif kind == "one_big":
        v[1234] = 9.0e4
    x = dev(v)
    cuts = [0, 1_000_000, 1_000_001, 2_222_222]          # includes an empty shard
    qw, sw = _whole(fp8q, x, fmt, rule)
    qs, ss, amax = _sharded(fp8q, x, cuts, fmt, rule)
    assert_codes_equal(qs, qw, fmt)
    for s in ss:
        assert_f32_equal(s, sw)
    a = np.abs(v)
    want = np.float32(np.nan) if np.isnan(a).any() else a.max()
    got = amax.view(np.float32)[0]
    assert (np.isnan(got) and np.isnan(want)) or got == want


def test_tensor_amax_bf16_and_empty(fp8q):
    x = workloads.c2_x()
    a = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_tensor_amax(dev(x), a, ws)
    want = np.abs((x.astype(np.uint32) << 16).view(np.float32)).max()
    assert host(a).view(np.float32)[0] == want
    fp8q.fp8q_tensor_amax(torch.empty(0, device="cuda"), a, ws)
    assert int(a.item()) == 0


def test_cast_to_fp8_sharded_one_rank_nccl(fp8q):
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        v = dev((np.random.default_rng(4).standard_normal(1 << 20) * 3).astype(np.float32))
        q, sc = fp8q.cast_to_fp8_sharded(v, "e5m2")
        qw, sw = _whole(fp8q, v, E5M2, 0)
        assert_codes_equal(host(q), qw, E5M2)
        assert_f32_equal(host(sc), sw)
    finally:
        dist.destroy_process_group()

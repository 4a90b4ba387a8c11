"""GPU parity for the fp8-compressed collectives (ColossalAI all_gather_fp8 /
all_gather_fp8_lagacy, all_to_all_fp8, all_to_all_single_fp8).

1. Ranks emulated on one GPU: every rank's record is packed by the library
   into its slot of one buffer (the state after the all-gather), the record
   bytes must equal the oracle's (header, codes and zero padding), and one
   unpack call must give every rank's tensor as the oracle decodes it.
2. A one-rank NCCL process group drives the helpers end to end.
"""
import socket

import numpy as np
import pytest
import torch

import workloads
from gpu_util import Guarded, dev, host
from helpers import assert_codes_equal, assert_f32_equal
from test_gpu_per_token import TORCH_DT

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2


def _input(g, n, xt, kind):
    v = g.standard_normal(n) * 10.0 ** g.uniform(-3, 3)
    if kind == "nonfinite" and n > 2:
        v[g.integers(0, n)] = np.inf
        v[g.integers(0, n)] = np.nan
    elif kind == "zero":
        v[:] = 0.0
    elif kind == "overflow" and n > 0:
        v[0] = 1.0e30                                    # e5m2 / e4m3 saturation edge
    v = v.astype(np.float32)
    if xt == F32:
        return v
    if xt == BF16:
        return workloads.to_bf16_bits(v)
    return v.astype(np.float16).view(np.uint16)


def _to_dev(x, xt):
    return dev(x, TORCH_DT[xt]) if xt != F32 else dev(x)


def _compare_records(got, want, n, fmt, head=16):
    """Header scale_inv (NaN as a class), header zeros, codes, padding zeros (head 16); the
    scale then the codes (head 4, the page's packed layout)."""
    assert got.size == want.size
    assert_f32_equal(got[:4].copy().view(np.float32), want[:4].copy().view(np.float32), name="scale_inv")
    np.testing.assert_array_equal(got[4:head], want[4:head])
    assert_codes_equal(got[head:head + n], want[head:head + n], fmt)
    np.testing.assert_array_equal(got[head + n:], want[head + n:])


def _compare_values(got, want, xt):
    if xt == F32:
        assert_f32_equal(got, want)
    else:
        g, w = got.view(np.uint16), want.view(np.uint16)
        exp = 0x7F80 if xt == BF16 else 0x7C00
        man = 0x007F if xt == BF16 else 0x03FF
        gn = ((g & exp) == exp) & ((g & man) != 0)
        wn = ((w & exp) == exp) & ((w & man) != 0)
        bad = (gn != wn) | (~gn & (g != w))
        assert not bad.any(), f"{bad.sum()} of {bad.size} differ; first at {np.flatnonzero(bad)[:5]}"


def _emulated_all_gather(fp8q, orc, xs, xt, fmt, rule):
    W, n = len(xs), np.asarray(xs[0]).size
    R = fp8q.record_bytes(n)
    assert fp8q.fp8q_record_bytes(n) == R
    combined = torch.full((W * R,), 0xAB, dtype=torch.uint8, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    for r, x in enumerate(xs):
        fp8q.fp8q_pack_record(_to_dev(x, xt), combined[r * R:(r + 1) * R], ws, fmt, rule)
    got = host(combined)
    for r, x in enumerate(xs):
        _compare_records(got[r * R:(r + 1) * R], orc.record(x, xt, fmt, rule), n, fmt)
    y = Guarded(W * n, TORCH_DT[xt] if xt != F32 else torch.float32)
    fp8q.fp8q_unpack_records(combined, W, n, y.t, fmt)
    y.check()
    ys = host(y.t)
    want = orc.all_gather_fp8(xs, xt, fmt, rule)
    for r in range(W):
        _compare_values(ys[r * n:(r + 1) * n], want[r], xt)


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 4095, 4096, 4097, 3 * 4096 + 17, 1_000_003])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_records_emulated_ranks(fp8q, orc, n, fmt):
    g = np.random.default_rng(n * 7 + fmt)
    for xt in (F32, BF16, F16):
        xs = [_input(g, n, xt, "normal") for _ in range(4)]
        _emulated_all_gather(fp8q, orc, xs, xt, fmt, 0)


@pytest.mark.parametrize("kind", ["nonfinite", "zero", "overflow"])
@pytest.mark.parametrize("rule", [0, 1])
def test_records_edge_values(fp8q, orc, kind, rule):
    g = np.random.default_rng(hash((kind, rule)) & 0xFFFF)
    for fmt in (E4M3FN, E5M2):
        xs = [_input(g, 5000, F32, kind), _input(g, 5000, F32, "normal")]
        _emulated_all_gather(fp8q, orc, xs, F32, fmt, rule)


@pytest.mark.parametrize("n", [100, 5000])
def test_records_many_ranks(fp8q, orc, n):
    """More records than one launch takes (48 records per launch when each
    has a body and a tail)."""
    g = np.random.default_rng(n)
    xs = [_input(g, n, BF16, "normal") for _ in range(97)]
    _emulated_all_gather(fp8q, orc, xs, BF16, E4M3FN, 0)


def test_records_full_size(fp8q, orc):
    """8 ranks x 16 Mi bf16 elements (a 32 MiB shard each): records equal
    the oracle's on sampled ranges; decoded values on sampled ranges."""
    W, n = 8, 1 << 24
    R = fp8q.record_bytes(n)
    g = np.random.default_rng(77)
    xs = [_input(g, n, BF16, "normal") for _ in range(W)]
    combined = torch.empty((W * R,), dtype=torch.uint8, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    for r, x in enumerate(xs):
        fp8q.fp8q_pack_record(_to_dev(x, BF16), combined[r * R:(r + 1) * R], ws, E5M2)
    y = torch.empty((W * n,), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_unpack_records(combined, W, n, y, E5M2)
    got_rec, got_y = host(combined), host(y)
    for r, x in enumerate(xs):
        want = orc.record(x, BF16, E5M2)
        _compare_records(got_rec[r * R:(r + 1) * R], want, n, E5M2)
        q = want[16:16 + n].reshape(1, n)
        s = want[:4].view(np.float32)
        for a in (0, n // 2 + 3, n - 9000):
            yo = orc.cast_from_fp8(q[:, a:a + 9000], s, orc.GRAN_TENSOR, E5M2, yt=BF16).reshape(-1)
            _compare_values(got_y[r * n + a:r * n + a + 9000], yo, BF16)


def test_record_arguments_checked(fp8q):
    x = torch.zeros(64, dtype=torch.float32, device="cuda")
    buf = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8q.Fp8qError, match="align"):
        fp8q.fp8q_pack_record(x, buf[8:8 + 96], ws, E4M3FN)
    with pytest.raises(fp8q.Fp8qError, match="align"):
        fp8q.fp8q_unpack_records(buf[4:], 1, 64, x, E4M3FN)
    y = torch.empty(64, dtype=torch.float32, device="cuda")
    fp8q.fp8q_pack_record(x, buf[:96], ws, E4M3FN)
    fp8q.fp8q_unpack_records(buf[:96], 1, 64, y, E4M3FN)
    assert (host(y) == 0).all()
    # an all-zero tensor takes amax 1: scale 448, scale_inv fl(1 / 448)
    assert host(buf[:4]).view(np.float32)[0] == np.float32(1.0) / np.float32(448.0)


class _OneRankNccl:
    def __enter__(self):
        import torch.distributed as dist
        s = socket.socket()
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
        s.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                device_id=torch.device("cuda", 0))
        return self

    def __exit__(self, *exc):
        import torch.distributed as dist
        dist.destroy_process_group()


def test_collectives_one_rank_nccl(fp8q, orc):
    g = np.random.default_rng(123)
    with _OneRankNccl():
        x = _input(g, 3 * 4096 + 5, BF16, "normal")
        xd = _to_dev(x, BF16)
        outs = [torch.empty_like(xd)]
        fp8q.all_gather_fp8(outs, xd, fp8_format="e5m2")
        _compare_values(host(outs[0]), orc.all_gather_fp8([x], BF16, E5M2)[0], BF16)
        flat = torch.empty((1, xd.numel()), dtype=torch.bfloat16, device="cuda")
        fp8q.all_gather_fp8(flat, xd, fp8_format="e4m3")
        _compare_values(host(flat).reshape(-1), orc.all_gather_fp8([x], BF16, E4M3FN)[0], BF16)
        # the page's own wire layout (4-byte scale, then the codes)
        fp8q.all_gather_fp8(flat, xd, fp8_format="e5m2", layout=fp8q.RECORD_PACKED4)
        _compare_values(host(flat).reshape(-1), orc.all_gather_fp8([x], BF16, E5M2, header=4)[0], BF16)
        # all_to_all_fp8: one tensor for the one rank
        y = [torch.empty_like(xd)]
        fp8q.all_to_all_fp8(y, [xd], fp8_format="e4m3")
        _compare_values(host(y[0]), orc.all_to_all_fp8([[x]], BF16, E4M3FN)[0][0], BF16)
        # all_to_all_single_fp8 over a [rows, cols] fp32 tensor
        v = (g.standard_normal((64, 1000)) * 5).astype(np.float32)
        vd = dev(v)
        out = torch.empty_like(vd)
        fp8q.all_to_all_single_fp8(out, vd, fp8_format="e5m2")
        _compare_values(host(out).reshape(-1), orc.all_to_all_single_fp8([v.reshape(-1)], F32, E5M2)[0], F32)


def _emulated_all_gather_packed4(fp8q, orc, xs, xt, fmt, rule):
    """The page's own wire layout (all_gather_fp8_lagacy, SCALE_BYTES = 4): each rank's record
    is its 4-byte scale then its codes, back to back; compared byte for byte with the oracle's
    records of that layout, and the decoded values bit for bit."""
    W, n = len(xs), np.asarray(xs[0]).size
    R = fp8q.record_bytes(n, fp8q.RECORD_PACKED4)
    assert R == 4 + n == fp8q.fp8q_record_bytes_ex(n, fp8q.RECORD_PACKED4)
    combined = Guarded(W * R, torch.uint8)
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    for r, x in enumerate(xs):
        fp8q.fp8q_pack_record_ex(_to_dev(x, xt), combined.t[r * R:(r + 1) * R], ws, fmt, rule, fp8q.RECORD_PACKED4)
    combined.check()
    got = host(combined.t)
    for r, x in enumerate(xs):
        want = orc.record(x, xt, fmt, rule, header=4)
        assert want.size == R
        _compare_records(got[r * R:(r + 1) * R], want, n, fmt, head=4)
    y = Guarded(W * n, TORCH_DT[xt] if xt != F32 else torch.float32)
    fp8q.fp8q_unpack_records_ex(combined.t, W, n, y.t, fmt, fp8q.RECORD_PACKED4)
    y.check()
    ys = host(y.t)
    want = orc.all_gather_fp8(xs, xt, fmt, rule, header=4)
    for r in range(W):
        _compare_values(ys[r * n:(r + 1) * n], want[r], xt)


@pytest.mark.parametrize("n", [4, 16, 20, 4096, 4100, 3 * 4096 + 20, 1_000_004])
@pytest.mark.parametrize("fmt", [E4M3FN, E5M2])
def test_records_packed4_emulated_ranks(fp8q, orc, n, fmt):
    g = np.random.default_rng(n * 11 + fmt)
    for xt in (F32, BF16):
        xs = [_input(g, n, xt, "normal") for _ in range(3)]
        _emulated_all_gather_packed4(fp8q, orc, xs, xt, fmt, 0)


@pytest.mark.parametrize("n", [1, 3, 4097])
def test_records_packed4_one_record_any_numel(fp8q, orc, n):
    """A single packed record takes any numel: its scale sits at the (4-byte aligned) start."""
    g = np.random.default_rng(n)
    _emulated_all_gather_packed4(fp8q, orc, [_input(g, n, F32, "nonfinite")], F32, E5M2, 1)


def test_records_packed4_arguments_checked(fp8q):
    x = torch.zeros(6, dtype=torch.float32, device="cuda")
    buf = torch.zeros(64, dtype=torch.uint8, device="cuda")
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    y = torch.empty(12, dtype=torch.float32, device="cuda")
    P4 = fp8q.RECORD_PACKED4
    with pytest.raises(fp8q.Fp8qError, match="align"):            # the scale would be unaligned
        fp8q.fp8q_pack_record_ex(x, buf[2:12], ws, E4M3FN, 0, P4)
    with pytest.raises(fp8q.Fp8qError, match="align"):            # record 1's scale at 4 + 6 = 10
        fp8q.fp8q_unpack_records_ex(buf[:20], 2, 6, y, E4M3FN, P4)
    fp8q.fp8q_pack_record_ex(x, buf[4:14], ws, E4M3FN, 0, P4)     # 4-byte aligned: accepted
    fp8q.fp8q_unpack_records_ex(buf[4:14], 1, 6, y[:6], E4M3FN, P4)
    assert (host(y[:6]) == 0).all()
    assert host(buf[4:8]).view(np.float32)[0] == np.float32(1.0) / np.float32(448.0)
    with pytest.raises(ValueError):
        fp8q.record_bytes(6, 8)

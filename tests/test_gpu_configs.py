"""GPU parity at the workloads' full sizes, in the exact launch configuration
that bench.py times (its Workload runs one step), against the CPU oracle:
full comparisons where the threaded oracle finishes in seconds, whole sampled
weights for the 3 GB grouped dequant."""
import numpy as np
import pytest
import torch

import bench
import workloads
from gpu_util import THREADS, host
from helpers import assert_codes_equal, assert_f32_equal, assert_out_equal, bf16_to_f32

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2


@pytest.fixture(scope="module")
def stepped(fp8q):
    wl = bench.Workload(torch.device("cuda", 0), fp8q)
    wl.step()
    wl.step()          # a second step over the same buffers must leave the same bytes
    torch.cuda.synchronize()
    return wl


def test_c1_small_per_token_and_round_trip(fp8q, orc):
    x = workloads.c1_x()
    q, s = fp8q.per_token_cast_to_fp8(bench._to_dev(x, "cuda", torch.bfloat16))
    y = fp8q.per_token_cast_back(q, s, torch.bfloat16)
    qo, so = orc.per_token_group_quant(x, BF16, 128, E4M3FN)
    assert_codes_equal(host(q), qo, E4M3FN)
    assert_f32_equal(host(s), so)
    assert_out_equal(host(y), orc.cast_from_fp8(qo, so, orc.GRAN_GROUP, E4M3FN, 128, BF16), BF16)
    assert (host(q)[3] == 0).all() and (host(s)[3].view(np.uint32) == 0x346FACAD).all()
    assert host(q)[7, 517] & 0x7F == 0x7E


def test_c2_per_token_full(stepped, orc):
    x = stepped.host["c2_x"]
    qo, so = orc.per_token_group_quant(x, BF16, 128, E4M3FN, threads=THREADS)
    assert_codes_equal(host(stepped.c2_q), qo, E4M3FN)
    assert_f32_equal(host(stepped.c2_s), so)
    yo = orc.cast_from_fp8(qo, so, orc.GRAN_GROUP, E4M3FN, 128, BF16, threads=THREADS)
    assert_out_equal(host(stepped.c2_y), yo, BF16)


def test_c2_outliers_land_on_fmax(stepped):
    """Invariant at full size: every group's amax element is +-448."""
    x = np.abs(bf16_to_f32(stepped.host["c2_x"])).reshape(4096, 56, 128)
    q = host(stepped.c2_q).reshape(4096, 56, 128)
    amax = x.max(axis=2, keepdims=True)
    hit = (x == amax) & (amax >= np.float32(1e-4))
    assert ((q[hit] & 0x7F) == 0x7E).all()


def test_c3_block_dequant_full(stepped, orc):
    yo = orc.block_dequant(stepped.host["c3_w"], stepped.host["c3_s"], E4M3FN, 128, BF16, threads=THREADS)
    assert_out_equal(host(stepped.c3_y), yo, BF16)


def test_c4a_per_channel_full(stepped, orc):
    qo, so = orc.cast_per_channel(stepped.host["c4a_x"], BF16, E4M3FN, threads=THREADS)
    assert_codes_equal(host(stepped.c4a_q), qo, E4M3FN)
    assert_f32_equal(host(stepped.c4a_s), so)
    assert (host(stepped.c4a_q)[4096] == 0).all() and host(stepped.c4a_s)[4096].view(np.uint32) == 0x3B124925


def test_c4b_per_tensor_full(stepped, orc):
    qo, so = orc.cast_per_tensor(stepped.host["c4b_v"], F32, E5M2, threads=4)
    assert_codes_equal(host(stepped.c4b_q), qo, E5M2)
    assert_f32_equal(host(stepped.c4b_s), so)


def test_c4c_per_tensor_zero(stepped):
    assert (host(stepped.c4c_q) == 0).all()
    assert host(stepped.c4c_s).view(np.uint32)[0] == 0x3B124925


@pytest.mark.parametrize("i", [0, 1, 37, 63, 64, 66, 71])
def test_c5_grouped_sampled_weights(stepped, orc, i):
    w, s = stepped.host["c5"][i]
    yo = orc.block_dequant(w, s, E4M3FN, 128, BF16, threads=THREADS)
    assert_out_equal(host(stepped.c5_y[i]), yo, BF16, name=f"weight {i}")


def test_c5_all_weights_row_samples(stepped, orc):
    """Every one of the 72 weights: its first, last and a middle row block."""
    g = np.random.default_rng(0)
    for i, (w, s) in enumerate(stepped.host["c5"]):
        M = w.shape[0]
        y = host(stepped.c5_y[i])
        for r0 in (0, M - 1 - (M - 1) % 128, int(g.integers(0, M))):
            r1 = min(M, r0 + 8)
            yo = orc.block_dequant(w, s, E4M3FN, 128, BF16, rows=(r0, r1))
            assert_out_equal(y[r0:r1], yo[r0:r1], BF16, name=f"weight {i} rows {r0}:{r1}")


# ---------------------------------------------------------------------------
# the fp8 products, in the launch configuration bench.py's matmul section times
# ---------------------------------------------------------------------------
def _mm_bound(got_bits, exact, mag, K):
    """The accumulation bound of the fp8 products: (ceil(K/32) + 1) * 2^-23 of sum |a * b|,
    2^-24 per k-block for the fine-grained fold, and one bf16 ulp of the output."""
    import torch
    got = torch.from_numpy(got_bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    rel = (-(-K // 32) + 1) * 2.0 ** -23 + (-(-K // 128)) * 2.0 ** -24
    e = np.floor(np.log2(np.maximum(np.abs(exact), 2.0 ** -126)))
    bad = ~(np.abs(got - exact) <= rel * mag + 2.0 ** (e - 7))
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outside the bound"


def test_matmul_workload_sampled_rows(stepped, orc):
    """bench.MatmulWorkload's own operands and launches: its per-token codes equal the oracle's
    (so the oracle's product starts from its own codes), then sampled rows of both products."""
    import torch
    mm = bench.MatmulWorkload(stepped)
    qo, so = orc.per_token_group_quant(stepped.host["c2_x"], BF16, 128, E4M3FN, threads=THREADS)
    assert_codes_equal(host(mm.q), qo, E4M3FN)
    assert_f32_equal(host(mm.sa), so)
    w, sb = workloads.mm_w_s()
    rows = [0, 5, 1000, 4095]
    wabs = np.abs(torch.from_numpy(w).view(torch.float8_e4m3fn).to(torch.float32).numpy())
    aabs = np.abs(torch.from_numpy(qo[rows]).view(torch.float8_e4m3fn).to(torch.float32).numpy())
    K = qo.shape[1]
    # fine-grained
    mm.ops["scaled_mm_blockwise"]()
    got = host(mm.out)
    mag = ((aabs * np.repeat(so[rows], 128, 1)) @ (wabs * np.repeat(np.repeat(sb, 128, 0), 128, 1)).T).astype(np.float64)
    for i, r in enumerate(rows):
        exact = orc.scaled_mm_blockwise(qo, E4M3FN, so, w, E4M3FN, sb, rows=(r, r + 1), threads=THREADS)[r]
        _mm_bound(got[r], exact, mag[i], K)
    # per-tensor, the scales bench.py uses (the first group's and the first block's)
    mm.ops["scaled_mm_per_tensor"]()
    got = host(mm.out)
    s1, s2 = float(so[0, 0]), float(sb[0, 0])
    mag = (aabs @ wabs.T).astype(np.float64) * float(np.float32(s1) * np.float32(s2))
    for i, r in enumerate(rows):
        exact = orc.scaled_mm(qo, E4M3FN, w, E4M3FN, s1, s2, rows=(r, r + 1), threads=THREADS)[r]
        _mm_bound(got[r], exact, mag[i], K)
    assert int(mm.status.item()) == 0


def test_end_to_end_units_give_the_device_step_bytes(stepped):
    """bench.py's end-to-end step cuts ops into row / weight units on three streams; its host
    outputs must equal the whole-op device step's outputs byte for byte."""
    want = {id(t): host(t).copy() for t in stepped.outputs()}
    e2e = bench.EndToEnd(stepped)
    assert len(e2e.units) > len(stepped.ops)
    e2e.step()
    torch.cuda.synchronize()
    for t in stepped.outputs():
        got = e2e.h[id(t)].view(torch.uint8).numpy() if t.element_size() == 1 else host(e2e.h[id(t)])
        np.testing.assert_array_equal(np.asarray(got).reshape(-1), want[id(t)].reshape(-1))

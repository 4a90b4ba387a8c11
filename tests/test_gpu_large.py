"""GPU parity above 2^32 elements: every kernel's indexing must be 64-bit.

Each case holds more than 2^32 elements (so byte offsets pass both 2^31 and
2^32 in every tensor), is drawn on the device by a seeded torch generator,
and is compared with the oracle bit for bit on sampled rows: the first
rows, the rows that hold elements 2^31 and 2^32, and the last rows.  The
output tensors sit between canary bytes, checked on the device."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import host
from helpers import assert_codes_equal, assert_f32_equal

pytestmark = pytest.mark.gpu

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
GRAN_TENSOR, GRAN_ROW, GRAN_GROUP, GRAN_BLOCK = 0, 1, 2, 3
GUARD = 4096


class DevGuarded:
    """An output tensor between canary bytes; the canaries are checked on the device."""

    def __init__(self, shape, dtype):
        numel = int(np.prod(shape))
        esz = torch.empty((), dtype=dtype).element_size()
        self.nbytes = numel * esz
        self.raw = torch.full((2 * GUARD + self.nbytes,), 0xA5, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def check(self):
        assert bool((self.raw[:GUARD] == 0xA5).all()), "write before an output tensor"
        assert bool((self.raw[GUARD + self.nbytes:] == 0xA5).all()), "write past an output tensor"


def _sample_rows(n_cols, n_rows, width=8):
    """Row ranges: the first rows, those holding elements 2^31 and 2^32, the last rows."""
    out = [(0, width)]
    for e in (1 << 31, 1 << 32):
        r = e // n_cols
        if r < n_rows:
            out.append((max(0, r - width // 2), min(n_rows, r + width // 2)))
    out.append((n_rows - width, n_rows))
    return out


def _bits(t):
    return host(t)


def test_per_token_and_round_trip_above_2_32(fp8q, orc):
    m, n = 600_000, 7168                                  # 4,300,800,000 elements
    assert m * n > 1 << 32
    x = workloads.device_normal((m, n), seed=9101)
    q = DevGuarded((m, n), torch.uint8)
    s = DevGuarded((m, n // 128), torch.float32)
    fp8q.fp8q_per_token_group_quant(x, q.t, s.t, 128, E4M3FN)
    y = DevGuarded((m, n), torch.bfloat16)
    fp8q.fp8q_cast_from_fp8(q.t, s.t, y.t, GRAN_GROUP, 128, E4M3FN)
    for g in (q, s, y):
        g.check()
    for r0, r1 in _sample_rows(n, m):
        xs = _bits(x[r0:r1])
        qo, so = orc.per_token_group_quant(xs, BF16, 128, E4M3FN)
        assert_codes_equal(_bits(q.t[r0:r1]), qo, E4M3FN, name=f"rows {r0}-{r1}")
        assert_f32_equal(_bits(s.t[r0:r1]), so, name=f"rows {r0}-{r1}")
        yo = orc.cast_from_fp8(qo, so, GRAN_GROUP, E4M3FN, gb=128, yt=BF16)
        np.testing.assert_array_equal(_bits(y.t[r0:r1]), yo)


def test_block_dequant_above_2_32(fp8q, orc):
    M, N = 262_150, 16_400                                # 4,299,260,000 codes; ragged in both
    assert M * N > 1 << 32
    w = workloads.device_codes((M, N), seed=9102)
    sm, sn = workloads.scale_shape(M, N)
    s_host = workloads.lognormal_scales(workloads.rng(9103), (sm, sn))
    s = torch.from_numpy(s_host).cuda()
    y = DevGuarded((M, N), torch.bfloat16)
    fp8q.fp8q_block_dequant(w, s, y.t, 128, E4M3FN)
    y.check()
    # slices that start on a block row, so the oracle takes one block row of s
    for r0, r1 in ((0, 16), (130_944, 130_960), (261_888, 261_904), (262_144, 262_150)):
        assert r0 % 128 == 0 and (r1 - 1) // 128 == r0 // 128
        b = r0 // 128
        yo = orc.block_dequant(_bits(w[r0:r1]), s_host[b:b + 1], E4M3FN, 128, BF16)
        np.testing.assert_array_equal(_bits(y.t[r0:r1]), yo, err_msg=f"rows {r0}-{r1}")


def test_per_channel_above_2_32(fp8q, orc):
    R, C = 524_300, 8192                                  # 4,295,065,600 elements
    assert R * C > 1 << 32
    x = workloads.device_normal((R, C), seed=9104)
    q = DevGuarded((R, C), torch.uint8)
    s = DevGuarded((R,), torch.float32)
    fp8q.fp8q_cast_per_channel(x, q.t, s.t, E5M2)
    q.check()
    s.check()
    for r0, r1 in _sample_rows(C, R):
        qo, so = orc.cast_per_channel(_bits(x[r0:r1]), BF16, E5M2)
        assert_codes_equal(_bits(q.t[r0:r1]), qo, E5M2, name=f"rows {r0}-{r1}")
        assert_f32_equal(_bits(s.t[r0:r1]), so, name=f"rows {r0}-{r1}")


def test_per_tensor_and_record_above_2_32(fp8q, orc):
    """fp16 [2^32 + 4099]: N(0, 0.01) with 3.0 planted past element 2^32, so
    the global amax is 3.0 (checked on the device); every sampled element's
    code then equals the oracle's per-tensor cast of the planted element
    together with the samples, since a code depends on its element and the
    amax only."""
    n = (1 << 32) + 4099
    x = workloads.device_normal((n,), seed=9105, dtype=torch.float16, row_scale=False, std=0.01)
    big = (1 << 32) + 1000
    x[big] = 3.0
    x[5] = -2.5
    assert float(x.abs().max()) == 3.0
    q = DevGuarded((n,), torch.uint8)
    s = DevGuarded((1,), torch.float32)
    ws = torch.empty(fp8q.fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_cast_per_tensor(x, q.t, s.t, ws, E4M3FN)
    amax = torch.empty(1, dtype=torch.int32, device="cuda")
    fp8q.fp8q_tensor_amax(x, amax, ws)
    rec = torch.empty((fp8q.record_bytes(n),), dtype=torch.uint8, device="cuda")
    fp8q.fp8q_pack_record(x, rec, ws, E4M3FN)
    y = DevGuarded((n,), torch.float16)
    fp8q.fp8q_unpack_records(rec, 1, n, y.t, E4M3FN)
    q.check()
    s.check()
    y.check()
    assert host(amax).view(np.float32)[0] == np.float32(3.0)
    ranges = [(0, 4096), ((1 << 31) - 100, (1 << 31) + 100), ((1 << 32) - 100, (1 << 32) + 1100), (n - 200, n)]
    xs = np.concatenate([_bits(x[big:big + 1])] + [_bits(x[a:b]) for a, b in ranges])
    qo, so = orc.cast_per_tensor(xs, F16, E4M3FN)
    assert_f32_equal(_bits(s.t), so)
    assert host(rec[:4]).view(np.float32)[0] == so[0]
    o = 1
    for a, b in ranges:
        assert_codes_equal(_bits(q.t[a:b]), qo[o:o + b - a], E4M3FN, name=f"elements {a}-{b}")
        assert_codes_equal(_bits(rec[16 + a:16 + b]), qo[o:o + b - a], E4M3FN, name=f"record {a}-{b}")
        yo = orc.cast_from_fp8(qo[o:o + b - a].reshape(1, -1), so, GRAN_TENSOR, E4M3FN, yt=F16).reshape(-1)
        np.testing.assert_array_equal(_bits(y.t[a:b]), yo, err_msg=f"decoded {a}-{b}")
        o += b - a


@pytest.fixture(autouse=True)
def _release_memory():
    yield
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# the fp8 products and linear_fp8's backward helpers
# ---------------------------------------------------------------------------
def _grid_codes_dev(shape, gen):
    """e4m3fn codes whose values are multiples of 1/8 with magnitude <= 4, drawn on the
    device: every partial sum of a product of such operands over K = 32 is an fp32 number."""
    codes = workloads.finite_e4m3fn_codes()
    v = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    keep = torch.from_numpy(codes[(np.abs(v) <= 4) & (v * 8 == np.round(v * 8))]).cuda()
    idx = torch.randint(0, keep.numel(), shape, generator=gen, device="cuda")
    return keep[idx]


@pytest.mark.parametrize("fine", [False, True], ids=["tensor", "blockwise"])
def test_scaled_mm_output_above_2_32(fp8q, orc, fine):
    """D [65552, 65552] bf16 (4,297,064,704 elements) from K = 32 exact-grid operands, with a
    bias: the sampled rows (the first, those holding elements 2^31 and 2^32, the last) equal
    the oracle's single-precision product bit for bit."""
    M = N = 65552
    K = 32
    gen = torch.Generator(device="cuda").manual_seed(9107 + fine)
    a = _grid_codes_dev((M, K), gen)
    b = _grid_codes_dev((N, K), gen)
    bias = (torch.randint(-512, 512, (N,), generator=gen, device="cuda") / 64.0).to(torch.bfloat16)
    d = DevGuarded((M, N), torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if fine:
        sa = torch.exp(torch.randn((M, 1), generator=gen, device="cuda") * 0.5 - 2.0)
        sb = torch.exp(torch.randn((-(-N // 128), 1), generator=gen, device="cuda") * 0.5 - 2.0)
        fp8q.fp8q_scaled_mm_blockwise(a, sa, b, sb, d.t, bias, status=st)
    else:
        sa = torch.tensor([0.375], device="cuda")
        sb = torch.tensor([1.25], device="cuda")
        fp8q.fp8q_scaled_mm(a, b, sa, sb, d.t, bias, status=st)
    d.check()
    assert int(st.item()) == 0
    b_h = host(b)
    bias_h = bias.float().cpu().numpy()
    for r0, r1 in _sample_rows(N, M):
        a_h = host(a[r0:r1])
        if fine:
            want = orc.scaled_mm_blockwise_rounded(a_h, E4M3FN, host(sa[r0:r1]), b_h, E4M3FN, host(sb),
                                                   bias=bias_h, yt=BF16)
        else:
            want = orc.scaled_mm_rounded(a_h, E4M3FN, b_h, E4M3FN, 0.375, 1.25, bias=bias_h, yt=BF16)
        np.testing.assert_array_equal(_bits(d.t[r0:r1]), want, err_msg=f"rows {r0}-{r1}")


def test_transpose_above_2_32(fp8q, orc):
    """uint8 [65552, 65552] (4.3 GB) transposed: the destination rows that start before 2^31,
    past 2^31 and past 2^32 bytes, and the last ones, against the oracle's transpose of the
    same source columns."""
    R = C = 65552
    gen = torch.Generator(device="cuda").manual_seed(9108)
    src = torch.randint(0, 256, (R, C), generator=gen, device="cuda", dtype=torch.uint8)
    dst = DevGuarded((C, R), torch.uint8)
    fp8q.fp8q_transpose_fp8(src, dst.t, R)
    dst.check()
    for c0, c1 in _sample_rows(R, C):
        cols = torch.arange(c0, c1, device="cuda")
        want = orc.transpose_u8(host(src[:, cols]))
        np.testing.assert_array_equal(host(dst.t[c0:c1]), want, err_msg=f"destination rows {c0}-{c1}")


def test_sum_rows_above_2_32(fp8q, orc):
    """bf16 [1,048,600, 4104] (4,303,454,400 elements) of integers in [-8, 8]: every partial
    sum is an fp32 integer, so the column sums are exact in any order and equal the oracle's
    binary64 sums rounded once to bf16; sampled columns include the partial last block."""
    R, C = 1_048_600, 4104
    gen = torch.Generator(device="cuda").manual_seed(9109)
    x = torch.randint(-8, 9, (R, C), generator=gen, device="cuda", dtype=torch.int8).to(torch.bfloat16)
    out = DevGuarded((C,), torch.bfloat16)
    fp8q.fp8q_sum_rows(x, out.t)
    out.check()
    for c0, c1 in [(0, 8), (2048, 2056), (4040, 4104)]:
        cols = torch.arange(c0, c1, device="cuda")
        exact = orc.sum_rows(host(x[:, cols]), BF16)
        want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(_bits(out.t[c0:c1]), want, err_msg=f"columns {c0}-{c1}")

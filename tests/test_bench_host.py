"""bench.py's algorithmic byte counts, checked against the figures derived
independently from the workload shapes (input read once per pass the method
needs, output written once), without a GPU: the Workload is built on torch's
meta device from zero-filled host arrays of the right shapes.  Also the choice of the timed
steps that carry the dominant op's event pair."""
import numpy as np
import torch

import bench
import workloads


def _zero_inputs():
    M3, N3 = workloads.C3_SHAPE
    return {
        "c2_x": np.zeros(workloads.C2_SHAPE, np.uint16),
        "c3_w": np.zeros((M3, N3), np.uint8),
        "c3_s": np.zeros(workloads.scale_shape(M3, N3), np.float32),
        "c4a_x": np.zeros(workloads.C4A_SHAPE, np.uint16),
        "c4b_v": np.zeros(workloads.C4B_NUMEL, np.float32),
        "c4c_v": np.zeros(workloads.C4C_NUMEL, np.uint16),
        "c5": [(np.zeros(sh, np.uint8), np.zeros(workloads.scale_shape(*sh), np.float32))
               for sh in workloads.C5_SHAPES],
    }


def test_step_bytes_match_the_derivation():
    import dequantisation_fp8q_token_b200 as fp8q
    wl = bench.Workload(torch.device("meta"), fp8q, _zero_inputs())
    b = {op.name: op.bytes for op in wl.ops}
    assert b["per_token_group_quant"] == 58_720_256 + 29_360_128 + 917_504 == 88_997_888
    assert b["cast_from_fp8_group"] == 88_997_888
    assert b["block_dequant"] == 132_120_576 + 264_241_152 + 32_256 == 396_393_984
    assert b["cast_per_channel"] == 134_217_728 + 67_108_864 + 32_768 == 201_359_360
    assert b["cast_per_tensor_f32_e5m2"] == 2 * 268_435_456 + 67_108_864 + 4 == 603_979_780
    assert b["cast_per_tensor_f16_zero"] == 2 * 2_097_152 + 1_048_576 + 4 == 5_242_884
    assert b["block_dequant_grouped"] == 995_524_096 * 3 + 243_456 == 2_986_815_744
    assert wl.step_bytes == sum(b.values())
    assert wl.launches_per_step == 9
    # e2e traffic: every input host->device, every output device->host
    bi = sum(t.numel() * t.element_size() for t in wl.inputs())
    bo = sum(t.numel() * t.element_size() for t in wl.outputs())
    assert bi == 58_720_256 + 132_120_576 + 32_256 + 134_217_728 + 268_435_456 + 2_097_152 + 995_524_096 + 243_456
    assert bo == (29_360_128 + 917_504 + 58_720_256 + 264_241_152 + 67_108_864 + 32_768 + 67_108_864 + 4
                  + 1_048_576 + 4 + 995_524_096 * 2)


def test_traffic_fingerprint_ignores_comments_only(tmp_path, monkeypatch):
    """The DRAM-traffic record stays valid across comment and whitespace edits of the kernel
    sources, and any change to their code voids it."""
    import bench
    csrc = tmp_path / "dequantisation_fp8q_token_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))

    def fp(text):
        (csrc / "k.cu").write_text(text)
        return bench.source_fingerprint(["k.cu"])

    base = fp("int f(int x) {\n    return x + 1;  // one more\n}\n")
    assert fp("/* a header */\nint f(int x) {\n  return x + 1;   // one more, said differently\n}\n") == base
    assert fp("int f(int x) {\n    return x + 2;  // one more\n}\n") != base
    assert fp("int f(int y) {\n    return y + 1;\n}\n") != base


def test_dominant_sample_steps():
    """The dominant op's event pairs in the timed region: about five, spread over the steps,
    never on the first timed step (which starts on an idle GPU) unless it is the only one."""
    import bench
    assert bench.dominant_sample_steps(1) == [0]
    assert bench.dominant_sample_steps(2) == [1]
    assert bench.dominant_sample_steps(5) == [1, 2, 3, 4]
    assert bench.dominant_sample_steps(20) == [3, 7, 11, 15, 19]
    assert bench.dominant_sample_steps(200) == [39, 79, 119, 159, 199]
    for k in range(2, 400):
        got = bench.dominant_sample_steps(k)
        assert 0 not in got and got and all(0 < s < k for s in got) and len(got) <= 9

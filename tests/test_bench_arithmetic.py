"""bench.py's byte and roofline arithmetic, on the CPU (no GPU, no library call).

The numbers these helpers produce go straight into the reported roofline fractions, so
they are pinned here against values fixed independently: the sizes of the workloads'
tensors, the im2col matrix size the tutorial page warns about (zskr §2.2: the X_col of a
K x K convolution holds K*K copies of the input), and plain arithmetic on the fields.
"""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from cnn_convolution_conv2d_b200 import workloads  # noqa: E402


def cfg(name, **kw):
    c = workloads.CONFIGS[name]
    return c.scaled(**kw) if kw else c


def test_step_bytes_are_the_tensors_once():
    c = cfg("pointwise1x1_bf16")
    x = 64 * 256 * 56 * 56 * 2
    w = 1024 * 256 * 2
    y = 64 * 1024 * 56 * 56 * 2
    assert bench.step_bytes(c) == x + w + 1024 * 2 + y == 514_328_576


def test_xcol_is_k_squared_copies_of_the_input_for_a_stride_1_same_conv():
    c = cfg("resnet3x3_bf16_nhwc")
    x_bytes = c.N * c.C_in * c.H * c.W * 2
    assert bench.xcol_bytes(c) == 9 * x_bytes          # 3x3, stride 1, pad 1: Ho = H
    assert abs(bench.xcol_bytes(c) / 1e6 - 924.8) < 0.1
    # the GEMM over X_col reads X_col and the packed weights, writes y (no bias)
    assert bench.explicit_kernel_bytes(c) == bench.xcol_bytes(c) + 2 * (256 * 9 * 256 + 64 * 256 * 56 * 56)


def test_main_kernel_bytes_follow_the_inputs_the_kernel_reads():
    stem = cfg("stem_bf16")                 # gather kernel: x read in place (NCHW); the packed
    assert bench.uses_gather(stem)          # weights it reads carry channels padded 3 -> 8
    assert bench.padded_channels(stem) == 8
    assert bench.main_kernel_bytes(stem) == bench.step_bytes(stem) + 64 * 49 * (8 - 3) * 2 == 61_064_320
    r3 = cfg("resnet3x3_bf16_nhwc")         # channels-last, 16-byte aligned: no copy
    assert not bench.uses_gather(r3)
    assert bench.main_kernel_bytes(r3) == bench.step_bytes(r3)
    r3n = r3.scaled(layout="nchw")          # NCHW: the kernel reads the channels-last copy (same size)
    assert bench.main_kernel_bytes(r3n) == bench.step_bytes(r3n)


PEAKS = {"hbm_gbs": 6544.7, "bf16_tflops": 1630.0, "bf16_tflops_sustained": 1371.8}


def test_roofline_picks_the_bound_by_the_ridge():
    r3 = cfg("resnet3x3_bf16_nhwc")         # 1145 FLOP/B: tensor-bound
    rl = bench.roofline(r3, 0.2, PEAKS, "measured", "none")
    assert rl["bound"] == "tensor" and rl["unit"] == "TFLOP/s" and rl["peak"] == 1371.8
    assert rl["achieved"] == pytest.approx(bench.flops(r3) / 0.2e-3 / 1e12)
    assert rl["frac"] == pytest.approx(rl["achieved"] / 1371.8)
    p1 = cfg("pointwise1x1_bf16")           # 205 FLOP/B: below the ridge, HBM-bound
    rl = bench.roofline(p1, 0.1, PEAKS, "measured", "none")
    assert rl["bound"] == "hbm" and rl["unit"] == "GB/s"
    assert rl["achieved"] == pytest.approx(514_328_576 / 0.1e-3 / 1e9)
    assert rl["traffic"] is None            # no committed counters for this name


def test_write_context_is_output_bytes_over_the_fill_rate():
    p1 = cfg("pointwise1x1_bf16")
    rl = bench.with_write_context(bench.roofline(p1, 0.137, PEAKS, "measured", "none"), p1, 0.137, 3850.0)
    wc = rl["write_context"]
    assert wc["output_bytes"] == 411_041_792
    assert wc["output_write_ms_at_fill_rate"] == pytest.approx(411_041_792 / 3850e9 * 1e3)
    assert wc["frac_of_write_bound"] == pytest.approx(wc["output_write_ms_at_fill_rate"] / 0.137)
    r3 = cfg("resnet3x3_bf16_nhwc")         # tensor-bound: no write context
    assert "write_context" not in bench.with_write_context(bench.roofline(r3, 0.2, PEAKS, "m", "x"), r3, 0.2, 1.0)


def test_fp32_above_the_tf32_ridge_is_tensor_bound_against_half_the_bf16_peak():
    k7 = cfg("k7_17x17_f32")                # 3379 FLOP/B, three TF32 products per multiply-add
    rl = bench.roofline(k7, 1.0, PEAKS, "measured", "none")
    assert rl["bound"] == "tensor" and rl["peak"] == pytest.approx(1371.8 * 0.5)
    assert rl["algorithmic_tflops"] == pytest.approx(bench.flops(k7) / 1e-3 / 1e12)
    assert rl["executed_tf32_tflops"] == pytest.approx(3 * rl["algorithmic_tflops"])
    assert rl["frac"] == pytest.approx(rl["executed_tf32_tflops"] / (1371.8 * 0.5))
    g = cfg("grouped_dilated_f32")          # 14 FLOP/B: memory-bound in any precision
    assert bench.roofline(g, 0.03, PEAKS, "measured", "none")["bound"] == "hbm"


def test_committed_traffic_is_void_when_the_kernel_source_changes(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.kernel_source_hash("igemm_kernel")
    entry = {"kernel": "igemm_kernel", "dram_bytes_read": 100.0, "dram_bytes_write": 20.0, "l2_write_bytes": 50.0}
    (prof / "traffic.json").write_text(json.dumps({
        "a": {**entry, "kernel_hash": good},
        "b": {**entry, "kernel_hash": "0" * 16},
        "c": {**entry, "kernel": "no_such_kernel", "kernel_hash": good},
        "d": {"kernel": "igemm_kernel", "kernel_hash": good, "dram_bytes_read": 1.0, "dram_bytes_write": 2.0},
        "e": {**entry, "kernel_hash": good, "dram_bytes_write": 80.0, "scale_to_full_launch": 2.0},
    }))
    csrc = os.path.join(ROOT, "cnn_convolution_conv2d_b200", "csrc")
    # read profiles from the temporary tree, kernel sources from the real one
    os.symlink(os.path.join(ROOT, "cnn_convolution_conv2d_b200"), tmp_path / "cnn_convolution_conv2d_b200")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.committed_traffic("a") == 150.0       # reads + the L2-side writes (above DRAM's count)
    assert bench.committed_traffic("b") is None
    assert bench.committed_traffic("c") is None
    assert bench.committed_traffic("d") is None        # no L2-side write count: not reported
    assert bench.committed_traffic("e") == 2.0 * 180.0  # DRAM writes above L2's, scaled to a full launch
    assert bench.committed_traffic("missing") is None
    assert os.path.isdir(csrc)

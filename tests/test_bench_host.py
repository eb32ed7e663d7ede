"""bench.py's workload arithmetic against independently worked figures.

The algorithmic GFLOP and minimum HBM bytes per launch below were worked out
from the workload definitions by hand (2*M*Cout*Cin*taps-that-read-a-frame;
x, w, bias, residual read once and y written once, 16-bit elements); they pin
the numbers every bench line divides by.
"""
import pytest

import bench
from seeded_inputs.workloads import WORKLOADS

# name: (algorithmic GFLOP, algorithmic MB, bound)
EXPECTED = {
    "cfg1": (0.2454, 0.71, "tensor"),   # 13 of 15 (frame, tap) pairs read a frame; nominal 0.283
    "cfg2": (521.8, 230.0, "tensor"),
    "cfg3": (1478.5, 228.1, "tensor"),
    "cfg4": (7015.8, 4061.0, "tensor"),
    "cfg5a": (130.5, 50.7, "tensor"),
    "cfg5b": (3826.8, 837.6, "tensor"),
    "cfg5c": (141.7, 830.7, "hbm"),
    "cfg5d": (77.3, 70.6, "tensor"),
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_algorithmic_work(name):
    gflop, mb, bound = EXPECTED[name]
    wl = WORKLOADS[name]
    assert bench.algorithmic_flops(wl) / 1e9 == pytest.approx(gflop, rel=2e-3, abs=2e-3)
    assert bench.algorithmic_bytes(wl) / 1e6 == pytest.approx(mb, rel=3e-3, abs=0.01)
    peaks = {"bf16_tflops": 1608.5, "hbm_gbs": 6545.0}
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    got = "tensor" if bench.algorithmic_flops(wl) / bench.algorithmic_bytes(wl) >= ridge else "hbm"
    assert got == bound


def test_nominal_counts_every_tap():
    assert bench.nominal_flops(WORKLOADS["cfg1"]) / 1e9 == pytest.approx(0.283, rel=2e-3)
    assert bench.nominal_flops(WORKLOADS["cfg2"]) == bench.algorithmic_flops(WORKLOADS["cfg2"])


def test_first_frame_counts_one_folded_tap():
    wl = WORKLOADS["cfg5d"]
    # nominal 3D work counts all three temporal taps of the single frame
    assert bench.nominal_flops(wl) == pytest.approx(3 * bench.algorithmic_flops(wl))


def test_zero_padding_taps_are_not_work():
    """cfg1: zero temporal padding 1 on 5 frames: 13 of the 15 (frame, tap) pairs read a frame."""
    wl = WORKLOADS["cfg1"]
    Do, Ho, Wo = bench.out_shape(wl)
    per_tap = 2.0 * wl.N * Ho * Wo * wl.Cout * wl.Cin * wl.kernel[1] * wl.kernel[2]
    assert bench.algorithmic_flops(wl) == pytest.approx(13 * per_tap)


def test_output_shapes():
    assert bench.out_shape(WORKLOADS["cfg2s"]) == (9, 128, 128)
    assert bench.out_shape(WORKLOADS["cfg1"]) == (5, 32, 32)
    assert bench.out_shape(WORKLOADS["cfg5d"]) == (1, 256, 256)


def test_backward_samples_cover_corners_and_stay_in_range():
    wl = WORKLOADS["cfg2"]
    for which in ("dgrad", "wgrad"):
        idx, total = bench._backward_samples(which, wl, 64, 3)
        assert idx.min() == 0 and idx.max() == total - 1
        assert len(set(idx.tolist())) == idx.size

"""CONV3D_LOG=1: every kernel launch reports the plan chosen for it on stderr.

The switch is read once per process, so each case runs in a fresh interpreter.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = """
import torch
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
x = si.tensor((1, 3, 8, 8, 64), 7, 0, 1.0, torch.bfloat16, "cuda")
w = si.tensor((64, 3, 3, 3, 64), 7, 1, (27 * 64) ** -0.5, torch.bfloat16, "cuda")
y = c3.conv3d(x, w)
dx = c3.conv3d_bwd_data(y, w, x.shape)
dw, db = c3.conv3d_bwd_weight(x, y, (3, 3, 3))
assert c3.poll_status() == c3.Status.OK
"""


def _run(log):
    env = dict(os.environ)
    env.pop("CONV3D_LOG", None)
    env["CONV3D_DGRAD_COMBINE"] = "1"   # this small case would take the fp32 front frames
    if log:
        env["CONV3D_LOG"] = "1"
    return subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_plan_log_reports_each_launch():
    r = _run(True)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stderr.splitlines() if l.startswith("libconv3d: ")]
    # forward, then the data gradient (its plan line and its one launch), then
    # the weight gradient
    assert any("implicit GEMM" in l and "16-bit output" in l for l in lines), lines
    # the data gradient: one launch whose frame-0 tiles also sum the 2 replicated copies
    assert any(l.startswith("libconv3d: data gradient: 3 frames x 1 samples in one launch, "
                            "frame 0 with its 2 replicated copies") for l in lines), lines
    assert sum("implicit GEMM" in l for l in lines) == 2, lines
    assert any(l.startswith("libconv3d: weight gradient") for l in lines), lines


def test_plan_log_is_silent_by_default():
    r = _run(False)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "libconv3d: " not in r.stderr


SPLIT_SCRIPT = """
import torch
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
# 3 frames of 80x80 in 128-pixel tiles, 64 channels: 150 tiles, i.e. one full
# round of 148 and a last round of 2 tiles, which the default rule splits
x = si.tensor((1, 3, 80, 80, 64), 7, 0, 1.0, torch.bfloat16, "cuda")
w = si.tensor((64, 3, 3, 3, 64), 7, 1, (27 * 64) ** -0.5, torch.bfloat16, "cuda")
y = c3.conv3d(x, w)
assert c3.poll_status() == c3.Status.OK
print(torch.cuda.get_device_properties(0).multi_processor_count)
"""


def test_plan_log_shows_the_tail_split():
    env = dict(os.environ)
    env["CONV3D_LOG"] = "1"
    env["CONV3D_SWAP"] = "0"     # the 128-pixel tiles (the transposed variant would make 75)
    env.pop("CONV3D_SPLIT", None)
    r = subprocess.run([sys.executable, "-c", SPLIT_SCRIPT], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    sms = int(r.stdout.split()[-1])
    lines = [l for l in r.stderr.splitlines() if "implicit GEMM" in l]
    assert len(lines) == 1, lines
    tail = 150 % sms
    if sms <= 150 and 0 < tail <= sms // 2:
        # 27 k-blocks a tile: pieces of at least 8 k-blocks, so 3 of them
        assert f"last {tail} tiles in 3 pieces" in lines[0], lines
    else:
        assert "in 1 pieces" in lines[0], lines


def test_plan_log_data_gradient_with_fp32_front_frames():
    """CONV3D_DGRAD_COMBINE=0: the data gradient writes the kt parts of frame 0
    in fp32 beside the 16-bit frames, then folds them."""
    env = dict(os.environ)
    env["CONV3D_LOG"] = "1"
    env["CONV3D_DGRAD_COMBINE"] = "0"
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stderr.splitlines() if l.startswith("libconv3d: ")]
    assert any("implicit GEMM" in l and "fp32 (front frames) and 16-bit output" in l
               for l in lines), lines
    assert any(l.startswith("libconv3d: data gradient: 3 front frames") for l in lines), lines


ROUNDS_SCRIPT = """
import sys
import torch
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
sms = torch.cuda.get_device_properties(0).multi_processor_count
rounds, extra = int(sys.argv[1]), int(sys.argv[2])
# 2 frames of H x 128 pixels in 128-pixel tiles, 64 channels (one channel tile):
# rounds * sms + extra tiles in all
tiles = rounds * sms + extra
H = tiles // 2
x = si.tensor((1, 2, H, 128, 64), 9, 0, 1.0, torch.bfloat16, "cuda")
w = si.tensor((64, 3, 3, 3, 64), 9, 1, (27 * 64) ** -0.5, torch.bfloat16, "cuda")
y = c3.conv3d(x, w)
assert c3.poll_status() == c3.Status.OK
print(tiles)
"""


@pytest.mark.parametrize("rounds,split", [(15, True), (16, False)])
def test_tail_split_only_below_sixteen_rounds(rounds, split):
    """A short last round (10 tiles) is split along K when the launch has fewer
    than 16 rounds of tiles, and left whole from 16 rounds up."""
    env = dict(os.environ)
    env["CONV3D_LOG"] = "1"
    env["CONV3D_SWAP"] = "0"
    env.pop("CONV3D_SPLIT", None)
    r = subprocess.run([sys.executable, "-c", ROUNDS_SCRIPT, str(rounds), "10"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    tiles = int(r.stdout.split()[-1])
    lines = [l for l in r.stderr.splitlines() if "implicit GEMM" in l]
    assert len(lines) == 1 and f"{tiles} tiles" in lines[0], lines
    if split:
        assert "last 10 tiles in 3 pieces" in lines[0], lines   # 27 k-blocks: pieces of >= 8
    else:
        assert "in 1 pieces" in lines[0], lines


COMBINE_SCRIPT = """
import sys
import torch
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
H = int(sys.argv[1])
shape = (1, 4, H, 128, 64)
w = si.tensor((64, 3, 3, 3, 64), 9, 1, (27 * 64) ** -0.5, torch.bfloat16, "cuda")
dy = si.tensor(shape, 9, 2, 1.0, torch.bfloat16, "cuda")
dx = c3.conv3d_bwd_data(dy, w, shape, (0, 1, 1), c3.TPAD_CAUSAL_REPLICATE)
assert c3.poll_status() == c3.Status.OK
print(torch.cuda.get_device_properties(0).multi_processor_count)
"""


@pytest.mark.parametrize("many", [True, False])
def test_data_gradient_front_rule(many):
    """By default the data gradient combines frame 0 with its replicated
    copies from 4 rounds of tiles up, and takes the fp32 front frames and the
    fold below that."""
    env = dict(os.environ)
    env["CONV3D_LOG"] = "1"
    env.pop("CONV3D_DGRAD_COMBINE", None)
    env.pop("CONV3D_SWAP", None)
    # 4 frames of H x 128 pixels, 64 channels: the transposed variant's
    # 256-pixel tiles give 4 * H / 2 tiles (H = 296: 592 = 4 rounds of 148)
    H = 296 if many else 8
    r = subprocess.run([sys.executable, "-c", COMBINE_SCRIPT, str(H)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    sms = int(r.stdout.split()[-1])
    lines = [l for l in r.stderr.splitlines() if l.startswith("libconv3d: data gradient")]
    assert len(lines) == 1, r.stderr[-2000:]
    if many and sms <= 148:
        assert "frame 0 with its 2 replicated copies" in lines[0], lines
    elif not many:
        assert "front frames and" in lines[0], lines

"""conv3d_kernel_launches(): the library's own count of the GPU kernels it
launched, which the benchmark reads around its timed region.  Each call below
enqueues a known set of the library's kernels; the counter must rise by
exactly that many (torch's own allocations and clears are not counted)."""
import pytest
import torch

import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3

pytestmark = pytest.mark.gpu

ZERO, CREP = c3.TPAD_ZERO, c3.TPAD_CAUSAL_REPLICATE


def _delta(fn):
    torch.cuda.synchronize()
    before = c3.kernel_launches()
    fn()
    assert c3.poll_status() == c3.Status.OK
    return c3.kernel_launches() - before


def _t(shape, stream, scale=1.0):
    return si.tensor(shape, 71, stream, scale, torch.bfloat16, "cuda")


def test_forward_launches():
    x = _t((1, 4, 16, 16, 64), 0)
    w = _t((64, 3, 3, 3, 64), 1, (27 * 64) ** -0.5)
    assert _delta(lambda: c3.conv3d(x, w, pad=(0, 1, 1), tpad=CREP)) == 1      # one main kernel
    x1 = _t((1, 1, 16, 16, 64), 2)
    assert _delta(lambda: c3.conv3d(x1, w, pad=(0, 1, 1), tpad=CREP)) == 2     # fold + main kernel


@pytest.mark.parametrize("combine,expect", [("1", 2), ("0", 3)])
def test_data_gradient_launches(combine, expect, monkeypatch):
    """Weight transform + one launch over every frame (+ the fold of frame 0's
    fp32 parts when they are not combined in the accumulator)."""
    monkeypatch.setenv("CONV3D_DGRAD_COMBINE", combine)
    w = _t((64, 3, 3, 3, 64), 1, (27 * 64) ** -0.5)
    dy = _t((1, 4, 16, 16, 64), 3)
    assert _delta(lambda: c3.conv3d_bwd_data(dy, w, (1, 4, 16, 16, 64), (0, 1, 1), CREP)) == expect
    dyz = _t((1, 4, 16, 16, 64), 4)
    assert _delta(lambda: c3.conv3d_bwd_data(dyz, w, (1, 4, 16, 16, 64), (1, 1, 1), ZERO)) == 2


def test_groupnorm_launches():
    x = _t((1, 2, 16, 16, 64), 5)
    stats = [None]

    def st():
        stats[0] = c3.groupnorm_stats(x, 32)
    assert _delta(st) == 2                                   # statistics + finalize
    assert _delta(lambda: c3.groupnorm_silu(x, stats[0], groups=32)) == 1


def test_weight_gradient_launches():
    x = _t((1, 4, 16, 16, 64), 6)
    dy = _t((1, 4, 16, 16, 64), 7)
    n = _delta(lambda: c3.conv3d_bwd_weight(x, dy, (3, 3, 3), pad=(0, 1, 1), tpad=CREP))
    assert 3 <= n <= 5, n    # clear, kernel, rounding (dw, then db), bias pass beside or after

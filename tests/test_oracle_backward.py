"""Pins for the oracle's backward pass (dx, dw, dbias of the convolution).

The adjoint identities tie the backward loops to the forward oracle, which is
pinned separately: for any upstream gradient g,
    <conv(x, w), g> = <x, dx(g)>,   <conv(x, w), g> = <w, dw(x, g)>,
    dbias = sum of g over pixels,
and torch.autograd in float64 (with the padding written as explicit ops)
checks the same gradients with a library routine.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import seeded_inputs as si

BF16 = oracle.BF16
ZERO, CREP, CZERO = oracle.TPAD_ZERO, oracle.TPAD_CAUSAL_REPLICATE, oracle.TPAD_CAUSAL_ZERO


HERE = os.path.dirname(os.path.abspath(__file__))


def dec(b):
    return oracle.decode16(b, BF16)


def bf16_bits(a):
    """float64 array -> bf16 bit patterns (values chosen exactly representable)."""
    t = torch.from_numpy(np.asarray(a, dtype=np.float64)).to(torch.float32).to(torch.bfloat16)
    return si.bits(t)


def test_golden_box_sum_backward():
    """Hand-worked adjoints of the all-ones 3x3x3 kernel on a 2-frame 3x3 clip
    (tests/golden/box_sum_backward.txt), in all three temporal padding modes."""
    rows = []
    with open(os.path.join(HERE, "golden", "box_sum_backward.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                mode, which, a, b, c, v = line.split()
                rows.append((int(mode), which, int(a), int(b), int(c), float(v)))
    assert len(rows) == 3 * (18 + 27 + 1)
    frame0 = np.arange(1, 10, dtype=np.float64).reshape(3, 3)
    x = np.stack([frame0, 10 * frame0]).reshape(1, 2, 3, 3, 1)
    w = np.ones((1, 3, 3, 3, 1))
    dy = np.stack([np.ones((3, 3)), 2 * np.ones((3, 3))]).reshape(1, 2, 3, 3, 1)
    for mode in (ZERO, CREP, CZERO):
        pad = (1, 1, 1) if mode == ZERO else (0, 1, 1)
        dx, dw, db = oracle.conv3d_backward(bf16_bits(x), bf16_bits(w), bf16_bits(dy), BF16,
                                            (3, 3, 3), (1, 1, 1), pad, mode)
        seen = 0
        for m, which, a, b, c, expect in rows:
            if m != mode:
                continue
            got = {"dx": lambda: dx[0, a, b, c, 0], "dw": lambda: dw[0, a, b, c, 0],
                   "db": lambda: db[0]}[which]()
            assert got == expect, (mode, which, a, b, c, got, expect)
            seen += 1
        assert seen == 46


def problem(N, Cin, D, H, W, Cout, k, stride, pad, tpad, seed):
    fan = Cin * k[0] * k[1] * k[2]
    xb = si.bits(si.tensor((N, D, H, W, Cin), seed, 0))
    wb = si.bits(si.tensor((Cout, *k, Cin), seed, 1, fan ** -0.5))
    out = oracle.output_shape(D, H, W, k, stride, pad, tpad)
    gb = si.bits(si.tensor((N, *out, Cout), seed, 5))
    return xb, wb, gb


CASES = [
    ((2, 3, 4, 5, 6, 4), (3, 3, 3), (1, 1, 1), (1, 1, 1), ZERO),
    ((1, 4, 5, 4, 4, 3), (3, 3, 3), (1, 1, 1), (0, 1, 1), CREP),
    ((1, 4, 5, 4, 4, 3), (3, 3, 3), (1, 1, 1), (0, 1, 1), CZERO),
    ((2, 2, 6, 5, 7, 3), (3, 3, 3), (2, 2, 2), (0, 1, 1), CREP),
    ((1, 3, 3, 6, 6, 2), (2, 3, 1), (1, 2, 1), (0, 0, 2), CZERO),
    ((1, 5, 2, 3, 3, 4), (1, 1, 1), (1, 1, 1), (0, 0, 0), ZERO),
]


@pytest.mark.parametrize("case", CASES)
def test_adjoint_identities(case):
    (N, Cin, D, H, W, Cout), k, stride, pad, tpad = case
    xb, wb, gb = problem(N, Cin, D, H, W, Cout, k, stride, pad, tpad, seed=3)
    y = oracle.conv3d(xb, wb, None, None, BF16, k, stride, pad, tpad)
    dx, dw, db = oracle.conv3d_backward(xb, wb, gb, BF16, k, stride, pad, tpad)
    g = dec(gb)
    lhs = float(np.sum(y * g))
    assert np.isclose(lhs, float(np.sum(dec(xb) * dx)), rtol=1e-12, atol=1e-12)
    assert np.isclose(lhs, float(np.sum(dec(wb) * dw)), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db, g.reshape(-1, Cout).sum(axis=0), rtol=1e-12, atol=1e-12)


def torch_grads(xd, wd, gd, k, stride, pad, tpad):
    x = torch.from_numpy(xd).permute(0, 4, 1, 2, 3).requires_grad_(True)
    w = torch.from_numpy(wd).permute(0, 4, 1, 2, 3).requires_grad_(True)
    kt = k[0]
    if tpad == ZERO:
        xp = F.pad(x, (0, 0, 0, 0, pad[0], pad[0]))
    elif tpad == CREP:
        xp = torch.cat([x[:, :, :1]] * (kt - 1) + [x], dim=2)
    else:
        xp = F.pad(x, (0, 0, 0, 0, kt - 1, 0))
    y = F.conv3d(xp, w, stride=stride, padding=(0, pad[1], pad[2]))
    y.backward(torch.from_numpy(gd).permute(0, 4, 1, 2, 3))
    return (x.grad.permute(0, 2, 3, 4, 1).numpy(), w.grad.permute(0, 2, 3, 4, 1).numpy())


@pytest.mark.parametrize("case", CASES)
def test_matches_torch_autograd_float64(case):
    (N, Cin, D, H, W, Cout), k, stride, pad, tpad = case
    xb, wb, gb = problem(N, Cin, D, H, W, Cout, k, stride, pad, tpad, seed=5)
    dx, dw, _ = oracle.conv3d_backward(xb, wb, gb, BF16, k, stride, pad, tpad)
    tdx, tdw = torch_grads(dec(xb), dec(wb), dec(gb), k, stride, pad, tpad)
    np.testing.assert_allclose(dx, tdx, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(dw, tdw, rtol=1e-10, atol=1e-10)


def test_causal_replicate_sends_front_gradients_to_frame_zero():
    """With causal replicate padding, dx of frame 0 = dx of the explicitly
    extended clip summed over frame 0 and its kt-1 copies (the adjoint of
    copying frame 0)."""
    N, Cin, D, H, W, Cout, k = 1, 3, 4, 4, 5, 2, (3, 3, 3)
    xb, wb, gb = problem(N, Cin, D, H, W, Cout, k, (1, 1, 1), (0, 1, 1), CREP, seed=7)
    dx, _, _ = oracle.conv3d_backward(xb, wb, gb, BF16, k, (1, 1, 1), (0, 1, 1), CREP)
    ext = np.concatenate([xb[:, :1]] * 2 + [xb], axis=1)
    # the extended clip under zero padding with pt = 0 has the same D output frames
    assert oracle.output_shape(D + 2, H, W, k, (1, 1, 1), (0, 1, 1), ZERO)[0] == D
    dxe, _, _ = oracle.conv3d_backward(ext, wb, gb, BF16, k, (1, 1, 1), (0, 1, 1), ZERO)
    np.testing.assert_allclose(dx[:, 0], dxe[:, :3].sum(axis=1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dx[:, 1:], dxe[:, 3:], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("case", CASES)
def test_elementwise_adjoints_match_torch_autograd(case):
    """The per-element gather forms (used at sizes the serial scatter cannot
    finish) against float64 autograd, on every element, and against the
    scatter form."""
    (N, Cin, D, H, W, Cout), k, stride, pad, tpad = case
    xb, wb, gb = problem(N, Cin, D, H, W, Cout, k, stride, pad, tpad, seed=11)
    tdx, tdw = torch_grads(dec(xb), dec(wb), dec(gb), k, stride, pad, tpad)
    pixels = np.arange(N * D * H * W)
    dx = oracle.conv3d_dx_at(wb, gb, BF16, xb.shape, k, stride, pad, tpad, pixels)
    np.testing.assert_allclose(dx, tdx.reshape(-1, Cin), rtol=1e-10, atol=1e-10)
    entries = np.arange(wb.size)[::-1].copy()          # any order
    dw = oracle.conv3d_dw_at(xb, gb, BF16, Cout, k, stride, pad, tpad, entries)
    np.testing.assert_allclose(dw, tdw.reshape(-1)[entries], rtol=1e-10, atol=1e-10)
    sdx, sdw, _ = oracle.conv3d_backward(xb, wb, gb, BF16, k, stride, pad, tpad)
    np.testing.assert_allclose(dx, sdx.reshape(-1, Cin), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dw, sdw.reshape(-1)[entries], rtol=1e-12, atol=1e-12)


def test_elementwise_adjoints_reject_bad_indices():
    xb, wb, gb = problem(1, 2, 3, 4, 4, 2, (3, 3, 3), (1, 1, 1), (1, 1, 1), ZERO, seed=1)
    with pytest.raises(ValueError):
        oracle.conv3d_dx_at(wb, gb, BF16, xb.shape, (3, 3, 3), (1, 1, 1), (1, 1, 1), ZERO,
                            [1 * 3 * 4 * 4])
    with pytest.raises(ValueError):
        oracle.conv3d_dw_at(xb, gb, BF16, 2, (3, 3, 3), (1, 1, 1), (1, 1, 1), ZERO, [-1])


# ---------------------------------------------------------------- cached-frames chunk mode

CACHED = oracle.TPAD_CAUSAL_CACHED

CACHED_CASES = [
    ((2, 3, 4, 5, 6, 4), (3, 3, 3), (1, 1, 1), (0, 1, 1)),
    ((1, 4, 3, 4, 4, 3), (3, 3, 3), (2, 2, 2), (0, 1, 1)),
    ((1, 3, 5, 6, 5, 2), (2, 3, 1), (1, 2, 1), (0, 0, 2)),
    ((1, 2, 1, 4, 4, 3), (3, 1, 3), (1, 1, 1), (0, 0, 1)),      # a one-frame chunk
]


def cached_problem(N, Cin, D, H, W, Cout, k, stride, pad, seed):
    fan = Cin * k[0] * k[1] * k[2]
    xb = si.bits(si.tensor((N, D, H, W, Cin), seed, 0))
    pb = si.bits(si.tensor((N, k[0] - 1, H, W, Cin), seed, 4))
    wb = si.bits(si.tensor((Cout, *k, Cin), seed, 1, fan ** -0.5))
    out = oracle.output_shape(D, H, W, k, stride, pad, CACHED)
    gb = si.bits(si.tensor((N, *out, Cout), seed, 5))
    return xb, pb, wb, gb


@pytest.mark.parametrize("case", CACHED_CASES)
def test_cached_backward_is_the_backward_of_the_joined_clip(case):
    """The chunk convolution is the plain convolution (zero padding, pt = 0) of
    the clip [prev; x]; its adjoints are those of the joined clip, split at
    frame kt-1 -- against the separately pinned backward, bit for bit (same
    products, same order)."""
    (N, Cin, D, H, W, Cout), k, stride, pad = case
    xb, pb, wb, gb = cached_problem(N, Cin, D, H, W, Cout, k, stride, pad, seed=13)
    joined = np.concatenate([pb, xb], axis=1)
    assert oracle.output_shape(D + k[0] - 1, H, W, k, stride, pad, ZERO) == \
        oracle.output_shape(D, H, W, k, stride, pad, CACHED)
    dx, dprev, dw, db = oracle.conv3d_backward_cached(xb, pb, wb, gb, BF16, k, stride, pad)
    jdx, jdw, jdb = oracle.conv3d_backward(joined, wb, gb, BF16, k, stride, pad, ZERO)
    np.testing.assert_array_equal(dprev, jdx[:, :k[0] - 1])
    np.testing.assert_array_equal(dx, jdx[:, k[0] - 1:])
    np.testing.assert_array_equal(dw, jdw)
    np.testing.assert_array_equal(db, jdb)


@pytest.mark.parametrize("case", CACHED_CASES)
def test_cached_backward_adjoint_identities(case):
    (N, Cin, D, H, W, Cout), k, stride, pad = case
    xb, pb, wb, gb = cached_problem(N, Cin, D, H, W, Cout, k, stride, pad, seed=17)
    y = oracle.conv3d(xb, wb, None, None, BF16, k, stride, pad, CACHED, prev_bits=pb)
    dx, dprev, dw, db = oracle.conv3d_backward_cached(xb, pb, wb, gb, BF16, k, stride, pad)
    g = dec(gb)
    lhs = float(np.sum(y * g))
    assert np.isclose(lhs, float(np.sum(dec(xb) * dx) + np.sum(dec(pb) * dprev)),
                      rtol=1e-12, atol=1e-12)
    assert np.isclose(lhs, float(np.sum(dec(wb) * dw)), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db, g.reshape(-1, Cout).sum(axis=0), rtol=1e-12, atol=1e-12)


def test_cached_backward_matches_torch_autograd_float64():
    (N, Cin, D, H, W, Cout), k, stride, pad = CACHED_CASES[0]
    xb, pb, wb, gb = cached_problem(N, Cin, D, H, W, Cout, k, stride, pad, seed=19)
    dx, dprev, dw, _ = oracle.conv3d_backward_cached(xb, pb, wb, gb, BF16, k, stride, pad)
    x = torch.from_numpy(dec(xb)).permute(0, 4, 1, 2, 3).requires_grad_(True)
    pv = torch.from_numpy(dec(pb)).permute(0, 4, 1, 2, 3).requires_grad_(True)
    w = torch.from_numpy(dec(wb)).permute(0, 4, 1, 2, 3).requires_grad_(True)
    y = F.conv3d(torch.cat([pv, x], dim=2), w, stride=stride, padding=(0, pad[1], pad[2]))
    y.backward(torch.from_numpy(dec(gb)).permute(0, 4, 1, 2, 3))
    np.testing.assert_allclose(dx, x.grad.permute(0, 2, 3, 4, 1).numpy(), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(dprev, pv.grad.permute(0, 2, 3, 4, 1).numpy(), rtol=1e-10,
                               atol=1e-10)
    np.testing.assert_allclose(dw, w.grad.permute(0, 2, 3, 4, 1).numpy(), rtol=1e-10, atol=1e-10)

"""conv3d_fwd_gn: GroupNorm + SiLU applied in the convolution's operand path.

The reference is the decoder block as the pages' pipeline runs it, composed
from the pinned oracle functions: h = silu(GroupNorm(x)) in fp64, rounded
once to the activation dtype (the value an unfused pipeline stores), then the
fp64 convolution of h with the bias and residual.  Every output element is
compared.  The fused call must also equal, bit for bit, the unfused pipeline
of the library itself (conv3d_groupnorm_silu, then conv3d_fwd without its tail
split): both feed the same 16-bit h to the same MMAs in the same order.
"""
import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from parity import assert_close

pytestmark = pytest.mark.gpu

ZERO, CREP, CZERO = c3.TPAD_ZERO, c3.TPAD_CAUSAL_REPLICATE, c3.TPAD_CAUSAL_ZERO
TD = {"bf16": torch.bfloat16, "f16": torch.float16}
OD = {"bf16": oracle.BF16, "f16": oracle.F16}


def make(N, Cin, D, H, W, Cout, kernel, seed, dtype, residual, mean=0.3, std=1.7):
    td = TD[dtype]
    x = (si.tensor((N, D, H, W, Cin), seed, 0, std, torch.float32, "cuda") + mean).to(td)
    fan = Cin * kernel[0] * kernel[1] * kernel[2]
    w = si.tensor((Cout, *kernel, Cin), seed, 1, fan ** -0.5, td, "cuda")
    b = si.tensor((Cout,), seed, 2, 0.1, td, "cuda")
    gamma = (si.tensor((Cin,), seed, 6, 0.2, torch.float32, "cuda") + 1.0).to(td)
    beta = si.tensor((Cin,), seed, 7, 0.2, td, "cuda")
    return x, w, b, gamma, beta


def reference(x, w, b, r, gamma, beta, G, pf, silu, kernel, stride, pad, tpad, dtype):
    h = oracle.groupnorm_silu(si.bits(x), si.bits(gamma), si.bits(beta), OD[dtype], G,
                              eps=1e-6, per_frame=pf, silu=silu)
    hb = si.bits(torch.from_numpy(h).to(TD[dtype]))            # one rounding, as stored
    return oracle.conv3d(hb, si.bits(w), si.bits(b), None if r is None else si.bits(r),
                         OD[dtype], kernel, stride, pad, tpad)


CASES = [
    # N, Cin, D, H, W, Cout, kernel, pad, tpad, dtype, groups, per_frame, silu, residual, swap
    (1, 64, 3, 9, 13, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16", 8, False, True, True, "0"),
    (2, 64, 3, 9, 13, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16", 8, True, True, False, "0"),
    (1, 128, 4, 20, 19, 96, (3, 3, 3), (0, 1, 1), CZERO, "bf16", 32, False, True, False, "0"),
    (1, 32, 5, 16, 16, 32, (3, 3, 3), (1, 1, 1), ZERO, "f16", 8, False, True, False, "0"),
    (1, 40, 3, 12, 12, 264, (3, 3, 3), (1, 1, 1), ZERO, "bf16", 10, False, False, True, "0"),
    (1, 64, 3, 16, 20, 128, (3, 3, 3), (0, 1, 1), CREP, "bf16", 16, True, True, True, "1"),
    (1, 256, 2, 16, 16, 128, (1, 1, 1), (0, 0, 0), ZERO, "bf16", 32, False, True, False, "1"),
    (1, 64, 1, 24, 24, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16", 32, False, True, True, "0"),
    (1, 192, 2, 11, 23, 200, (3, 3, 3), (0, 2, 0), CREP, "f16", 16, True, True, True, "0"),
]


@pytest.mark.parametrize("case", CASES)
def test_fused_groupnorm_conv_every_element(case, monkeypatch):
    N, Cin, D, H, W, Cout, k, pad, tpad, dt, G, pf, silu, res, swap = case
    monkeypatch.setenv("CONV3D_SWAP", swap)
    stride = (1, 1, 1)
    x, w, b, gamma, beta = make(N, Cin, D, H, W, Cout, k, 60 + Cin, dt, res)
    out = c3.output_shape(D, H, W, k, stride, pad, tpad)
    r = si.tensor((N, *out, Cout), 61, 3, 1.0, TD[dt], "cuda") if res else None
    stats = c3.groupnorm_stats(x, G, eps=1e-6, per_frame=pf)
    y = c3.conv3d_gn(x, stats, gamma, beta, w, b, r, groups=G, per_frame=pf, apply_silu=silu,
                     stride=stride, pad=pad, tpad=tpad)
    assert c3.poll_status() == c3.Status.OK
    ref = reference(x, w, b, r, gamma, beta, G, pf, silu, k, stride, pad, tpad, dt)
    assert_close(y.double().cpu().numpy(), ref, str(case))
    # the library's own unfused pipeline gives the same bits (its convolution
    # without the tail split, which the GroupNorm instances do not have)
    monkeypatch.setenv("CONV3D_SPLIT", "0")
    h = c3.groupnorm_silu(x, stats, gamma, beta, groups=G, per_frame=pf, apply_silu=silu)
    y2 = torch.empty_like(y)
    c3.conv3d_fwd(h, w, b, r, y2, stride, pad, tpad)
    assert c3.poll_status() == c3.Status.OK
    assert torch.equal(y, y2)


def test_fused_groupnorm_does_not_split(monkeypatch):
    # the GroupNorm instances have no tail split; a forced split is ignored
    monkeypatch.setenv("CONV3D_SPLIT", "3")
    x, w, b, gamma, beta = make(1, 64, 3, 9, 13, 64, (3, 3, 3), 71, "bf16", False)
    stats = c3.groupnorm_stats(x, 8, eps=1e-6)
    y = c3.conv3d_gn(x, stats, gamma, beta, w, b, groups=8)
    assert c3.poll_status() == c3.Status.OK
    ref = reference(x, w, b, None, gamma, beta, 8, False, True, (3, 3, 3), (1, 1, 1), (0, 1, 1),
                    CREP, "bf16")
    assert_close(y.double().cpu().numpy(), ref, "fused, split requested")


OUT_CASES = [
    # N, Cin, D, H, W, Cout, kernel, pad, tpad, out_groups, swap, split, in_gn
    (2, 64, 3, 9, 13, 64, (3, 3, 3), (0, 1, 1), CREP, 8, "0", "", True),
    (1, 64, 3, 16, 20, 128, (3, 3, 3), (0, 1, 1), CREP, 32, "1", "", False),
    (1, 40, 3, 12, 12, 264, (3, 3, 3), (1, 1, 1), ZERO, 33, "0", "", False),   # 8 channels a group
    (1, 64, 3, 9, 13, 64, (3, 3, 3), (0, 1, 1), CREP, 64, "0", "3", True),     # 1 channel a group
    (1, 256, 2, 16, 16, 128, (1, 1, 1), (0, 0, 0), ZERO, 4, "1", "", False),   # 32 channels a group
]


@pytest.mark.parametrize("case", OUT_CASES)
def test_output_statistics_gathered_by_the_epilogue(case, monkeypatch):
    N, Cin, D, H, W, Cout, k, pad, tpad, G, swap, split, in_gn = case
    monkeypatch.setenv("CONV3D_SWAP", swap)
    if split:
        monkeypatch.setenv("CONV3D_SPLIT", split)
    x, w, b, gamma, beta = make(N, Cin, D, H, W, Cout, k, 80 + G, "bf16", False)
    stats = c3.groupnorm_stats(x, 8, eps=1e-6) if in_gn else None
    y, ys = c3.conv3d_gn(x, stats, gamma if in_gn else None, beta if in_gn else None, w, b,
                         groups=8, pad=pad, tpad=tpad, out_groups=G, out_eps=1e-5)
    assert c3.poll_status() == c3.Status.OK
    # the definition over the stored (rounded) y, in fp64
    yd = oracle.decode16(si.bits(y), oracle.BF16).reshape(N, -1, G, Cout // G)
    mu = yd.mean(axis=(1, 3))
    var = yd.var(axis=(1, 3))
    got = ys.cpu().numpy()
    np.testing.assert_allclose(got[..., 0], mu, rtol=0, atol=1e-5 * np.sqrt(var).max())
    np.testing.assert_allclose(got[..., 1], 1.0 / np.sqrt(var + 1e-5), rtol=1e-4)
    # and the library's statistics pass over y
    ref = c3.groupnorm_stats(y, G, eps=1e-5).cpu().numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-6)

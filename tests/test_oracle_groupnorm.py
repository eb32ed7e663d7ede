"""Pins for the oracle's GroupNorm + SiLU (the normalisation and activation in
front of each decoder convolution: stable-diffusion.cpp discussion "Exe Heavy
Metal", GROUP_NORM; news.bugfactory.tech, fused GroupNorm + SiLU kernel)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import seeded_inputs as si

BF16 = oracle.BF16


def rand_x(shape, seed, mean=0.0, std=1.0):
    t = si.tensor(shape, seed, 0, std) + mean
    return si.bits(t.to(torch.bfloat16))


def dec(bits):
    return oracle.decode16(bits, BF16)


@pytest.mark.parametrize("groups", [1, 4, 8])
@pytest.mark.parametrize("per_frame", [False, True])
def test_matches_torch_group_norm_and_silu(groups, per_frame):
    N, D, H, W, C = 2, 3, 4, 5, 16
    xb = rand_x((N, D, H, W, C), 3, mean=0.5, std=2.0)
    gb = si.bits(si.tensor((C,), 3, 1, 0.5) + 1.0)
    bb = si.bits(si.tensor((C,), 3, 2, 0.3))
    y = oracle.groupnorm_silu(xb, gb, bb, BF16, groups, eps=1e-6, per_frame=per_frame)
    x = torch.from_numpy(dec(xb))                       # N D H W C
    if per_frame:
        xt = x.reshape(N * D, H, W, C).permute(0, 3, 1, 2)       # (N*D) C H W
    else:
        xt = x.permute(0, 4, 1, 2, 3)                            # N C D H W
    z = F.group_norm(xt, groups, torch.from_numpy(dec(gb)), torch.from_numpy(dec(bb)), eps=1e-6)
    ref = F.silu(z)
    ref = (ref.permute(0, 2, 3, 1).reshape(N, D, H, W, C) if per_frame
           else ref.permute(0, 2, 3, 4, 1))
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-10, atol=1e-10)


def test_normalised_groups_have_zero_mean_unit_variance():
    N, D, H, W, C, G = 1, 2, 6, 6, 12, 3
    xb = rand_x((N, D, H, W, C), 5, mean=3.0, std=0.7)
    z = oracle.groupnorm_silu(xb, None, None, BF16, G, eps=0.0, silu=False)
    zg = z.reshape(-1, G, C // G)
    assert np.allclose(zg.mean(axis=(0, 2)), 0.0, atol=1e-12)
    assert np.allclose(zg.var(axis=(0, 2)), 1.0, atol=1e-12)


def test_constant_group_gives_beta_then_silu():
    """Zero variance: every element normalises to 0, so z = beta and y = silu(beta)."""
    N, D, H, W, C = 1, 2, 3, 3, 4
    xb = si.bits(torch.full((N, D, H, W, C), 1.75, dtype=torch.bfloat16))
    bb = si.bits(torch.tensor([0.5, -1.0, 2.0, 0.0], dtype=torch.bfloat16))
    y = oracle.groupnorm_silu(xb, None, bb, BF16, 2, eps=1e-5)
    beta = dec(bb)
    expect = beta / (1.0 + np.exp(-beta))
    assert np.allclose(y, np.broadcast_to(expect, y.shape), rtol=0, atol=1e-15)


def test_silu_closed_form_points():
    """SiLU(0) = 0, SiLU(z) - SiLU(-z) = z (odd part is the identity)."""
    N, D, H, W, C = 1, 1, 2, 2, 2
    xb = si.bits(torch.tensor([-1.0, 1.0] * 4, dtype=torch.bfloat16).reshape(N, D, H, W, C))
    z = oracle.groupnorm_silu(xb, None, None, BF16, 1, eps=0.0, silu=False)
    y = oracle.groupnorm_silu(xb, None, None, BF16, 1, eps=0.0, silu=True)
    # the two channels normalise to -1 and +1
    assert np.allclose(z[..., 0], -1.0) and np.allclose(z[..., 1], 1.0)
    assert np.allclose(y[..., 1] - y[..., 0], 1.0, atol=1e-15)


def test_rejects_channel_count_not_divisible():
    xb = rand_x((1, 1, 2, 2, 6), 1)
    with pytest.raises(ValueError):
        oracle.groupnorm_silu(xb, None, None, BF16, 4)

"""GPU GroupNorm (+ SiLU) against the fp64 oracle (parity tolerance of the
convolution: max|err| <= 1e-2 max|ref|, relative L1 <= 2e-3)."""
import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from parity import assert_close

pytestmark = pytest.mark.gpu

DT = {"bf16": (torch.bfloat16, oracle.BF16), "f16": (torch.float16, oracle.F16)}


def make(shape, seed, dtype, mean=0.0, std=1.0):
    td, _ = DT[dtype]
    C = shape[-1]
    x = (si.tensor(shape, seed, 0, std, torch.float32, "cuda") + mean).to(td)
    gamma = (si.tensor((C,), seed, 1, 0.2, torch.float32, "cuda") + 1.0).to(td)
    beta = si.tensor((C,), seed, 2, 0.2, td, "cuda")
    return x, gamma, beta


CASES = [
    # shape, groups, per_frame, dtype, mean, std
    ((2, 3, 9, 13, 64), 8, False, "bf16", 0.0, 1.0),
    ((2, 3, 9, 13, 64), 8, True, "bf16", 0.5, 2.0),
    ((1, 4, 7, 6, 96), 32, False, "bf16", -1.0, 0.5),    # 3 channels per group: vectors span groups
    ((1, 2, 16, 16, 256), 32, True, "f16", 0.0, 1.0),
    ((1, 5, 11, 3, 40), 5, False, "f16", 3.0, 0.7),      # mean large against the spread
    ((1, 2, 33, 47, 512), 32, False, "bf16", 0.0, 1.0),  # many chunks per set
]


@pytest.mark.parametrize("silu_form", ["tanh", "exp"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{'x'.join(map(str, c[0]))}-g{c[1]}-pf{int(c[2])}-{c[3]}")
def test_groupnorm_silu_every_element(case, silu_form, monkeypatch):
    # the default one-special-function SiLU (tanh) and the exp/division form
    monkeypatch.setenv("CONV3D_GN_SILU", silu_form)
    shape, G, pf, dt, mean, std = case
    x, gamma, beta = make(shape, 7, dt, mean, std)
    stats = c3.groupnorm_stats(x, G, eps=1e-6, per_frame=pf)
    y = c3.groupnorm_silu(x, stats, gamma, beta, groups=G, per_frame=pf)
    torch.cuda.synchronize()
    _, od = DT[dt]
    ref = oracle.groupnorm_silu(si.bits(x), si.bits(gamma), si.bits(beta), od, G, eps=1e-6,
                                per_frame=pf)
    assert_close(y.double().cpu().numpy(), ref, str(case))


def test_statistics_match_the_definition():
    x, _, _ = make((2, 3, 10, 12, 64), 9, "bf16", 0.25, 1.5)
    stats = c3.groupnorm_stats(x, 16, eps=1e-5).cpu().numpy()
    xd = oracle.decode16(si.bits(x), oracle.BF16).reshape(2, -1, 16, 4)
    mu = xd.mean(axis=(1, 3))
    var = xd.var(axis=(1, 3))
    np.testing.assert_allclose(stats[..., 0], mu, rtol=0, atol=1e-6)
    np.testing.assert_allclose(stats[..., 1], 1.0 / np.sqrt(var + 1e-5), rtol=1e-6)


def test_in_place_and_without_silu():
    x, gamma, beta = make((1, 2, 8, 8, 64), 11, "bf16", 0.0, 1.0)
    xb = si.bits(x).copy()
    stats = c3.groupnorm_stats(x, 8)
    c3.groupnorm_silu(x, stats, gamma, beta, y=x, groups=8, apply_silu=False)
    torch.cuda.synchronize()
    ref = oracle.groupnorm_silu(xb, si.bits(gamma), si.bits(beta), oracle.BF16, 8, eps=1e-6,
                                silu=False)
    assert_close(x.double().cpu().numpy(), ref)


def test_silu_tanh_form_over_the_whole_bf16_range(monkeypatch):
    # every bf16 value in [-40, 40] as a pre-activation (gamma 1, beta 0, and
    # statistics that make the normalisation the identity), against the exact
    # silu in fp64: the default tanh form must stay within the parity bounds
    # element by element, including the far negative tail where sigmoid is tiny
    monkeypatch.delenv("CONV3D_GN_SILU", raising=False)
    codes = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = oracle.decode16(codes, oracle.BF16)
    keep = np.isfinite(vals) & (np.abs(vals) <= 40.0)
    v = vals[keep]
    v = v[: (v.size // 8) * 8]
    x = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).cuda().view(1, 1, 1, -1, 8)
    stats = torch.tensor([[[0.0, 1.0]]], dtype=torch.float64, device="cuda")
    y = c3.groupnorm_silu(x, stats, None, None, groups=1, per_frame=False)
    torch.cuda.synchronize()
    got = y.double().cpu().numpy().ravel()
    ref = v / (1.0 + np.exp(-v))
    err = np.abs(got - ref)
    # each element: within bf16 rounding of the exact value plus 2^-10 of |z|/2
    bound = np.abs(ref) * 2.0 ** -8 + np.abs(v) * 2.0 ** -11 + 1e-30
    assert np.all(err <= bound), float((err / bound).max())

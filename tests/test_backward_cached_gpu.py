"""GPU backward pass of the cached-frames chunk mode against the oracle.

conv3d_bwd_data_cached gives dx and the gradient of the kt-1 cached frames
(dprev); conv3d_bwd_weight_cached gives dw and dbias with the taps that read
frames before the chunk reading the cached frames.  Every element is compared
with the oracle's adjoints (parity tolerance), in the single-CTA and the
transposed kernel variants; the weight gradient also in its CTA-pair and
swapped variants.  A clip trained in two chunks must reproduce the whole-clip
gradients (each chunk's dprev added to the chunk before).
"""
import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from parity import assert_close

pytestmark = pytest.mark.gpu

CACHED, CZERO = c3.TPAD_CAUSAL_CACHED, c3.TPAD_CAUSAL_ZERO
TD = {"bf16": (torch.bfloat16, oracle.BF16), "f16": (torch.float16, oracle.F16)}


def chunk_problem(N, Cin, D, H, W, Cout, k, pad, seed, dt, stride=(1, 1, 1)):
    td, od = TD[dt]
    fan = Cin * k[0] * k[1] * k[2]
    x = si.tensor((N, D, H, W, Cin), seed, 0, 1.0, td, "cuda")
    prev = si.tensor((N, k[0] - 1, H, W, Cin), seed, 4, 1.0, td, "cuda")
    w = si.tensor((Cout, *k, Cin), seed, 1, fan ** -0.5, td, "cuda")
    out = oracle.output_shape(D, H, W, k, stride, pad, CACHED)
    dy = si.tensor((N, *out, Cout), seed, 5, 1.0, td, "cuda")
    return x, prev, w, dy, od


CASES = [
    # N, Cin, D, H, W, Cout, kernel, pad, dtype
    (1, 64, 4, 10, 12, 64, (3, 3, 3), (0, 1, 1), "bf16"),
    (2, 64, 3, 9, 13, 128, (3, 3, 3), (0, 1, 1), "bf16"),
    (1, 32, 5, 8, 8, 48, (3, 3, 3), (0, 1, 1), "f16"),
    (1, 48, 3, 11, 10, 40, (2, 3, 3), (0, 0, 1), "bf16"),
    (1, 64, 1, 12, 12, 64, (3, 3, 3), (0, 1, 1), "bf16"),        # a one-frame chunk
    (1, 128, 2, 16, 16, 64, (1, 1, 1), (0, 0, 0), "bf16"),       # no cached frames
]


@pytest.fixture(params=["single", "swap"])
def variant(request, monkeypatch):
    monkeypatch.setenv("CONV3D_CTA_PAIR", "0")
    monkeypatch.setenv("CONV3D_SWAP", "1" if request.param == "swap" else "0")
    return request.param


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:6])) + f"-k{''.join(map(str, c[6]))}-{c[8]}")
def test_bwd_data_cached_every_element(case, variant):
    N, Cin, D, H, W, Cout, k, pad, dt = case
    x, prev, w, dy, od = chunk_problem(N, Cin, D, H, W, Cout, k, pad, 500 + Cin, dt)
    dx, dprev = c3.conv3d_bwd_data_cached(dy, w, x.shape, pad)
    assert c3.poll_status() == c3.Status.OK
    rdx, rdprev, _, _ = oracle.conv3d_backward_cached(si.bits(x), si.bits(prev), si.bits(w),
                                                      si.bits(dy), od, k, (1, 1, 1), pad)
    assert_close(dx.double().cpu().numpy(), rdx, f"dx {case}")
    if k[0] > 1:
        assert_close(dprev.double().cpu().numpy(), rdprev, f"dprev {case}")
    else:
        assert dprev is None


WGRAD_ENV = {
    "plain": {"CONV3D_WGRAD_PAIR": "0", "CONV3D_WGRAD_SWAP": "0"},
    "pair": {"CONV3D_WGRAD_PAIR": "1", "CONV3D_WGRAD_SWAP": "0"},
    "swapped": {"CONV3D_WGRAD_SWAP": "1"},
}

WCASES = [
    # N, Cin, D, H, W, Cout, kernel, stride, pad, dtype
    (1, 64, 4, 10, 12, 64, (3, 3, 3), (1, 1, 1), (0, 1, 1), "bf16"),
    (2, 128, 3, 9, 13, 256, (3, 3, 3), (1, 1, 1), (0, 1, 1), "bf16"),
    (1, 64, 5, 12, 12, 128, (3, 3, 3), (2, 2, 2), (0, 1, 1), "bf16"),    # strided
    (1, 64, 1, 12, 12, 64, (3, 3, 3), (1, 1, 1), (0, 1, 1), "f16"),      # one-frame chunk
]


@pytest.mark.parametrize("wvariant", sorted(WGRAD_ENV))
@pytest.mark.parametrize("case", WCASES, ids=lambda c: "x".join(map(str, c[:6])) + f"-s{''.join(map(str, c[7]))}-{c[9]}")
def test_bwd_weight_cached_every_element(case, wvariant, monkeypatch):
    for key, v in WGRAD_ENV[wvariant].items():
        monkeypatch.setenv(key, v)
    N, Cin, D, H, W, Cout, k, stride, pad, dt = case
    if wvariant == "swapped" and Cin % 64:
        pytest.skip("the swapped weight gradient needs Cin % 64 == 0")
    x, prev, w, dy, od = chunk_problem(N, Cin, D, H, W, Cout, k, pad, 600 + Cin, dt, stride)
    dw, db = c3.conv3d_bwd_weight_cached(x, prev, dy, k, stride, pad)
    assert c3.poll_status() == c3.Status.OK
    _, _, rdw, rdb = oracle.conv3d_backward_cached(si.bits(x), si.bits(prev), si.bits(w),
                                                   si.bits(dy), od, k, stride, pad)
    assert_close(dw.double().cpu().numpy(), rdw, f"dw {case} {wvariant}")
    assert_close(db.double().cpu().numpy(), rdb, f"dbias {case} {wvariant}")


def test_two_chunks_reproduce_the_whole_clip_gradients():
    # a 7-frame clip under the causal zero rule = chunk A (frames 0-3, causal
    # zero) then chunk B (frames 4-6, cached = A's last two frames)
    N, Cin, D, H, W, Cout, k, pad = 1, 64, 7, 10, 12, 64, (3, 3, 3), (0, 1, 1)
    x = si.tensor((N, D, H, W, Cin), 71, 0, 1.0, torch.bfloat16, "cuda")
    w = si.tensor((Cout, *k, Cin), 71, 1, (Cin * 27) ** -0.5, torch.bfloat16, "cuda")
    dy = si.tensor((N, D, H, W, Cout), 71, 5, 1.0, torch.bfloat16, "cuda")
    xa, xb = x[:, :4].contiguous(), x[:, 4:].contiguous()
    dya, dyb = dy[:, :4].contiguous(), dy[:, 4:].contiguous()
    dxa = c3.conv3d_bwd_data(dya, w, xa.shape, pad, CZERO)
    dxb, dprev = c3.conv3d_bwd_data_cached(dyb, w, xb.shape, pad)
    dwa, dba = c3.conv3d_bwd_weight(xa, dya, k, (1, 1, 1), pad, CZERO)
    dwb, dbb = c3.conv3d_bwd_weight_cached(xb, xa[:, 2:].contiguous(), dyb, k, (1, 1, 1), pad)
    assert c3.poll_status() == c3.Status.OK
    rdx, rdw, rdb = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), oracle.BF16, k,
                                           (1, 1, 1), pad, CZERO)
    dx = torch.cat([dxa, dxb], dim=1).double()
    dx[:, 2:4] += dprev.double()
    assert_close(dx.cpu().numpy(), rdx, "chunked dx")
    assert_close((dwa.double() + dwb.double()).cpu().numpy(), rdw, "chunked dw")
    assert_close((dba.double() + dbb.double()).cpu().numpy(), rdb, "chunked dbias")
    assert np.isfinite(dx.cpu().numpy()).all()

"""The tail split of the forward kernel against the oracle.

When the last round of the persistent grid is at most half full, conv3d_fwd
cuts each of its tiles into pieces along K; every piece stores an fp32 partial
and the piece that completes a tile sums them in piece order before the usual
epilogue (bias, residual, one rounding).  CONV3D_SPLIT=n forces n pieces on
small problems, so that every output element can be compared with the oracle,
including pieces that hold no k-block at all (taps that read only padding) and
the transposed variant; one problem is large enough for the default rule.
"""
import pytest
import torch

import video_vae_convolution_implicit_b200 as c3
from parity import assert_close, oracle_ref, problem

pytestmark = pytest.mark.gpu

ZERO, CREP, CZERO = c3.TPAD_ZERO, c3.TPAD_CAUSAL_REPLICATE, c3.TPAD_CAUSAL_ZERO


def run(p):
    Do, Ho, Wo = p["out"]
    y = torch.full((p["N"], Do, Ho, Wo, p["Cout"]), float("nan"), dtype=p["x"].dtype,
                   device="cuda")
    c3.conv3d_fwd(p["x"], p["w"], p["bias"], p["residual"], y, p["stride"], p["pad"], p["tpad"])
    assert c3.poll_status() == c3.Status.OK
    return y


FORCED = [
    # pieces, swap, (N, Cin, D, H, W, Cout, kernel, pad, tpad, dtype, residual)
    (3, "0", (1, 64, 3, 9, 13, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16", True)),
    (2, "0", (1, 128, 4, 20, 19, 96, (3, 3, 3), (0, 1, 1), CZERO, "bf16", False)),
    (8, "0", (1, 64, 2, 8, 8, 64, (3, 3, 3), (3, 1, 1), ZERO, "bf16", True)),   # empty pieces
    (8, "0", (1, 40, 3, 12, 12, 264, (3, 3, 3), (1, 1, 1), ZERO, "bf16", True)),  # 2 N tiles
    (4, "1", (1, 64, 3, 16, 20, 128, (3, 3, 3), (0, 1, 1), CREP, "bf16", True)),  # transposed
    (5, "0", (1, 32, 5, 32, 32, 32, (3, 3, 3), (1, 1, 1), ZERO, "f16", False)),
    (2, "1", (1, 256, 2, 16, 16, 128, (1, 1, 1), (0, 0, 0), ZERO, "bf16", False)),  # pointwise
    (3, "0", (1, 64, 1, 24, 24, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16", True)),   # first frame
]


@pytest.mark.parametrize("pieces,swap,case", FORCED)
def test_forced_split_every_element(pieces, swap, case, monkeypatch):
    monkeypatch.setenv("CONV3D_SPLIT", str(pieces))
    monkeypatch.setenv("CONV3D_SWAP", swap)
    N, Cin, D, H, W, Cout, k, pad, tpad, dtype, res = case
    p = problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=40 + pieces, dtype=dtype, residual=res)
    y = run(p)
    assert_close(y.double().cpu().numpy(), oracle_ref(p), f"split {pieces} {case}")
    # bitwise the same on a second call (the partials are summed in piece order)
    assert torch.equal(run(p), y)


def test_default_rule_splits_a_short_last_round(monkeypatch):
    # 3 frames of 80x80 in 128-pixel tiles = 150 tiles: one full round of 148
    # and a last round of 2, which the default rule cuts into pieces
    monkeypatch.delenv("CONV3D_SPLIT", raising=False)
    monkeypatch.setenv("CONV3D_SWAP", "0")      # 128-pixel tiles: 150 of them
    p = problem(1, 64, 3, 80, 80, 64, (3, 3, 3), (0, 1, 1), CREP, seed=47, residual=True)
    y = run(p)
    assert_close(y.double().cpu().numpy(), oracle_ref(p), "default split")
    monkeypatch.setenv("CONV3D_SPLIT", "0")
    y0 = run(p)
    assert_close(y0.double().cpu().numpy(), oracle_ref(p), "no split")

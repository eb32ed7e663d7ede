"""The main kernel with eight epilogue warps against the oracle.

Where a tile has at most 8 k-blocks (pointwise layers, few input channels)
the tensor cores finish a tile sooner than four warps can drain its
accumulator, so the plan gives the kernel eight epilogue warps: warps q and
q+4 share TMEM lane quarter q, one taking the even 32-column chunks and one
the odd.  CONV3D_EPI8=1 forces them on any plain or split launch and =0 turns
them off; every output element is compared with the oracle either way,
including channel counts whose last chunk is partly or wholly past Cout,
residual chunks fetched two of a warp's chunks ahead, the transposed variant,
tail-split pieces (one ticket per epilogue warp) and the data gradient of a
pointwise layer.
"""
import os
import subprocess
import sys

import pytest
import torch

import oracle
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from parity import assert_close, oracle_ref, problem
from test_backward_gpu import grads_problem

pytestmark = pytest.mark.gpu

ZERO, CREP = c3.TPAD_ZERO, c3.TPAD_CAUSAL_REPLICATE
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    # swap, split, (N, Cin, D, H, W, Cout, kernel, pad, tpad, dtype, residual)
    ("0", "0", (1, 256, 2, 16, 20, 256, (1, 1, 1), (0, 0, 0), ZERO, "bf16", True)),
    ("1", "0", (1, 256, 2, 16, 20, 256, (1, 1, 1), (0, 0, 0), ZERO, "bf16", True)),
    ("0", "0", (1, 64, 3, 9, 13, 96, (3, 3, 3), (0, 1, 1), CREP, "bf16", True)),    # 3 chunks
    ("0", "0", (2, 32, 2, 7, 9, 40, (1, 1, 1), (0, 0, 0), ZERO, "f16", True)),      # chunk 1 partly live
    ("1", "0", (1, 128, 2, 11, 13, 72, (1, 1, 1), (0, 0, 0), ZERO, "bf16", False)), # ragged pixels
    ("0", "0", (1, 64, 2, 12, 12, 264, (1, 1, 1), (0, 0, 0), ZERO, "bf16", True)),  # 2 N tiles
    ("1", "3", (1, 64, 3, 16, 20, 128, (3, 3, 3), (0, 1, 1), CREP, "bf16", True)),  # split, transposed
    ("0", "4", (1, 40, 3, 12, 12, 264, (3, 3, 3), (1, 1, 1), ZERO, "bf16", True)),  # split, 2 N tiles
    ("0", "2", (1, 256, 2, 16, 16, 256, (1, 1, 1), (0, 0, 0), ZERO, "f16", False)),
]


def _run(p):
    Do, Ho, Wo = p["out"]
    y = torch.full((p["N"], Do, Ho, Wo, p["Cout"]), float("nan"), dtype=p["x"].dtype,
                   device="cuda")
    c3.conv3d_fwd(p["x"], p["w"], p["bias"], p["residual"], y, p["stride"], p["pad"], p["tpad"])
    assert c3.poll_status() == c3.Status.OK
    return y


@pytest.mark.parametrize("epi8", ["1", "0"])
@pytest.mark.parametrize("swap,split,case", CASES,
                         ids=lambda c: c if isinstance(c, str) else "x".join(map(str, c[:6])))
def test_forward_every_element(swap, split, case, epi8, monkeypatch):
    monkeypatch.setenv("CONV3D_EPI8", epi8)
    monkeypatch.setenv("CONV3D_SWAP", swap)
    monkeypatch.setenv("CONV3D_SPLIT", split)
    monkeypatch.setenv("CONV3D_CTA_PAIR", "0")
    N, Cin, D, H, W, Cout, k, pad, tpad, dt, res = case
    p = problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=900 + Cin + Cout, dtype=dt, residual=res)
    y = _run(p)
    assert_close(y.double().cpu().numpy(), oracle_ref(p), f"epi8={epi8} {case}")
    if split != "0":
        assert torch.equal(_run(p), y)   # partials summed in piece order


@pytest.mark.parametrize("epi8", ["1", "0"])
def test_pointwise_data_gradient(epi8, monkeypatch):
    monkeypatch.setenv("CONV3D_EPI8", epi8)
    x, w, dy, od = grads_problem(1, 256, 3, 12, 14, 128, (1, 1, 1), (0, 0, 0), ZERO, 61, "bf16")
    dx = c3.conv3d_bwd_data(dy, w, x.shape, (0, 0, 0), ZERO)
    assert c3.poll_status() == c3.Status.OK
    ref, _, _ = oracle.conv3d_backward(si.bits(x), si.bits(w), si.bits(dy), od, (1, 1, 1),
                                       (1, 1, 1), (0, 0, 0), ZERO)
    assert_close(dx.double().cpu().numpy(), ref, f"dx epi8={epi8}")


RULE_SCRIPT = """
import torch
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
x = si.tensor((1, 2, 16, 16, 256), 5, 0, 1.0, torch.bfloat16, "cuda")
w1 = si.tensor((128, 1, 1, 1, 256), 5, 1, 256 ** -0.5, torch.bfloat16, "cuda")
w3 = si.tensor((128, 3, 3, 3, 256), 5, 2, (27 * 256) ** -0.5, torch.bfloat16, "cuda")
c3.conv3d(x, w1, pad=(0, 0, 0), tpad=c3.TPAD_ZERO)
c3.conv3d(x, w3, pad=(1, 1, 1), tpad=c3.TPAD_ZERO)
assert c3.poll_status() == c3.Status.OK
"""


def test_default_rule_takes_eight_warps_for_short_k_only():
    env = dict(os.environ)
    env["CONV3D_LOG"] = "1"
    env.pop("CONV3D_EPI8", None)
    r = subprocess.run([sys.executable, "-c", RULE_SCRIPT], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stderr.splitlines() if "implicit GEMM" in l]
    assert len(lines) == 2, lines
    assert "with 8 epilogue warps" in lines[0], lines      # 4 k-blocks a tile
    assert "with 8 epilogue warps" not in lines[1], lines  # 108 k-blocks a tile

"""conv3d_fwd_noalloc: the entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at all -- a host framework that owns every
device allocation through its own allocator, a latency-critical path where an
allocation could stall or fail, a deployment with a device-memory budget fixed
at start-up.  conv3d_fwd_noalloc allocates nothing: its only scratch (the
folded first-frame weight) is a fixed 16 MiB array inside the library.  These
tests call it through the C ABI on first-frame problems, which use that
scratch, and check two calls in a row against the output of the existing
conv3d_fwd within the parity tolerance.  This file sorts last so that a run
stopping at the first failure has already run every other test.
"""
import pytest
import torch

import video_vae_convolution_implicit_b200 as c3
from parity import errors, problem

pytestmark = pytest.mark.gpu

CREP = c3.TPAD_CAUSAL_REPLICATE


def _noalloc(p, y):
    Do, Ho, Wo = p["out"]
    st = c3.conv3d_fwd_noalloc_ptr(
        p["x"].data_ptr(), p["w"].data_ptr(), p["bias"].data_ptr(),
        None if p["residual"] is None else p["residual"].data_ptr(), y.data_ptr(),
        p["N"], p["Cin"], p["D"], p["H"], p["W"], p["Cout"], p["kernel"], (1, 1, 1), p["pad"],
        p["tpad"], c3.BF16 if p["dtype"] == "bf16" else c3.F16,
        torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_conv3d_fwd_on_two_calls_in_a_row():
    cases = [
        problem(2, 64, 1, 24, 24, 64, (3, 3, 3), (0, 1, 1), CREP, seed=21, residual=True),
        problem(1, 128, 1, 16, 20, 96, (3, 3, 3), (0, 1, 1), CREP, seed=22, dtype="f16"),
    ]
    for p in cases:
        Do, Ho, Wo = p["out"]
        shape = (p["N"], Do, Ho, Wo, p["Cout"])
        y_old = torch.empty(shape, dtype=p["x"].dtype, device="cuda")
        c3.conv3d_fwd(p["x"], p["w"], p["bias"], p["residual"], y_old, (1, 1, 1), p["pad"], p["tpad"])
        y_new = torch.full(shape, float("nan"), dtype=p["x"].dtype, device="cuda")
        assert _noalloc(p, y_new) == c3.Status.OK, c3.last_error()
        assert c3.poll_status() == c3.Status.OK
        assert torch.isfinite(y_new).all()
        max_ratio, rel_l1 = errors(y_new.double().cpu().numpy(), y_old.double().cpu().numpy())
        assert max_ratio <= 1e-2 and rel_l1 <= 2e-3, (max_ratio, rel_l1)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 1024 -> 1024 first frame needs 2 * 1024*9*1024 * 2 bytes > 16 MiB of fold scratch
    p = problem(1, 1024, 1, 2, 2, 1024, (3, 3, 3), (0, 1, 1), CREP, seed=23)
    y = torch.full((1, 1, 2, 2, 1024), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(p, y) == c3.Status.WORKSPACE
    assert "16777216" in c3.last_error()
    torch.cuda.synchronize()
    assert (y == 3.0).all()

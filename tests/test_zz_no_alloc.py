"""conv3d_fwd_noalloc: the entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at all -- a host framework that owns every
device allocation through its own allocator, a latency-critical path where an
allocation could stall or fail, a deployment with a device-memory budget fixed
at start-up.  conv3d_fwd_noalloc allocates nothing: its only scratch (the
folded first-frame weight) is a fixed 16 MiB array inside the library.

These tests call it through the C ABI on first-frame problems, which use that
scratch.  It runs the same fold kernel and main kernel on the same bits as
conv3d_fwd (with conv3d_fwd's tail split and 8-bit lo product off, which
noalloc never uses), so the
two must agree bit for bit, on two calls in a row, with the
larger problem first so that the second call runs over leftover scratch
beyond its own size; one output is also checked against the fp64 oracle, and
free device memory must not change across the calls.  This file sorts last so
that a run stopping at the first failure has already run every other test.
"""
import pytest
import torch

import video_vae_convolution_implicit_b200 as c3
from parity import assert_close, oracle_ref, problem

pytestmark = pytest.mark.gpu

CREP = c3.TPAD_CAUSAL_REPLICATE


def _noalloc(p, y):
    st = c3.conv3d_fwd_noalloc_ptr(
        p["x"].data_ptr(), p["w"].data_ptr(), p["bias"].data_ptr(),
        None if p["residual"] is None else p["residual"].data_ptr(), y.data_ptr(),
        p["N"], p["Cin"], p["D"], p["H"], p["W"], p["Cout"], p["kernel"], (1, 1, 1), p["pad"],
        p["tpad"], c3.BF16 if p["dtype"] == "bf16" else c3.F16,
        torch.cuda.current_stream().cuda_stream)
    return st


def _out(p, fill=float("nan")):
    Do, Ho, Wo = p["out"]
    return torch.full((p["N"], Do, Ho, Wo, p["Cout"]), fill, dtype=p["x"].dtype, device="cuda")


def test_noalloc_equals_conv3d_fwd_bit_for_bit_on_two_calls_in_a_row(monkeypatch):
    # conv3d_fwd_noalloc never splits its tiles along K (that needs scratch
    # beyond the fold) and keeps the lo part of the folded weight in 16 bits
    # (an 8-bit copy of x would need scratch too), so it is compared with
    # conv3d_fwd with the split off and the 16-bit lo part (the default)
    monkeypatch.setenv("CONV3D_SPLIT", "0")
    monkeypatch.setenv("CONV3D_LO8", "0")
    # the larger fold first (2 * 192*9*160 16-bit values), then a smaller one
    # (2 * 64*9*64) that runs over the larger one's leftover scratch
    big = problem(1, 160, 1, 20, 28, 192, (3, 3, 3), (0, 1, 1), CREP, seed=24, residual=True)
    small = problem(2, 64, 1, 24, 24, 64, (3, 3, 3), (0, 1, 1), CREP, seed=21, residual=True)
    half = problem(1, 128, 1, 16, 20, 96, (3, 3, 3), (0, 1, 1), CREP, seed=22, dtype="f16")
    cases = [big, small, half]
    refs = []
    for p in cases:
        y_old = _out(p)
        c3.conv3d_fwd(p["x"], p["w"], p["bias"], p["residual"], y_old, (1, 1, 1), p["pad"],
                      p["tpad"])
        refs.append(y_old)
    assert c3.poll_status() == c3.Status.OK
    # two rounds: the second runs every case again over the first round's scratch
    for _ in range(2):
        for p, y_old in zip(cases, refs):
            y_new = _out(p)
            assert _noalloc(p, y_new) == c3.Status.OK, c3.last_error()
            assert c3.poll_status() == c3.Status.OK
            assert torch.equal(y_new, y_old), "noalloc output differs from conv3d_fwd"
    # and the small case directly against the oracle, on every element
    y = _out(small)
    assert _noalloc(small, y) == c3.Status.OK, c3.last_error()
    assert c3.poll_status() == c3.Status.OK
    assert_close(y.double().cpu().numpy(), oracle_ref(small), "noalloc vs oracle")


def test_noalloc_allocates_no_device_memory():
    p = problem(1, 128, 1, 32, 32, 128, (3, 3, 3), (0, 1, 1), CREP, seed=25)
    y = _out(p, 0.0)
    # warm: kernels loaded and the scratch address looked up
    assert _noalloc(p, y) == c3.Status.OK, c3.last_error()
    assert c3.poll_status() == c3.Status.OK
    c3.release()              # drops conv3d_fwd's cached workspace, if any
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        assert _noalloc(p, y) == c3.Status.OK, c3.last_error()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert c3.poll_status() == c3.Status.OK


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 1024 -> 1024 first frame needs 2 * 1024*9*1024 * 2 bytes > 16 MiB of fold scratch
    p = problem(1, 1024, 1, 2, 2, 1024, (3, 3, 3), (0, 1, 1), CREP, seed=23)
    y = torch.full((1, 1, 2, 2, 1024), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(p, y) == c3.Status.WORKSPACE
    assert "16777216" in c3.last_error()
    torch.cuda.synchronize()
    assert (y == 3.0).all()

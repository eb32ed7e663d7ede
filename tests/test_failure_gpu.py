"""Failure detection inside the convolution kernels themselves.

conv3d_test_arm_stall makes the next kernel launch's TMA producer skip the
copies of its first pipeline stage, so the tensor-core issuer waits on a stage
that never fills.  That wait is bounded (here 50 ms): it must run out, every
role of every CTA must leave its loop, drain what it has in flight (copies,
tensor-core work, residual prefetches, TMA stores; for a CTA pair the even
CTA settles the stages only one of the two CTAs issued) and free tensor
memory, and the call must report CONV3D_ERR_TIMEOUT through
conv3d_poll_status -- without a fault, so that the very next call on the same
context is correct again (checked against the oracle).
"""
import time

import pytest
import torch

import oracle
import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from parity import assert_close, oracle_ref, problem

pytestmark = pytest.mark.gpu

CREP = c3.TPAD_CAUSAL_REPLICATE
LIMIT_MS = 50

FWD_VARIANTS = {
    "single": {"CONV3D_SWAP": "0", "CONV3D_CTA_PAIR": "0"},
    "transposed": {"CONV3D_SWAP": "1", "CONV3D_CTA_PAIR": "0"},
    "pair": {"CONV3D_SWAP": "0", "CONV3D_CTA_PAIR": "1"},
}


@pytest.fixture(autouse=True)
def _disarm():
    yield
    c3.test_arm_stall(0)
    c3.poll_status()


def _stalled(call):
    """Runs `call` with one armed launch; returns (status, seconds)."""
    assert c3.poll_status() == c3.Status.OK
    c3.test_arm_stall(1, LIMIT_MS)
    t0 = time.perf_counter()
    call()
    st = c3.poll_status()
    return st, time.perf_counter() - t0


@pytest.mark.parametrize("variant", sorted(FWD_VARIANTS))
def test_forward_kernel_times_out_and_recovers(variant, monkeypatch):
    for k, v in FWD_VARIANTS[variant].items():
        monkeypatch.setenv(k, v)
    # several tiles per CTA, a residual (prefetches in flight at the abort)
    p = problem(1, 64, 3, 40, 40, 128, (3, 3, 3), (0, 1, 1), CREP, seed=31, residual=True)
    Do, Ho, Wo = p["out"]
    y = torch.empty((1, Do, Ho, Wo, 128), dtype=torch.bfloat16, device="cuda")

    def call():
        c3.conv3d_fwd(p["x"], p["w"], p["bias"], p["residual"], y, (1, 1, 1), p["pad"], p["tpad"])

    st, dt = _stalled(call)
    assert st == c3.Status.TIMEOUT, c3.status_string(st)
    assert dt < 5.0, dt
    # the context is intact: the next call is correct
    y.fill_(float("nan"))
    call()
    assert c3.poll_status() == c3.Status.OK
    assert_close(y.double().cpu().numpy(), oracle_ref(p), f"after a timeout ({variant})")


WGRAD_VARIANTS = {
    # name: (env, Cout)
    "plain": ({"CONV3D_WGRAD_PAIR": "0", "CONV3D_WGRAD_SWAP": "0"}, 256),
    "pair": ({"CONV3D_WGRAD_PAIR": "1", "CONV3D_WGRAD_SWAP": "0"}, 256),
    "swapped": ({"CONV3D_WGRAD_SWAP": "1"}, 128),
}


@pytest.mark.parametrize("variant", sorted(WGRAD_VARIANTS))
def test_weight_gradient_kernel_times_out_and_recovers(variant, monkeypatch):
    env, Cout = WGRAD_VARIANTS[variant]
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    N, Cin, D, H, W = 1, 128, 3, 24, 24
    kernel, pad = (3, 3, 3), (0, 1, 1)
    p = problem(N, Cin, D, H, W, Cout, kernel, pad, CREP, seed=32)
    out = p["out"]
    dy = si.tensor((N, *out, Cout), 32, 5, 1.0, torch.bfloat16, "cuda")

    def call():
        return c3.conv3d_bwd_weight(p["x"], dy, kernel, (1, 1, 1), pad, CREP)

    st, dt = _stalled(call)
    assert st == c3.Status.TIMEOUT, c3.status_string(st)
    assert dt < 5.0, dt
    dw, db = call()
    assert c3.poll_status() == c3.Status.OK
    _, rdw, rdb = oracle.conv3d_backward(si.bits(p["x"]), si.bits(p["w"]), si.bits(dy),
                                         oracle.BF16, kernel, (1, 1, 1), pad, CREP)
    assert_close(dw.double().cpu().numpy(), rdw, f"dw after a timeout ({variant})")
    assert_close(db.double().cpu().numpy(), rdb, f"dbias after a timeout ({variant})")

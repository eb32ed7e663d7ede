"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Small problems are compared on every output element; the full-size workloads
are compared on sampled rows (borders, first/last frames, first/last tiles,
random interior points) that the oracle evaluates one by one, in the same
launch configuration the bench times.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
import video_vae_convolution_implicit_b200 as c3
from seeded_inputs.workloads import WORKLOADS
from parity import assert_close, oracle_ref, problem, sample_rows

pytestmark = pytest.mark.gpu

ZERO, CREP, CZERO = c3.TPAD_ZERO, c3.TPAD_CAUSAL_REPLICATE, c3.TPAD_CAUSAL_ZERO
CACHED = c3.TPAD_CAUSAL_CACHED


def run(p, residual_into_y=False, workspace=None):
    Do, Ho, Wo = p["out"]
    y = torch.empty((p["N"], Do, Ho, Wo, p["Cout"]), dtype=p["x"].dtype, device="cuda")
    res = p["residual"]
    if residual_into_y:
        y.copy_(res)
        res = y
    c3.conv3d_fwd(p["x"], p["w"], p["bias"], res, y, p["stride"], p["pad"], p["tpad"],
                  workspace=workspace, prev=p["prev"])
    assert c3.poll_status() == c3.Status.OK
    return y


def full_check(p, **kw):
    ref = oracle_ref(p)
    y = run(p, **kw)
    return assert_close(y.double().cpu().numpy(), ref, str({k: p[k] for k in ("N", "Cin", "Cout", "D", "H", "W", "kernel", "stride", "pad", "tpad")}))


# ------------------------------------------------------------------ small, every element

SMALL = [
    # N, Cin, D, H, W, Cout, kernel, pad, tpad, dtype, residual
    (1, 32, 5, 32, 32, 32, (3, 3, 3), (1, 1, 1), ZERO, "f16", False),      # workload cfg1 shape
    (2, 64, 3, 9, 13, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16", True),      # ragged frame < 1 tile
    (1, 128, 4, 20, 19, 96, (3, 3, 3), (0, 1, 1), CZERO, "bf16", False),  # 3 tiles/frame, ragged
    (1, 40, 3, 12, 12, 264, (3, 3, 3), (1, 1, 1), ZERO, "bf16", True),    # partial chunk, 2 N tiles
    (1, 8, 3, 6, 7, 8, (3, 3, 3), (0, 1, 1), CREP, "bf16", False),        # minimal channels
    (1, 256, 2, 16, 16, 128, (1, 1, 1), (0, 0, 0), ZERO, "bf16", False),  # pointwise
    (1, 64, 4, 10, 14, 64, (1, 3, 3), (0, 1, 1), CREP, "bf16", False),
    (1, 64, 5, 10, 10, 32, (3, 1, 1), (0, 0, 0), CREP, "f16", False),
    (2, 64, 4, 9, 9, 48, (2, 3, 3), (0, 1, 1), CZERO, "bf16", True),
    (1, 64, 6, 8, 8, 64, (3, 3, 3), (0, 1, 1), ZERO, "bf16", False),      # zero pt=0: Do = D-2
    (1, 64, 3, 8, 8, 64, (3, 3, 3), (2, 1, 1), ZERO, "bf16", False),      # pt=2: edge frames 1 tap
    (1, 64, 2, 8, 8, 64, (3, 3, 3), (3, 1, 1), ZERO, "bf16", True),       # windows fully in padding
    (1, 192, 2, 11, 23, 200, (3, 3, 3), (0, 2, 0), CREP, "f16", True),    # asymmetric pads
    (3, 16, 2, 5, 5, 24, (3, 3, 3), (0, 1, 1), CREP, "bf16", False),
    (2, 64, 3, 9, 13, 64, (3, 3, 3), (0, 1, 1), CACHED, "bf16", True),    # cached previous frames
    (1, 128, 1, 20, 19, 128, (3, 3, 3), (0, 1, 1), CACHED, "f16", False), # one-frame chunk
    (1, 40, 4, 12, 12, 72, (2, 3, 3), (0, 1, 1), CACHED, "bf16", False),
    (1, 64, 3, 1, 1, 64, (3, 3, 3), (0, 1, 1), CREP, "bf16", False),      # 1x1 frames
    (2, 32, 2, 1, 7, 48, (3, 3, 3), (1, 1, 1), ZERO, "f16", True),        # one-row frames
    (1, 64, 2, 3, 300, 64, (3, 3, 3), (0, 1, 1), CZERO, "bf16", False),   # rows longer than a tile
]


@pytest.fixture(params=["single", "pair", "swap"])
def cta_mode(request, monkeypatch):
    """Run a test with each kernel variant: one CTA per 128-pixel tile (M = pixels),
    a CTA pair per 256-pixel tile (cta_group::2), or the transposed product
    (M = 128 channels, N = 256 pixels)."""
    monkeypatch.setenv("CONV3D_CTA_PAIR", "1" if request.param == "pair" else "0")
    monkeypatch.setenv("CONV3D_SWAP", "1" if request.param == "swap" else "0")
    return request.param


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "x".join(map(str, c[:6])) + f"-k{''.join(map(str, c[6]))}-t{c[8]}-{c[9]}")
def test_small_every_element(case, cta_mode):
    N, Cin, D, H, W, Cout, k, pad, tpad, dt, res = case
    p = problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=100 + Cin + Cout, dtype=dt, residual=res)
    full_check(p)


def test_no_bias_no_residual(cta_mode):
    p = problem(1, 64, 3, 10, 12, 64, (3, 3, 3), (0, 1, 1), CREP, seed=3, bias=False)
    full_check(p)


def test_residual_in_place(cta_mode):
    p = problem(1, 64, 3, 10, 12, 64, (3, 3, 3), (0, 1, 1), CREP, seed=4, residual=True)
    full_check(p, residual_into_y=True)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_first_frame_fold(dt, cta_mode):
    """D=1 with causal replicate padding runs the folded 2D path."""
    p = problem(2, 64, 1, 24, 24, 64, (3, 3, 3), (0, 1, 1), CREP, seed=5, dtype=dt, residual=True)
    full_check(p)


def test_first_frame_fold_explicit_workspace():
    p = problem(1, 128, 1, 16, 20, 64, (3, 3, 3), (0, 1, 1), CREP, seed=6)
    need = c3.workspace_bytes(128, 64, (3, 3, 3), 1, CREP)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ref = oracle_ref(p)
    y = run(p, workspace=ws)
    assert_close(y.double().cpu().numpy(), ref)


def test_first_frame_causal_zero_uses_last_tap_only():
    p = problem(1, 64, 1, 16, 16, 64, (3, 3, 3), (0, 1, 1), CZERO, seed=7)
    full_check(p)


# ------------------------------------------------------------------ robustness

def test_every_output_written_and_no_overrun(cta_mode):
    """Poison y with NaN, put a canary after it: all of y is written, the canary is not."""
    p = problem(1, 64, 3, 11, 13, 40, (3, 3, 3), (0, 1, 1), CREP, seed=8, residual=True)
    Do, Ho, Wo = p["out"]
    n = p["N"] * Do * Ho * Wo * p["Cout"]
    buf = torch.full((n + 4096,), float("nan"), dtype=torch.bfloat16, device="cuda")
    buf[n:] = 1234.0
    y = buf[:n].view(p["N"], Do, Ho, Wo, p["Cout"])
    c3.conv3d_fwd(p["x"], p["w"], p["bias"], p["residual"], y, (1, 1, 1), p["pad"], p["tpad"])
    assert c3.poll_status() == c3.Status.OK
    assert torch.isfinite(y).all()
    assert (buf[n:] == 1234.0).all()
    assert_close(y.double().cpu().numpy(), oracle_ref(p))


def test_deterministic_bitwise(cta_mode):
    p = problem(1, 256, 3, 32, 32, 256, (3, 3, 3), (0, 1, 1), CREP, seed=9, residual=True)
    y1 = run(p)
    y2 = run(p)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_rejected_call_leaves_y_untouched():
    p = problem(1, 64, 2, 8, 8, 64, (3, 3, 3), (0, 1, 1), CREP, seed=10)
    y = torch.full((1, 2, 8, 8, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    st = c3.conv3d_fwd_ptr(p["x"].data_ptr(), p["w"].data_ptr(), None, None, y.data_ptr(),
                           1, 64, 2, 8, 8, 64, (3, 3, 3), (1, 9, 9), (0, 1, 1), CREP, c3.BF16, 0)
    assert st == c3.Status.UNSUPPORTED
    torch.cuda.synchronize()
    assert (y == 7.0).all()


def test_bounded_wait_reports_timeout():
    """The device wait gives up after its limit and reports it; the context stays usable."""
    import time
    t0 = time.time()
    assert c3.selftest_wait_timeout(50) == c3.Status.TIMEOUT
    assert time.time() - t0 < 5.0
    assert c3.poll_status() == c3.Status.OK       # the word was cleared
    p = problem(1, 64, 3, 10, 12, 64, (3, 3, 3), (0, 1, 1), CREP, seed=3, bias=False)
    full_check(p)                                 # and the GPU still computes


# ------------------------------------------------------------------ full-size workloads, sampled

@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workload_sampled(name, monkeypatch):
    """Full-size workloads in the launch configuration the bench times (automatic choice)."""
    monkeypatch.delenv("CONV3D_CTA_PAIR", raising=False)
    monkeypatch.delenv("CONV3D_SWAP", raising=False)
    wl = WORKLOADS[name]
    p = problem(wl.N, wl.Cin, wl.D, wl.H, wl.W, wl.Cout, wl.kernel, wl.pad, wl.tpad, wl.seed,
                wl.dtype, True, wl.residual, stride=wl.stride)
    y = run(p)
    Do, Ho, Wo = p["out"]
    rows = sample_rows(wl.N, Do, Ho, Wo, n_random=256, seed=wl.seed)
    ref = oracle_ref(p, rows=rows)
    got = y.view(-1, wl.Cout)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    assert_close(got, ref, name)
    assert torch.isfinite(y).all()


@pytest.mark.parametrize("first", [CREP, CZERO])
def test_chunked_decoding_equals_whole_clip(first, cta_mode, monkeypatch):
    """A clip convolved in one call equals the same clip convolved chunk by
    chunk (first chunk: the causal rule; later chunks: conv3d_fwd_cached with
    the previous chunk's last kt-1 input frames), bit for bit: every tile sums
    the same products in the same order.  Without the tail split, which cuts
    different tiles of the whole clip and of a chunk along K (the results then
    differ only by the fp32 summation order of those tiles)."""
    monkeypatch.setenv("CONV3D_SPLIT", "0")
    N, Cin, D, H, W, Cout = 1, 64, 9, 16, 20, 128
    p = problem(N, Cin, D, H, W, Cout, (3, 3, 3), (0, 1, 1), first, seed=51, residual=True)
    whole = run(p)
    parts, t0 = [], 0
    for size in (4, 1, 4):
        sl = slice(t0, t0 + size)
        x = p["x"][:, sl].contiguous()
        res = p["residual"][:, sl].contiguous()
        y = torch.empty((N, size, H, W, Cout), dtype=x.dtype, device="cuda")
        if t0 == 0:
            c3.conv3d_fwd(x, p["w"], p["bias"], res, y, (1, 1, 1), (0, 1, 1), first)
        else:
            prev = p["x"][:, t0 - 2:t0].contiguous()
            c3.conv3d_fwd(x, p["w"], p["bias"], res, y, (1, 1, 1), (0, 1, 1), CACHED, prev=prev)
        assert c3.poll_status() == c3.Status.OK
        parts.append(y)
        t0 += size
    assert torch.equal(torch.cat(parts, dim=1).view(torch.int16), whole.view(torch.int16))


STRIDED = [
    # N, Cin, D, H, W, Cout, kernel, stride, pad, tpad, dtype, residual
    (1, 64, 5, 16, 20, 64, (3, 3, 3), (1, 2, 2), (0, 1, 1), CREP, "bf16", False),   # spatial downsample
    (1, 128, 9, 18, 17, 128, (3, 3, 3), (2, 2, 2), (0, 1, 1), CREP, "bf16", True),  # causal 2x2x2
    (2, 64, 6, 12, 12, 96, (3, 3, 3), (2, 1, 1), (1, 1, 1), ZERO, "f16", False),    # temporal only
    (1, 32, 4, 10, 23, 40, (3, 3, 3), (1, 1, 2), (0, 0, 1), CZERO, "bf16", False),  # width only
    (1, 64, 3, 15, 15, 64, (1, 3, 3), (1, 3, 3), (0, 1, 1), CREP, "bf16", False),   # stride 3
    (1, 64, 5, 12, 12, 64, (3, 3, 3), (2, 2, 2), (0, 1, 1), CACHED, "bf16", False), # cached + stride
    (1, 256, 2, 16, 16, 128, (1, 1, 1), (1, 2, 2), (0, 0, 0), ZERO, "bf16", False), # strided 1x1x1
]


@pytest.mark.parametrize("case", STRIDED, ids=lambda c: f"s{''.join(map(str, c[7]))}-k{''.join(map(str, c[6]))}-t{c[9]}-{c[10]}")
def test_strided_every_element(case, cta_mode):
    N, Cin, D, H, W, Cout, k, stride, pad, tpad, dt, res = case
    p = problem(N, Cin, D, H, W, Cout, k, pad, tpad, seed=200 + Cin + Cout, dtype=dt,
                residual=res, stride=stride)
    full_check(p)


def test_strided_first_frame_fold(cta_mode):
    p = problem(1, 64, 1, 24, 24, 64, (3, 3, 3), (0, 1, 1), CREP, seed=61, stride=(2, 2, 2))
    full_check(p)

"""The C ABI: exports, host-side validation and error codes (no GPU needed).

Validation runs before any CUDA call, so these tests pass fake, never
dereferenced device addresses and check that the library answers with the
documented status code.
"""
import ctypes
import os
import re

import pytest
import torch

import video_vae_convolution_implicit_b200 as c3
from video_vae_convolution_implicit_b200 import Status

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# fake, 256-byte aligned, widely separated "device" addresses (never touched)
X, Wt, B, R, Y = 0x100000000, 0x200000000, 0x300000000, 0x400000000, 0x500000000


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"CONV3D_API\s+[\w\s\*]*?\b(conv3d_\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert "conv3d_fwd" in names and "conv3d_fwd_ws" in names
    lib = ctypes.CDLL(c3.lib_path)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for s in range(8):
        assert c3.status_string(s) and c3.status_string(s) != "unknown status"
    assert c3.status_string(99) == "unknown status"


@pytest.mark.parametrize("D,H,W,k,pad,tpad,expect", [
    (9, 128, 128, (3, 3, 3), (0, 1, 1), c3.TPAD_CAUSAL_REPLICATE, (9, 128, 128)),
    (5, 32, 32, (3, 3, 3), (1, 1, 1), c3.TPAD_ZERO, (5, 32, 32)),
    (5, 32, 32, (3, 3, 3), (0, 1, 1), c3.TPAD_ZERO, (3, 32, 32)),
    (1, 256, 256, (3, 3, 3), (0, 1, 1), c3.TPAD_CAUSAL_ZERO, (1, 256, 256)),
    (33, 128, 128, (1, 1, 1), (0, 0, 0), c3.TPAD_ZERO, (33, 128, 128)),
    (4, 7, 9, (2, 3, 1), (0, 0, 2), c3.TPAD_CAUSAL_REPLICATE, (4, 5, 13)),
    (3, 16, 16, (3, 3, 3), (0, 1, 1), c3.TPAD_CAUSAL_CACHED, (3, 16, 16)),
])
def test_output_shape(D, H, W, k, pad, tpad, expect):
    assert c3.output_shape(D, H, W, k, (1, 1, 1), pad, tpad) == expect


@pytest.mark.parametrize("stride", [(1, 2, 2), (2, 2, 2), (2, 1, 3)])
def test_output_shape_strided_matches_oracle(stride):
    import oracle
    for tpad in (c3.TPAD_ZERO, c3.TPAD_CAUSAL_REPLICATE, c3.TPAD_CAUSAL_ZERO):
        pad = (1, 1, 1) if tpad == c3.TPAD_ZERO else (0, 1, 1)
        assert c3.output_shape(9, 17, 20, (3, 3, 3), stride, pad, tpad) == \
            oracle.output_shape(9, 17, 20, (3, 3, 3), stride, pad, tpad)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_strided_call_passes_validation_without_gpu():
    assert call(stride=(2, 2, 2)) == Status.CUDA


def test_output_shape_rejects_empty():
    with pytest.raises(c3.Conv3dError):
        c3.output_shape(1, 2, 2, (3, 3, 3), (1, 1, 1), (0, 0, 0), c3.TPAD_ZERO)


def test_workspace_bytes():
    # first-frame fold: (hi, lo) x Cout*kh*kw*Cin 16-bit values, rounded up to 256 bytes
    assert c3.workspace_bytes(256, 256, (3, 3, 3), 1, c3.TPAD_CAUSAL_REPLICATE) == 2 * 256 * 9 * 256 * 2
    assert c3.workspace_bytes(8, 8, (3, 3, 3), 1, c3.TPAD_CAUSAL_REPLICATE) == 2304
    assert c3.workspace_bytes(256, 256, (3, 3, 3), 2, c3.TPAD_CAUSAL_REPLICATE) == 0
    assert c3.workspace_bytes(256, 256, (3, 3, 3), 1, c3.TPAD_CAUSAL_ZERO) == 0
    assert c3.workspace_bytes(256, 256, (1, 3, 3), 1, c3.TPAD_CAUSAL_REPLICATE) == 0


def call(**kw):
    a = dict(x=X, w=Wt, bias=B, residual=None, y=Y, N=1, Cin=64, D=4, H=16, W=16, Cout=64,
             kernel=(3, 3, 3), stride=(1, 1, 1), pad=(0, 1, 1), tpad=c3.TPAD_CAUSAL_REPLICATE,
             dtype=c3.BF16, stream=None)
    a.update(kw)
    return c3.conv3d_fwd_ptr(**a)


@pytest.mark.parametrize("kw,expect", [
    (dict(x=None), Status.INVALID_ARG),
    (dict(w=None), Status.INVALID_ARG),
    (dict(y=None), Status.INVALID_ARG),
    (dict(N=0), Status.INVALID_ARG),
    (dict(Cin=-8), Status.INVALID_ARG),
    (dict(dtype=7), Status.INVALID_ARG),
    (dict(tpad=9), Status.INVALID_ARG),
    (dict(kernel=(3, 0, 3)), Status.INVALID_ARG),
    (dict(pad=(1, 1, 1)), Status.INVALID_ARG),            # pt must be 0 in causal modes
    (dict(pad=(0, -1, 1), tpad=c3.TPAD_ZERO), Status.INVALID_ARG),
    (dict(H=1, pad=(0, 0, 1)), Status.INVALID_ARG),        # padded input smaller than kernel
    (dict(stride=(1, 9, 9)), Status.UNSUPPORTED),          # TMA traversal strides are <= 8
    (dict(Cin=12), Status.UNSUPPORTED),
    (dict(Cout=20), Status.UNSUPPORTED),
    (dict(kernel=(3, 9, 3)), Status.UNSUPPORTED),
    (dict(x=X + 8), Status.ALIGNMENT),
    (dict(y=Y + 2), Status.ALIGNMENT),
    (dict(bias=B + 4), Status.ALIGNMENT),
    (dict(residual=R + 8), Status.ALIGNMENT),
    (dict(y=X + 256), Status.INVALID_ARG),                 # y overlaps x
    (dict(residual=Y + 4096), Status.INVALID_ARG),         # residual partially overlaps y
    (dict(tpad=c3.TPAD_CAUSAL_CACHED), Status.INVALID_ARG),  # needs conv3d_fwd_cached's prev
])
def test_validation_errors(kw, expect):
    assert call(**kw) == expect
    assert c3.last_error()


def test_ws_entry_point_requires_workspace_for_first_frame():
    a = dict(x=X, w=Wt, bias=B, residual=None, y=Y, N=1, Cin=64, D=1, H=16, W=16, Cout=64,
             kernel=(3, 3, 3), stride=(1, 1, 1), pad=(0, 1, 1), tpad=c3.TPAD_CAUSAL_REPLICATE,
             dtype=c3.BF16, stream=None)
    assert c3.conv3d_fwd_ws_ptr(**a, workspace=None, ws_bytes=0) == Status.WORKSPACE
    need = c3.workspace_bytes(64, 64, (3, 3, 3), 1, c3.TPAD_CAUSAL_REPLICATE)
    assert c3.conv3d_fwd_ws_ptr(**a, workspace=0x600000000, ws_bytes=need - 1) == Status.WORKSPACE
    assert c3.conv3d_fwd_ws_ptr(**a, workspace=0x600000010, ws_bytes=need) == Status.ALIGNMENT
    assert c3.conv3d_fwd_ws_ptr(**a, workspace=Wt, ws_bytes=need) == Status.INVALID_ARG
    # the main kernel reads bias and residual after the fold wrote the workspace
    assert c3.conv3d_fwd_ws_ptr(**a, workspace=B, ws_bytes=need) == Status.INVALID_ARG
    a["residual"] = R
    assert c3.conv3d_fwd_ws_ptr(**a, workspace=R, ws_bytes=need) == Status.INVALID_ARG
    assert "residual" in c3.last_error()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_reports_cuda_error():
    # a well-formed problem gets past validation and fails at the first CUDA call
    assert call() == Status.CUDA
    assert c3.last_error()


def test_selftest_rejects_bad_limits():
    assert c3.selftest_wait_timeout(0) == Status.INVALID_ARG
    assert c3.selftest_wait_timeout(20000) == Status.INVALID_ARG


def test_torch_wrapper_rejects_host_tensors():
    x = torch.zeros(1, 2, 4, 4, 8, dtype=torch.bfloat16)
    w = torch.zeros(8, 3, 3, 3, 8, dtype=torch.bfloat16)
    y = torch.zeros(1, 2, 4, 4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        c3.conv3d_fwd(x, w, None, None, y)


P = 0x700000000   # fake cached-frames address


def call_cached(**kw):
    a = dict(x=X, prev=P, w=Wt, bias=B, residual=None, y=Y, N=1, Cin=64, D=4, H=16, W=16, Cout=64,
             kernel=(3, 3, 3), stride=(1, 1, 1), pad=(0, 1, 1), dtype=c3.BF16, stream=None)
    a.update(kw)
    return c3.conv3d_fwd_cached_ptr(**a)


@pytest.mark.parametrize("kw,expect", [
    (dict(prev=None), Status.INVALID_ARG),                 # kt > 1 needs the cached frames
    (dict(prev=P + 8), Status.ALIGNMENT),
    (dict(prev=Y + 512), Status.INVALID_ARG),              # prev overlaps y
    (dict(pad=(1, 1, 1)), Status.INVALID_ARG),
    (dict(stride=(9, 1, 1)), Status.UNSUPPORTED),
])
def test_cached_entry_validation(kw, expect):
    assert call_cached(**kw) == expect


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_cached_entry_without_gpu_reports_cuda_error():
    assert call_cached() == Status.CUDA
    assert call_cached(prev=None, kernel=(1, 3, 3)) == Status.CUDA   # kt = 1 needs no prev


# ---------------------------------------------------------------- GroupNorm entry points

ST = 0x800000000   # fake stats address


@pytest.mark.parametrize("kw,expect", [
    (dict(x=None), Status.INVALID_ARG),
    (dict(C=96, groups=7), Status.INVALID_ARG),            # C % groups
    (dict(C=12, groups=3), Status.UNSUPPORTED),            # C % 8
    (dict(x=X + 8), Status.ALIGNMENT),
    (dict(stats=ST + 4), Status.ALIGNMENT),
    (dict(stats=None), Status.INVALID_ARG),
    (dict(eps=-1.0), Status.INVALID_ARG),
    (dict(dtype=5), Status.INVALID_ARG),
])
def test_groupnorm_stats_validation(kw, expect):
    a = dict(x=X, N=1, D=2, H=4, W=4, C=64, groups=8, per_frame=0, eps=1e-6, dtype=c3.BF16,
             stats=ST, stream=None)
    a.update(kw)
    assert c3.groupnorm_stats_ptr(**a) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(y=None), Status.INVALID_ARG),
    (dict(y=Y + 2), Status.ALIGNMENT),
    (dict(gamma=B + 8), Status.ALIGNMENT),
    (dict(C=64, groups=6), Status.INVALID_ARG),
])
def test_groupnorm_silu_validation(kw, expect):
    a = dict(x=X, stats=ST, gamma=B, beta=None, y=Y, N=1, D=2, H=4, W=4, C=64, groups=8,
             per_frame=0, apply_silu=1, dtype=c3.BF16, stream=None)
    a.update(kw)
    assert c3.groupnorm_silu_ptr(**a) == expect


# ---------------------------------------------------------------- backward entry points

WS = 0x900000000   # fake workspace address


def call_bwd_data(**kw):
    a = dict(dy=Y, w=Wt, dx=X, N=1, Cin=64, D=4, H=16, W=16, Cout=64, kernel=(3, 3, 3),
             stride=(1, 1, 1), pad=(0, 1, 1), tpad=c3.TPAD_CAUSAL_REPLICATE, dtype=c3.BF16,
             workspace=WS, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return c3.conv3d_bwd_data_ptr(**a)


def call_bwd_weight(**kw):
    a = dict(x=X, dy=Y, dw=Wt, dbias=B, N=1, Cin=64, D=4, H=16, W=16, Cout=64, kernel=(3, 3, 3),
             stride=(1, 1, 1), pad=(0, 1, 1), tpad=c3.TPAD_CAUSAL_REPLICATE, dtype=c3.BF16,
             workspace=WS, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return c3.conv3d_bwd_weight_ptr(**a)


def test_bwd_workspace_bytes():
    # flipped weight + (replicate padding) the fp32 gradient of frames -2..0
    wt = 64 * 27 * 64 * 2
    split = 160 * (128 * 256 * 4 + 64)       # the tail-split region: 160 pieces, 8 tickets each
    assert c3.bwd_data_workspace_bytes(1, 64, 4, 16, 16, 64, (3, 3, 3), (0, 1, 1),
                                       c3.TPAD_CAUSAL_REPLICATE) == wt + 3 * 16 * 16 * 64 * 4 + split
    assert c3.bwd_data_workspace_bytes(2, 64, 4, 16, 16, 64, (3, 3, 3), (1, 1, 1),
                                       c3.TPAD_ZERO) == wt + split
    # the cached-frames data gradient needs the flipped weight only
    assert c3.bwd_data_workspace_bytes(2, 64, 4, 16, 16, 64, (3, 3, 3), (0, 1, 1),
                                       c3.TPAD_CAUSAL_CACHED) == wt
    dw = 64 * 27 * 32 * 4
    assert c3.bwd_weight_workspace_bytes(32, 64, (3, 3, 3)) >= dw + 64 * 4


@pytest.mark.parametrize("kw,expect", [
    (dict(stride=(2, 1, 1)), Status.UNSUPPORTED),          # temporal stride
    (dict(stride=(2, 2, 2)), Status.UNSUPPORTED),
    (dict(tpad=c3.TPAD_CAUSAL_CACHED), Status.UNSUPPORTED),
    (dict(pad=(0, 3, 1)), Status.UNSUPPORTED),             # pad > kernel extent - 1 at stride 1
    (dict(workspace=None), Status.WORKSPACE),
    (dict(ws_bytes=64), Status.WORKSPACE),
    (dict(workspace=WS + 16), Status.ALIGNMENT),
    (dict(dx=X + 2), Status.ALIGNMENT),
    (dict(Cin=12), Status.UNSUPPORTED),
])
def test_bwd_data_validation(kw, expect):
    assert call_bwd_data(**kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(dw=None), Status.INVALID_ARG),
    (dict(tpad=c3.TPAD_CAUSAL_CACHED), Status.UNSUPPORTED),
    (dict(dbias=B + 4), Status.ALIGNMENT),
    (dict(workspace=None), Status.WORKSPACE),
    (dict(ws_bytes=1024), Status.WORKSPACE),
    (dict(workspace=WS + 128), Status.ALIGNMENT),
    (dict(workspace=X + 4096), Status.INVALID_ARG),        # workspace overlaps x
    (dict(Cout=20), Status.UNSUPPORTED),
])
def test_bwd_weight_validation(kw, expect):
    assert call_bwd_weight(**kw) == expect


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_bwd_entries_without_gpu_report_cuda_error():
    assert call_bwd_data() == Status.CUDA
    assert call_bwd_weight() == Status.CUDA
    assert call_bwd_weight(stride=(2, 2, 2), dbias=None) == Status.CUDA   # strided wgrad is valid


def test_autograd_function_is_exported():
    assert issubclass(c3.Conv3dFunction, torch.autograd.Function)
    assert callable(c3.conv3d_autograd)


def test_arm_stall_rejects_bad_arguments():
    # the failure-detection hook validates before touching anything
    for launches, ms in ((-1, 50), (1, 0), (1, 20000)):
        with pytest.raises(c3.Conv3dError):
            c3.test_arm_stall(launches, ms)
    c3.test_arm_stall(0, 50)


def test_fused_groupnorm_entry_validates_before_any_launch():
    S = 0x600000000      # fake stats, gamma, beta
    args = (X, S, S + 0x10000, S + 0x20000)
    rest = (Wt, B, None, Y, 1, 64, 3, 8, 8, 64, (3, 3, 3), (1, 1, 1), (0, 1, 1))
    assert c3.conv3d_gn_ptr(*args, 8, 0, 1, *rest, c3.TPAD_CAUSAL_CACHED, c3.BF16, None) == \
        Status.UNSUPPORTED
    assert c3.conv3d_gn_ptr(*args, 7, 0, 1, *rest, c3.TPAD_CAUSAL_REPLICATE, c3.BF16, None) == \
        Status.INVALID_ARG                                   # 7 groups do not divide 64
    assert c3.conv3d_gn_ptr(*args, 8, 2, 1, *rest, c3.TPAD_CAUSAL_REPLICATE, c3.BF16, None) == \
        Status.INVALID_ARG                                   # per_frame must be 0 or 1
    bad = (X, S + 4, S + 0x10000, S + 0x20000)
    assert c3.conv3d_gn_ptr(*bad, 8, 0, 1, *rest, c3.TPAD_CAUSAL_REPLICATE, c3.BF16, None) == \
        Status.ALIGNMENT                                     # stats not 8-byte aligned

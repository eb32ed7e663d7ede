"""Python binding of libconv3d: implicit-GEMM 3D convolution on B200 (sm_100a).

Argument marshalling only.  Every step of the convolution runs in the CUDA
library ``libconv3d.so`` (built from ``csrc/`` by ``build.py``); torch is used
here for device memory and streams.  There is no fallback: if the library is
missing or fails to load, importing this package raises.

Operation (engineering.drawthings.ai, "Metal conv3d" post; Qwen Image post,
"Video VAE" section): y = conv3d(x, w) + bias + residual with NDHWC
activations, [Cout, kt, kh, kw, Cin] weights, spatial zero padding, strides
and a temporal padding mode (zero, causal replicate-first-frame, causal zero,
or the cached frames of the previous chunk).  Also: the GroupNorm + SiLU pass
in front of a decoder convolution (groupnorm_stats / groupnorm_silu), the
backward pass (conv3d_bwd_data, conv3d_bwd_weight) and a torch.autograd
wrapper over both directions (Conv3dFunction / conv3d_autograd).  Each call has
a raw-pointer twin (``*_ptr``) that returns the library's status code.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "TPAD_ZERO", "TPAD_CAUSAL_REPLICATE", "TPAD_CAUSAL_ZERO", "TPAD_CAUSAL_CACHED", "F16", "BF16",
    "Status", "Conv3dError", "lib_path", "status_string", "last_error", "kernel_launches",
    "conv3d", "conv3d_fwd", "conv3d_fwd_ptr", "conv3d_fwd_ws_ptr", "conv3d_fwd_noalloc_ptr",
    "conv3d_fwd_cached_ptr", "conv3d_gn", "conv3d_gn_ptr", "output_shape", "workspace_bytes",
    "groupnorm_stats", "groupnorm_silu", "groupnorm_stats_ptr", "groupnorm_silu_ptr",
    "conv3d_bwd_data", "conv3d_bwd_data_ptr", "bwd_data_workspace_bytes",
    "conv3d_bwd_weight", "conv3d_bwd_weight_ptr", "bwd_weight_workspace_bytes",
    "conv3d_bwd_data_cached", "conv3d_bwd_weight_cached",
    "Conv3dFunction", "conv3d_autograd",
    "poll_status", "selftest_wait_timeout", "release", "test_arm_stall",
]

F16 = 0
BF16 = 1
TPAD_ZERO = 0
TPAD_CAUSAL_REPLICATE = 1
TPAD_CAUSAL_ZERO = 2
TPAD_CAUSAL_CACHED = 3


class Status:
    OK = 0
    INVALID_ARG = 1
    UNSUPPORTED = 2
    ALIGNMENT = 3
    CUDA = 4
    TIMEOUT = 5
    DEVICE_CHECK = 6
    WORKSPACE = 7


class Conv3dError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libconv3d status {status}: {message}")
        self.status = status


_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "libconv3d.so")

if not os.path.exists(lib_path):
    raise ImportError(f"{lib_path} is missing: build it with "
                      "`python video_vae_convolution_implicit_b200/build.py` (nvcc, sm_100a)")
_lib = ctypes.CDLL(lib_path)

_i3 = ctypes.c_int * 3
_vp = ctypes.c_void_p
_c = ctypes.c_int

_lib.conv3d_fwd.restype = _c
_lib.conv3d_fwd.argtypes = [_vp] * 5 + [_c] * 6 + [_i3] * 3 + [_c, _c, _vp]
_lib.conv3d_fwd_ws.restype = _c
_lib.conv3d_fwd_ws.argtypes = [_vp] * 5 + [_c] * 6 + [_i3] * 3 + [_c, _c, _vp, ctypes.c_size_t, _vp]
_lib.conv3d_fwd_cached.restype = _c
_lib.conv3d_fwd_cached.argtypes = [_vp] * 6 + [_c] * 6 + [_i3] * 3 + [_c, _vp]
_lib.conv3d_groupnorm_stats.restype = _c
_lib.conv3d_groupnorm_stats.argtypes = [_vp] + [_c] * 7 + [ctypes.c_float, _c, _vp, _vp]
_lib.conv3d_groupnorm_silu.restype = _c
_lib.conv3d_groupnorm_silu.argtypes = [_vp] * 5 + [_c] * 8 + [_c, _vp]
_lib.conv3d_bwd_data.restype = _c
_lib.conv3d_bwd_data.argtypes = [_vp] * 3 + [_c] * 6 + [_i3] * 3 + [_c, _c, _vp, ctypes.c_size_t,
                                                                   _vp]
_lib.conv3d_bwd_data_workspace_bytes.restype = ctypes.c_size_t
_lib.conv3d_bwd_data_workspace_bytes.argtypes = [_c] * 6 + [_i3, _i3, _c]
_lib.conv3d_bwd_weight.restype = _c
_lib.conv3d_bwd_weight.argtypes = [_vp] * 4 + [_c] * 6 + [_i3] * 3 + [_c, _c, _vp,
                                                                     ctypes.c_size_t, _vp]
_lib.conv3d_bwd_data_cached.restype = _c
_lib.conv3d_bwd_data_cached.argtypes = [_vp] * 4 + [_c] * 6 + [_i3] * 3 + [_c, _vp, ctypes.c_size_t,
                                                                          _vp]
_lib.conv3d_bwd_weight_cached.restype = _c
_lib.conv3d_bwd_weight_cached.argtypes = [_vp] * 5 + [_c] * 6 + [_i3] * 3 + [_c, _vp,
                                                                            ctypes.c_size_t, _vp]
_lib.conv3d_bwd_weight_workspace_bytes.restype = ctypes.c_size_t
_lib.conv3d_bwd_weight_workspace_bytes.argtypes = [_c, _c, _i3]
_lib.conv3d_fwd_noalloc.restype = _c
_lib.conv3d_fwd_noalloc.argtypes = [_vp] * 5 + [_c] * 6 + [_i3] * 3 + [_c, _c, _vp]
_lib.conv3d_workspace_bytes.restype = ctypes.c_size_t
_lib.conv3d_workspace_bytes.argtypes = [_c, _c, _i3, _c, _c]
_lib.conv3d_output_shape.restype = _c
_lib.conv3d_output_shape.argtypes = [_c, _c, _c, _i3, _i3, _i3, _c, _i3]
_lib.conv3d_poll_status.restype = _c
_lib.conv3d_poll_status.argtypes = [_vp]
_lib.conv3d_status_string.restype = ctypes.c_char_p
_lib.conv3d_status_string.argtypes = [_c]
_lib.conv3d_last_error.restype = ctypes.c_char_p
_lib.conv3d_last_error.argtypes = []
_lib.conv3d_kernel_launches.restype = ctypes.c_ulonglong
_lib.conv3d_kernel_launches.argtypes = []
_lib.conv3d_release.restype = None
_lib.conv3d_release.argtypes = []
_lib.conv3d_selftest_wait_timeout.restype = _c
_lib.conv3d_selftest_wait_timeout.argtypes = [_c]
_lib.conv3d_fwd_gn.restype = _c
_lib.conv3d_fwd_gn.argtypes = ([_vp, _vp, _vp, _vp, _c, _c, _c] + [_vp] * 4 + [_c] * 6 + [_i3] * 3
                                + [_c, _c, _vp, _c, ctypes.c_float, _vp])
_lib.conv3d_test_arm_stall.restype = _c
_lib.conv3d_test_arm_stall.argtypes = [_c, _c]


def raw_library() -> ctypes.CDLL:
    """The loaded ctypes handle of libconv3d.so."""
    return _lib


def status_string(status: int) -> str:
    return _lib.conv3d_status_string(status).decode()


def last_error() -> str:
    return _lib.conv3d_last_error().decode()


def kernel_launches() -> int:
    """GPU kernels the library has launched in this process (counted at enqueue)."""
    return int(_lib.conv3d_kernel_launches())


def _check(status: int) -> None:
    if status != Status.OK:
        raise Conv3dError(status, f"{status_string(status)}: {last_error()}")


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t == torch.float16:
        return F16
    raise TypeError(f"libconv3d computes in bf16 or fp16, got {t}")


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def output_shape(D, H, W, kernel, stride=(1, 1, 1), pad=(0, 1, 1), tpad=TPAD_CAUSAL_REPLICATE):
    out = _i3()
    _check(_lib.conv3d_output_shape(D, H, W, _i3(*kernel), _i3(*stride), _i3(*pad), tpad, out))
    return tuple(out)


def workspace_bytes(Cin, Cout, kernel, D, tpad) -> int:
    return int(_lib.conv3d_workspace_bytes(Cin, Cout, _i3(*kernel), D, tpad))


def conv3d_fwd_ptr(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride, pad, tpad,
                   dtype, stream) -> int:
    """Raw-pointer call of conv3d_fwd; returns the status code (no raise)."""
    return _lib.conv3d_fwd(x, w, bias, residual, y, N, Cin, D, H, W, Cout, _i3(*kernel),
                           _i3(*stride), _i3(*pad), tpad, dtype, stream)


def conv3d_fwd_ws_ptr(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride, pad, tpad,
                      dtype, workspace, ws_bytes, stream) -> int:
    """Raw-pointer call of conv3d_fwd_ws; returns the status code (no raise)."""
    return _lib.conv3d_fwd_ws(x, w, bias, residual, y, N, Cin, D, H, W, Cout, _i3(*kernel),
                              _i3(*stride), _i3(*pad), tpad, dtype, workspace, ws_bytes, stream)


def conv3d_fwd_noalloc_ptr(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride, pad,
                           tpad, dtype, stream) -> int:
    """Raw-pointer call of conv3d_fwd_noalloc (for callers that cannot allocate
    device memory; its first-frame scratch is a fixed 16 MiB array inside the
    library).  Returns the status code (no raise)."""
    return _lib.conv3d_fwd_noalloc(x, w, bias, residual, y, N, Cin, D, H, W, Cout, _i3(*kernel),
                                   _i3(*stride), _i3(*pad), tpad, dtype, stream)


def conv3d_fwd_cached_ptr(x, prev, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride,
                          pad, dtype, stream) -> int:
    """Raw-pointer call of conv3d_fwd_cached (one chunk of a causal conv whose
    front padding is the previous chunk's last kt-1 frames).  Returns the status."""
    return _lib.conv3d_fwd_cached(x, prev, w, bias, residual, y, N, Cin, D, H, W, Cout,
                                  _i3(*kernel), _i3(*stride), _i3(*pad), dtype, stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def conv3d_fwd(x: torch.Tensor, w: torch.Tensor, bias, residual, y: torch.Tensor,
               stride=(1, 1, 1), pad=(0, 1, 1), tpad=TPAD_CAUSAL_REPLICATE, stream=None,
               workspace: torch.Tensor | None = None, prev: torch.Tensor | None = None
               ) -> torch.Tensor:
    """Enqueue y = conv3d(x, w) + bias + residual on ``stream`` (default: current stream).

    x: [N, D, H, W, Cin]; w: [Cout, kt, kh, kw, Cin]; bias: [Cout] or None;
    residual: y's shape or None; y: [N, Do, Ho, Wo, Cout].  All contiguous CUDA
    tensors of one dtype (bf16 or fp16).  With ``workspace`` (a uint8 CUDA
    tensor) the call goes through conv3d_fwd_ws and never allocates.  With
    tpad=TPAD_CAUSAL_CACHED, ``prev`` ([N, kt-1, H, W, Cin]) holds the frames
    before x and the call goes through conv3d_fwd_cached.
    """
    for name, t in (("x", x), ("w", w), ("y", y), ("bias", bias), ("residual", residual),
                    ("prev", prev)):
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dtype != x.dtype:
            raise TypeError(f"{name} has dtype {t.dtype}, x has {x.dtype}")
    if x.dim() != 5 or w.dim() != 5:
        raise ValueError("x must be [N,D,H,W,Cin] and w [Cout,kt,kh,kw,Cin]")
    N, D, H, W, Cin = x.shape
    Cout, kt, kh, kw, Cin_w = w.shape
    if Cin_w != Cin:
        raise ValueError("w's last extent must equal Cin")
    out = output_shape(D, H, W, (kt, kh, kw), stride, pad, tpad)
    if tuple(y.shape) != (N, *out, Cout):
        raise ValueError(f"y must be {(N, *out, Cout)}, got {tuple(y.shape)}")
    if residual is not None and tuple(residual.shape) != tuple(y.shape):
        raise ValueError("residual must have y's shape")
    if bias is not None and tuple(bias.shape) != (Cout,):
        raise ValueError("bias must be [Cout]")
    code = _dtype_code(x.dtype)
    s = _stream_handle(stream)
    if tpad == TPAD_CAUSAL_CACHED:
        if prev is not None and tuple(prev.shape) != (N, kt - 1, H, W, Cin):
            raise ValueError(f"prev must be {(N, kt - 1, H, W, Cin)}")
        st = conv3d_fwd_cached_ptr(_ptr(x), _ptr(prev), _ptr(w), _ptr(bias), _ptr(residual),
                                   _ptr(y), N, Cin, D, H, W, Cout, (kt, kh, kw), stride, pad, code,
                                   s)
    elif workspace is None:
        st = conv3d_fwd_ptr(_ptr(x), _ptr(w), _ptr(bias), _ptr(residual), _ptr(y), N, Cin, D, H,
                            W, Cout, (kt, kh, kw), stride, pad, tpad, code, s)
    else:
        st = conv3d_fwd_ws_ptr(_ptr(x), _ptr(w), _ptr(bias), _ptr(residual), _ptr(y), N, Cin, D,
                               H, W, Cout, (kt, kh, kw), stride, pad, tpad, code,
                               _ptr(workspace), workspace.numel() * workspace.element_size(), s)
    _check(st)
    return y


def conv3d(x: torch.Tensor, w: torch.Tensor, bias=None, residual=None, stride=(1, 1, 1),
           pad=(0, 1, 1), tpad=TPAD_CAUSAL_REPLICATE, stream=None, prev=None) -> torch.Tensor:
    """Allocate y (torch) and run :func:`conv3d_fwd`."""
    N, D, H, W, _ = x.shape
    Cout, kt, kh, kw, _ = w.shape
    out = output_shape(D, H, W, (kt, kh, kw), stride, pad, tpad)
    y = torch.empty((N, *out, Cout), dtype=x.dtype, device=x.device)
    return conv3d_fwd(x, w, bias, residual, y, stride, pad, tpad, stream, prev=prev)


def conv3d_gn_ptr(x, stats, gamma, beta, groups, per_frame, apply_silu, w, bias, residual, y, N,
                  Cin, D, H, W, Cout, kernel, stride, pad, tpad, dtype, stream, out_stats=None,
                  out_groups=0, out_eps=1e-6) -> int:
    """Raw-pointer call of conv3d_fwd_gn; returns the status code (no raise)."""
    return _lib.conv3d_fwd_gn(x, stats, gamma, beta, groups, int(per_frame), int(apply_silu), w,
                              bias, residual, y, N, Cin, D, H, W, Cout, _i3(*kernel),
                              _i3(*stride), _i3(*pad), tpad, dtype, out_stats, int(out_groups),
                              float(out_eps), stream)


def conv3d_gn(x: torch.Tensor, stats, gamma, beta, w: torch.Tensor, bias=None,
              residual=None, y: torch.Tensor | None = None, groups: int | None = None,
              per_frame: bool = False, apply_silu: bool = True, stride=(1, 1, 1), pad=(0, 1, 1),
              tpad=TPAD_CAUSAL_REPLICATE, out_groups: int = 0, out_eps: float = 1e-6,
              stream=None):
    """y = conv3d(silu(GroupNorm(x)), w) + bias + residual with the GroupNorm + SiLU
    applied as the convolution reads x (``stats`` from groupnorm_stats over x, or
    None for plain x).  With ``out_groups`` > 0 also returns the per-sample
    GroupNorm statistics of y ([N, out_groups, 2] float64): (y, out_stats)."""
    N, D, H, W, Cin = x.shape
    Cout, kt, kh, kw, _ = w.shape
    groups = (stats.shape[1] if stats is not None else 1) if groups is None else groups
    if y is None:
        out = output_shape(D, H, W, (kt, kh, kw), stride, pad, tpad)
        y = torch.empty((N, *out, Cout), dtype=x.dtype, device=x.device)
    for name, t in (("x", x), ("w", w), ("y", y)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
            raise ValueError(f"{name} must be a contiguous CUDA tensor of x's dtype")
    if stats is not None and (stats.dtype != torch.float64 or not stats.is_cuda):
        raise ValueError("stats must be a float64 CUDA tensor")
    out_stats = (torch.empty((N, out_groups, 2), dtype=torch.float64, device=x.device)
                 if out_groups > 0 else None)
    _check(conv3d_gn_ptr(x.data_ptr(), _ptr(stats), _ptr(gamma), _ptr(beta), groups,
                         per_frame, apply_silu, w.data_ptr(), _ptr(bias), _ptr(residual),
                         y.data_ptr(), N, Cin, D, H, W, Cout, (kt, kh, kw), stride, pad, tpad,
                         _dtype_code(x.dtype), _stream_handle(stream), _ptr(out_stats), out_groups,
                         out_eps))
    return (y, out_stats) if out_stats is not None else y


def poll_status(stream=None) -> int:
    """Synchronise ``stream`` and return (and clear) the device status word."""
    return int(_lib.conv3d_poll_status(_stream_handle(stream)))


def selftest_wait_timeout(timeout_ms: int) -> int:
    """Run the bounded-wait self test; returns Status.TIMEOUT when it works."""
    return int(_lib.conv3d_selftest_wait_timeout(timeout_ms))


def release() -> None:
    _lib.conv3d_release()


def test_arm_stall(launches: int, timeout_ms: int = 50) -> None:
    """Failure-detection test hook: the next ``launches`` convolution-kernel
    launches stall on their first pipeline stage and abort after ``timeout_ms``
    (poll_status then returns Status.TIMEOUT).  0 disarms."""
    _check(_lib.conv3d_test_arm_stall(int(launches), int(timeout_ms)))


def groupnorm_stats_ptr(x, N, D, H, W, C, groups, per_frame, eps, dtype, stats, stream) -> int:
    """Raw-pointer call of conv3d_groupnorm_stats; returns the status code."""
    return _lib.conv3d_groupnorm_stats(x, N, D, H, W, C, groups, int(per_frame), eps, dtype, stats,
                                       stream)


def groupnorm_silu_ptr(x, stats, gamma, beta, y, N, D, H, W, C, groups, per_frame, apply_silu,
                       dtype, stream) -> int:
    """Raw-pointer call of conv3d_groupnorm_silu; returns the status code."""
    return _lib.conv3d_groupnorm_silu(x, stats, gamma, beta, y, N, D, H, W, C, groups,
                                      int(per_frame), int(apply_silu), dtype, stream)


def groupnorm_stats(x: torch.Tensor, groups: int, eps: float = 1e-6, per_frame: bool = False,
                    stats: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """{mean, 1/sqrt(var+eps)} per (sample [, frame], group) of an NDHWC tensor, as a
    float64 CUDA tensor [sets, groups, 2] (``stats`` is reused when given)."""
    if not x.is_cuda or not x.is_contiguous() or x.dim() != 5:
        raise ValueError("x must be a contiguous CUDA tensor [N, D, H, W, C]")
    N, D, H, W, C = x.shape
    sets = N * D if per_frame else N
    if stats is None:
        stats = torch.empty((sets, groups, 2), dtype=torch.float64, device=x.device)
    elif tuple(stats.shape) != (sets, groups, 2) or stats.dtype != torch.float64:
        raise ValueError(f"stats must be float64 {(sets, groups, 2)}")
    _check(groupnorm_stats_ptr(x.data_ptr(), N, D, H, W, C, groups, per_frame, eps,
                               _dtype_code(x.dtype), stats.data_ptr(), _stream_handle(stream)))
    return stats


def groupnorm_silu(x: torch.Tensor, stats: torch.Tensor, gamma=None, beta=None, y=None,
                   groups: int | None = None, per_frame: bool = False, apply_silu: bool = True,
                   stream=None) -> torch.Tensor:
    """y = silu((x - mean) * rstd * gamma + beta) with ``stats`` from groupnorm_stats.
    ``y`` may be ``x`` (in place); it is allocated when None."""
    if not x.is_cuda or not x.is_contiguous() or x.dim() != 5:
        raise ValueError("x must be a contiguous CUDA tensor [N, D, H, W, C]")
    N, D, H, W, C = x.shape
    groups = stats.shape[1] if groups is None else groups
    if y is None:
        y = torch.empty_like(x)
    for name, t in (("gamma", gamma), ("beta", beta)):
        if t is not None and (tuple(t.shape) != (C,) or t.dtype != x.dtype or not t.is_cuda):
            raise ValueError(f"{name} must be a CUDA [C] tensor of x's dtype")
    _check(groupnorm_silu_ptr(x.data_ptr(), stats.data_ptr(), _ptr(gamma), _ptr(beta),
                              y.data_ptr(), N, D, H, W, C, groups, per_frame, apply_silu,
                              _dtype_code(x.dtype), _stream_handle(stream)))
    return y


def conv3d_bwd_data_ptr(dy, w, dx, N, Cin, D, H, W, Cout, kernel, stride, pad, tpad, dtype,
                        workspace, ws_bytes, stream) -> int:
    """Raw-pointer call of conv3d_bwd_data; returns the status code."""
    return _lib.conv3d_bwd_data(dy, w, dx, N, Cin, D, H, W, Cout, _i3(*kernel), _i3(*stride),
                                _i3(*pad), tpad, dtype, workspace, ws_bytes, stream)


def bwd_data_workspace_bytes(N, Cin, D, H, W, Cout, kernel, pad, tpad) -> int:
    return int(_lib.conv3d_bwd_data_workspace_bytes(N, Cin, D, H, W, Cout, _i3(*kernel), _i3(*pad),
                                                    tpad))


def conv3d_bwd_data(dy: torch.Tensor, w: torch.Tensor, x_shape, pad=(0, 1, 1),
                    tpad=TPAD_CAUSAL_REPLICATE, dx: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream=None,
                    stride=(1, 1, 1)) -> torch.Tensor:
    """dx for the forward problem x [x_shape] -> y (dy has y's shape); temporal
    stride 1, spatial strides up to 8."""
    N, D, H, W, Cin = x_shape
    Cout, kt, kh, kw, _ = w.shape
    if dx is None:
        dx = torch.empty(tuple(x_shape), dtype=dy.dtype, device=dy.device)
    need = bwd_data_workspace_bytes(N, Cin, D, H, W, Cout, (kt, kh, kw), pad, tpad)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dy.device)
    for name, t in (("dy", dy), ("w", w), ("dx", dx)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != dy.dtype:
            raise ValueError(f"{name} must be a contiguous CUDA tensor of dy's dtype")
    _check(conv3d_bwd_data_ptr(dy.data_ptr(), w.data_ptr(), dx.data_ptr(), N, Cin, D, H, W, Cout,
                               (kt, kh, kw), tuple(stride), pad, tpad, _dtype_code(dy.dtype),
                               workspace.data_ptr(), workspace.numel(), _stream_handle(stream)))
    return dx


def conv3d_bwd_weight_ptr(x, dy, dw, dbias, N, Cin, D, H, W, Cout, kernel, stride, pad, tpad,
                          dtype, workspace, ws_bytes, stream) -> int:
    """Raw-pointer call of conv3d_bwd_weight; returns the status code."""
    return _lib.conv3d_bwd_weight(x, dy, dw, dbias, N, Cin, D, H, W, Cout, _i3(*kernel),
                                  _i3(*stride), _i3(*pad), tpad, dtype, workspace, ws_bytes,
                                  stream)


def bwd_weight_workspace_bytes(Cin, Cout, kernel) -> int:
    return int(_lib.conv3d_bwd_weight_workspace_bytes(Cin, Cout, _i3(*kernel)))


def conv3d_bwd_weight(x: torch.Tensor, dy: torch.Tensor, kernel, stride=(1, 1, 1), pad=(0, 1, 1),
                      tpad=TPAD_CAUSAL_REPLICATE, with_bias: bool = True,
                      workspace: torch.Tensor | None = None, stream=None):
    """(dw, dbias) for the forward problem x -> y with upstream gradient dy."""
    N, D, H, W, Cin = x.shape
    Cout = dy.shape[-1]
    dw = torch.empty((Cout, *kernel, Cin), dtype=x.dtype, device=x.device)
    db = torch.empty((Cout,), dtype=x.dtype, device=x.device) if with_bias else None
    need = bwd_weight_workspace_bytes(Cin, Cout, kernel)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    for name, t in (("x", x), ("dy", dy)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
            raise ValueError(f"{name} must be a contiguous CUDA tensor of x's dtype")
    _check(conv3d_bwd_weight_ptr(x.data_ptr(), dy.data_ptr(), dw.data_ptr(), _ptr(db), N, Cin, D,
                                 H, W, Cout, tuple(kernel), stride, pad, tpad,
                                 _dtype_code(x.dtype), workspace.data_ptr(), workspace.numel(),
                                 _stream_handle(stream)))
    return dw, db


def conv3d_bwd_data_cached(dy: torch.Tensor, w: torch.Tensor, x_shape, pad=(0, 1, 1),
                           with_prev: bool = True, workspace: torch.Tensor | None = None,
                           stream=None):
    """(dx, dprev) for one chunk of the cached-frames mode (stride 1): dprev is
    the gradient of the kt-1 cached frames (None when with_prev is false)."""
    N, D, H, W, Cin = x_shape
    Cout, kt, kh, kw, _ = w.shape
    dx = torch.empty(tuple(x_shape), dtype=dy.dtype, device=dy.device)
    dprev = (torch.empty((N, kt - 1, H, W, Cin), dtype=dy.dtype, device=dy.device)
             if with_prev and kt > 1 else None)
    need = bwd_data_workspace_bytes(N, Cin, D, H, W, Cout, (kt, kh, kw), pad, TPAD_CAUSAL_CACHED)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dy.device)
    for name, t in (("dy", dy), ("w", w)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != dy.dtype:
            raise ValueError(f"{name} must be a contiguous CUDA tensor of dy's dtype")
    _check(_lib.conv3d_bwd_data_cached(dy.data_ptr(), w.data_ptr(), dx.data_ptr(), _ptr(dprev), N,
                                       Cin, D, H, W, Cout, _i3(kt, kh, kw), _i3(1, 1, 1),
                                       _i3(*pad), _dtype_code(dy.dtype), workspace.data_ptr(),
                                       workspace.numel(), _stream_handle(stream)))
    return dx, dprev


def conv3d_bwd_weight_cached(x: torch.Tensor, prev: torch.Tensor | None, dy: torch.Tensor, kernel,
                             stride=(1, 1, 1), pad=(0, 1, 1), with_bias: bool = True,
                             workspace: torch.Tensor | None = None, stream=None):
    """(dw, dbias) for one chunk of the cached-frames mode; prev: the cached frames."""
    N, D, H, W, Cin = x.shape
    Cout = dy.shape[-1]
    dw = torch.empty((Cout, *kernel, Cin), dtype=x.dtype, device=x.device)
    db = torch.empty((Cout,), dtype=x.dtype, device=x.device) if with_bias else None
    need = bwd_weight_workspace_bytes(Cin, Cout, kernel)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    for name, t in (("x", x), ("dy", dy), ("prev", prev)):
        if t is not None and (not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype):
            raise ValueError(f"{name} must be a contiguous CUDA tensor of x's dtype")
    _check(_lib.conv3d_bwd_weight_cached(x.data_ptr(), _ptr(prev), dy.data_ptr(), dw.data_ptr(),
                                         _ptr(db), N, Cin, D, H, W, Cout, _i3(*kernel),
                                         _i3(*stride), _i3(*pad), _dtype_code(x.dtype),
                                         workspace.data_ptr(), workspace.numel(),
                                         _stream_handle(stream)))
    return dw, db


class Conv3dFunction(torch.autograd.Function):
    """torch.autograd wrapper: forward through conv3d_fwd, backward through
    conv3d_bwd_data (dx; temporal stride 1) and conv3d_bwd_weight (dw, dbias).
    The residual's gradient is dy itself.  Marshalling only: every product runs
    in the library's kernels, none in torch."""

    @staticmethod
    def forward(ctx, x, w, bias, residual, stride, pad, tpad):
        y = conv3d(x, w, bias, residual, stride, pad, tpad)
        ctx.save_for_backward(x, w)
        ctx.conf = (tuple(stride), tuple(pad), tpad, bias is not None, residual is not None)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, w = ctx.saved_tensors
        stride, pad, tpad, has_bias, has_res = ctx.conf
        dy = dy.contiguous()
        dx = dw = db = dres = None
        if ctx.needs_input_grad[0]:
            if stride[0] != 1:
                raise NotImplementedError("the input gradient supports temporal stride 1 only")
            dx = conv3d_bwd_data(dy, w, x.shape, pad, tpad, stride=stride)
        if ctx.needs_input_grad[1] or (has_bias and ctx.needs_input_grad[2]):
            dw, db = conv3d_bwd_weight(x, dy, tuple(w.shape[1:4]), stride, pad, tpad,
                                       with_bias=has_bias)
            if not ctx.needs_input_grad[1]:
                dw = None
        if has_res and ctx.needs_input_grad[3]:
            dres = dy
        return dx, dw, db, dres, None, None, None


def conv3d_autograd(x, w, bias=None, residual=None, stride=(1, 1, 1), pad=(0, 1, 1),
                    tpad=TPAD_CAUSAL_REPLICATE):
    """y = conv3d(x, w) + bias + residual with gradients for x, w, bias and residual."""
    return Conv3dFunction.apply(x, w, bias, residual, tuple(stride), tuple(pad), tpad)

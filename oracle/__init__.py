"""CPU oracle for the 3D convolution -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct fp64 definition that the
CUDA library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the library package
never does, and the two share no code.

The arithmetic lives in ``conv3d_oracle.c`` (compiled with gcc and OpenMP by
:func:`build`); this module only marshals numpy arrays through ctypes.

Citations (page title, section):
  * engineering.drawthings.ai, "Metal conv3d" post -- conv3d computed as an
    implicit GEMM "similar to 2D convolution": the result is the plain
    convolution sum, which is what the oracle evaluates directly.
  * engineering.drawthings.ai, Qwen Image post, "Video VAE" -- causal 3D
    convolution whose frames before the first are padding (zero for Wan);
    a first-frame 3D conv reduces to a 2D conv with adjusted weights.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(brute force, closed forms, invariants and a library cross-check); the pages
print no worked numeric example, so no pin comes from printed page values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "conv3d_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_conv3d.so")

F16 = 0
BF16 = 1
TPAD_ZERO = 0
TPAD_CAUSAL_REPLICATE = 1
TPAD_CAUSAL_ZERO = 2
TPAD_CAUSAL_CACHED = 3

_lib = None


def build(force: bool = False) -> str:
    """Compile conv3d_oracle.c into liboracle_conv3d.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64p = ctypes.POINTER(ctypes.c_int64)
        u16p = ctypes.c_void_p
        lib.oracle_conv3d_f64.restype = ctypes.c_int
        lib.oracle_conv3d_f64.argtypes = (
            [u16p, u16p, u16p, u16p, u16p, ctypes.c_int]
            + [ctypes.c_int] * 16
            + [i64p, ctypes.c_int64, ctypes.c_void_p]
        )
        lib.oracle_output_shape.restype = ctypes.c_int
        lib.oracle_output_shape.argtypes = [ctypes.c_int] * 13 + [ctypes.POINTER(ctypes.c_int)]
        lib.oracle_decode16.restype = None
        lib.oracle_decode16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_conv3d_backward_f64.restype = ctypes.c_int
        lib.oracle_conv3d_backward_f64.argtypes = (
            [u16p, u16p, u16p, ctypes.c_int] + [ctypes.c_int] * 16
            + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p])
        lib.oracle_conv3d_backward_cached_f64.restype = ctypes.c_int
        lib.oracle_conv3d_backward_cached_f64.argtypes = (
            [u16p, u16p, u16p, u16p, ctypes.c_int] + [ctypes.c_int] * 14
            + [ctypes.c_void_p] * 4)
        for fn in (lib.oracle_conv3d_dx_at_f64, lib.oracle_conv3d_dw_at_f64):
            fn.restype = ctypes.c_int
            fn.argtypes = ([u16p, u16p, ctypes.c_int] + [ctypes.c_int] * 16
                           + [i64p, ctypes.c_int64, ctypes.c_void_p])
        lib.oracle_groupnorm_silu_f64.restype = ctypes.c_int
        lib.oracle_groupnorm_silu_f64.argtypes = (
            [u16p, u16p, u16p] + [ctypes.c_int] * 8 + [ctypes.c_double, ctypes.c_int, ctypes.c_void_p])
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def decode16(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Exact decode of 16-bit patterns (bf16 or fp16) to float64."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_decode16(bits.ctypes.data, out.ctypes.data, bits.size, dtype)
    return out


def output_shape(D, H, W, kernel, stride, pad, tpad):
    """(Do, Ho, Wo) for the padding rule of ``tpad`` (see conv3d_oracle.c)."""
    out = (ctypes.c_int * 3)()
    rc = _load().oracle_output_shape(D, H, W, *kernel, *stride, *pad, tpad, out)
    if rc != 0:
        raise ValueError("ill-formed convolution shape")
    return tuple(out)


def conv3d(x_bits, w_bits, bias_bits, res_bits, dtype, kernel, stride, pad, tpad, rows=None,
           prev_bits=None):
    """fp64 oracle convolution.

    x_bits: uint16 [N,D,H,W,Cin]; w_bits: uint16 [Cout,kt,kh,kw,Cin];
    bias_bits: uint16 [Cout] or None; res_bits: uint16 [N,Do,Ho,Wo,Cout] or None;
    prev_bits: uint16 [N,kt-1,H,W,Cin], the cached frames before x (mode 3 only).
    rows: optional int64 array of flat output-pixel indices m; when given the
    result is [len(rows), Cout], else [N,Do,Ho,Wo,Cout].  Unrounded float64.
    """
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    N, D, H, W, Cin = x_bits.shape
    Cout, kt, kh, kw, Cin_w = w_bits.shape
    if Cin_w != Cin or tuple(kernel) != (kt, kh, kw):
        raise ValueError("weight shape does not match x / kernel")
    Do, Ho, Wo = output_shape(D, H, W, kernel, stride, pad, tpad)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    r = None if res_bits is None else np.ascontiguousarray(res_bits, dtype=np.uint16)
    if b is not None and b.shape != (Cout,):
        raise ValueError("bias shape")
    if r is not None and r.shape != (N, Do, Ho, Wo, Cout):
        raise ValueError("residual shape")
    pv = None
    if tpad == TPAD_CAUSAL_CACHED and kt > 1:
        if prev_bits is None:
            raise ValueError("the cached mode needs prev")
        pv = np.ascontiguousarray(prev_bits, dtype=np.uint16)
        if pv.shape != (N, kt - 1, H, W, Cin):
            raise ValueError("prev shape")
    if rows is None:
        out = np.empty((N, Do, Ho, Wo, Cout), dtype=np.float64)
        rows_p, n_rows = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.empty((rows.size, Cout), dtype=np.float64)
        rows_p, n_rows = rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), rows.size
    rc = _load().oracle_conv3d_f64(
        x_bits.ctypes.data, None if pv is None else pv.ctypes.data, w_bits.ctypes.data,
        None if b is None else b.ctypes.data,
        None if r is None else r.ctypes.data,
        dtype, N, Cin, D, H, W, Cout, kt, kh, kw, *stride, *pad, tpad,
        rows_p, n_rows, out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return out


def groupnorm_silu(x_bits, gamma_bits, beta_bits, dtype, groups, eps=1e-6, per_frame=False,
                   silu=True):
    """fp64 GroupNorm (+ SiLU) of a [N,D,H,W,C] tensor of 16-bit patterns.

    Statistics per (sample, group), or per (sample, frame, group) with
    per_frame.  gamma/beta: [C] patterns or None.  Returns unrounded float64.
    """
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    N, D, H, W, C = x_bits.shape
    g = None if gamma_bits is None else np.ascontiguousarray(gamma_bits, dtype=np.uint16)
    b = None if beta_bits is None else np.ascontiguousarray(beta_bits, dtype=np.uint16)
    out = np.empty(x_bits.shape, dtype=np.float64)
    rc = _load().oracle_groupnorm_silu_f64(
        x_bits.ctypes.data, None if g is None else g.ctypes.data,
        None if b is None else b.ctypes.data, dtype, N, D, H, W, C, groups, int(per_frame),
        float(eps), int(silu), out.ctypes.data)
    if rc != 0:
        raise ValueError("channels must be a multiple of groups")
    return out


def conv3d_backward(x_bits, w_bits, dy_bits, dtype, kernel, stride, pad, tpad):
    """fp64 adjoints of :func:`conv3d` for the upstream gradient ``dy_bits``
    (y's shape): returns (dx [N,D,H,W,Cin], dw [Cout,kt,kh,kw,Cin], dbias [Cout])."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    dy_bits = np.ascontiguousarray(dy_bits, dtype=np.uint16)
    N, D, H, W, Cin = x_bits.shape
    Cout = w_bits.shape[0]
    Do, Ho, Wo = output_shape(D, H, W, kernel, stride, pad, tpad)
    if dy_bits.shape != (N, Do, Ho, Wo, Cout):
        raise ValueError("dy shape")
    dx = np.empty(x_bits.shape, dtype=np.float64)
    dw = np.empty(w_bits.shape, dtype=np.float64)
    db = np.empty((Cout,), dtype=np.float64)
    rc = _load().oracle_conv3d_backward_f64(
        x_bits.ctypes.data, w_bits.ctypes.data, dy_bits.ctypes.data, dtype, N, Cin, D, H, W, Cout,
        *kernel, *stride, *pad, tpad, dx.ctypes.data, dw.ctypes.data, db.ctypes.data)
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return dx, dw, db


def conv3d_backward_cached(x_bits, prev_bits, w_bits, dy_bits, dtype, kernel, stride, pad):
    """fp64 adjoints of :func:`conv3d` in the cached-frames mode (prev_bits the
    previous chunk's last kt-1 frames [N, kt-1, H, W, Cin]): returns
    (dx, dprev, dw, dbias)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    dy_bits = np.ascontiguousarray(dy_bits, dtype=np.uint16)
    N, D, H, W, Cin = x_bits.shape
    Cout = w_bits.shape[0]
    kt = kernel[0]
    if prev_bits is not None:
        prev_bits = np.ascontiguousarray(prev_bits, dtype=np.uint16)
        if prev_bits.shape != (N, kt - 1, H, W, Cin):
            raise ValueError("prev shape")
    Do, Ho, Wo = output_shape(D, H, W, kernel, stride, pad, TPAD_CAUSAL_CACHED)
    if dy_bits.shape != (N, Do, Ho, Wo, Cout):
        raise ValueError("dy shape")
    dx = np.empty(x_bits.shape, dtype=np.float64)
    dprev = np.zeros((N, kt - 1, H, W, Cin), dtype=np.float64)
    dw = np.empty(w_bits.shape, dtype=np.float64)
    db = np.empty((Cout,), dtype=np.float64)
    rc = _load().oracle_conv3d_backward_cached_f64(
        x_bits.ctypes.data, None if prev_bits is None else prev_bits.ctypes.data,
        w_bits.ctypes.data, dy_bits.ctypes.data, dtype, N, Cin, D, H, W, Cout, *kernel, *stride,
        pad[1], pad[2], dx.ctypes.data, dprev.ctypes.data if kt > 1 else None, dw.ctypes.data,
        db.ctypes.data)
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return dx, dprev, dw, db


def conv3d_dx_at(w_bits, dy_bits, dtype, x_shape, kernel, stride, pad, tpad, pixels):
    """fp64 dx at the given flat input pixels ((n*D + f)*H + h)*W + w: [len, Cin]."""
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    dy_bits = np.ascontiguousarray(dy_bits, dtype=np.uint16)
    N, D, H, W, Cin = x_shape
    Cout = w_bits.shape[0]
    if dy_bits.shape != (N, *output_shape(D, H, W, kernel, stride, pad, tpad), Cout):
        raise ValueError("dy shape")
    pixels = np.ascontiguousarray(pixels, dtype=np.int64)
    out = np.empty((pixels.size, Cin), dtype=np.float64)
    rc = _load().oracle_conv3d_dx_at_f64(
        w_bits.ctypes.data, dy_bits.ctypes.data, dtype, N, Cin, D, H, W, Cout, *kernel, *stride,
        *pad, tpad, pixels.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), pixels.size,
        out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return out


def conv3d_dw_at(x_bits, dy_bits, dtype, Cout, kernel, stride, pad, tpad, entries):
    """fp64 dw at the given flat indices into [Cout, kt, kh, kw, Cin]: [len]."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    dy_bits = np.ascontiguousarray(dy_bits, dtype=np.uint16)
    N, D, H, W, Cin = x_bits.shape
    if dy_bits.shape != (N, *output_shape(D, H, W, kernel, stride, pad, tpad), Cout):
        raise ValueError("dy shape")
    entries = np.ascontiguousarray(entries, dtype=np.int64)
    out = np.empty(entries.size, dtype=np.float64)
    rc = _load().oracle_conv3d_dw_at_f64(
        x_bits.ctypes.data, dy_bits.ctypes.data, dtype, N, Cin, D, H, W, Cout, *kernel, *stride,
        *pad, tpad, entries.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), entries.size,
        out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return out

"""Shared helpers for the GPU-vs-oracle parity tests.

The tolerance is the one fixed for bf16/fp16 inputs with fp32 accumulation:
    max |y - y_ref| <= 1e-2 * max |y_ref|
    sum |y - y_ref| / sum |y_ref| <= 2e-3            (mean relative error, L1 form)
y_ref is the oracle's unrounded fp64 result on the same 16-bit inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import seeded_inputs as si

MAX_REL = 1e-2
MEAN_REL = 2e-3

TORCH_DTYPE = {"bf16": torch.bfloat16, "f16": torch.float16}
ORACLE_DTYPE = {"bf16": oracle.BF16, "f16": oracle.F16}


def problem(N, Cin, D, H, W, Cout, kernel, pad, tpad, seed, dtype="bf16", bias=True,
            residual=False, device="cuda", stride=(1, 1, 1)):
    out = oracle.output_shape(D, H, W, kernel, stride, pad, tpad)
    cached = tpad == oracle.TPAD_CAUSAL_CACHED
    p = si.conv3d_problem(N, Cin, D, H, W, Cout, kernel, out, seed, TORCH_DTYPE[dtype], bias,
                          residual, device, prev_frames=kernel[0] - 1 if cached else 0)
    p.update(dict(N=N, Cin=Cin, D=D, H=H, W=W, Cout=Cout, kernel=tuple(kernel), pad=tuple(pad),
                  tpad=tpad, dtype=dtype, out=out, stride=tuple(stride)))
    return p


def oracle_ref(p, rows=None):
    """fp64 oracle on the exact bits the GPU saw (all pixels, or the given rows)."""
    return oracle.conv3d(si.bits(p["x"]), si.bits(p["w"]),
                         None if p["bias"] is None else si.bits(p["bias"]),
                         None if p["residual"] is None else si.bits(p["residual"]),
                         ORACLE_DTYPE[p["dtype"]], p["kernel"], p["stride"], p["pad"], p["tpad"],
                         rows=rows, prev_bits=None if p["prev"] is None else si.bits(p["prev"]))


def errors(y: np.ndarray, ref: np.ndarray):
    err = np.abs(y - ref)
    max_ratio = float(err.max() / max(np.abs(ref).max(), 1e-30))
    rel_l1 = float(err.sum() / max(np.abs(ref).sum(), 1e-30))
    return max_ratio, rel_l1


def assert_close(y: np.ndarray, ref: np.ndarray, what=""):
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    max_ratio, rel_l1 = errors(y, ref)
    assert max_ratio <= MAX_REL, f"{what}: max|err|/max|ref| = {max_ratio:.3e}"
    assert rel_l1 <= MEAN_REL, f"{what}: relative L1 error = {rel_l1:.3e}"
    return max_ratio, rel_l1


def sample_rows(N, Do, Ho, Wo, n_random=256, seed=0):
    """Rows (flat output pixels) that cover the borders, the first/last frames,
    the first and last 128-pixel tile of those frames, and random interior points."""
    HoWo = Ho * Wo
    rows = set()
    frames = sorted({0, 1, Do // 2, Do - 1} & set(range(Do)))
    for n in sorted({0, N - 1}):
        for to in frames:
            base = (n * Do + to) * HoWo
            for pix in list(range(min(130, HoWo))) + list(range(max(0, HoWo - 130), HoWo)):
                rows.add(base + pix)
            for ho in (0, Ho // 2, Ho - 1):
                for wo in (0, 1, Wo // 2, Wo - 2, Wo - 1):
                    if 0 <= wo < Wo:
                        rows.add(base + ho * Wo + wo)
    rng = np.random.default_rng(seed)
    M = N * Do * HoWo
    rows.update(int(v) for v in rng.integers(0, M, n_random))
    return np.array(sorted(rows), dtype=np.int64)

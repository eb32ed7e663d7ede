"""Seeded synthetic inputs shared by the tests, the bench and the oracle side.

This module holds no convolution arithmetic: it only draws numbers.  Both the
CUDA path and the oracle receive the same 16-bit patterns produced here.

Generator (counter-based, so any element can be drawn independently and the
result does not depend on torch's RNG or its version):

  * SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): state advances by the golden-ratio increment
    0x9E3779B97F4A7C15 and each output is the state passed through the
    64-bit finaliser  z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
    z *= 0x94D049BB133111EB; z ^= z>>31.
  * Stream key for (seed, stream): base = finalise(seed * 2^32 + stream).
    Draw j of the stream is finalise(base + (j+1) * increment) (mod 2^64).
  * Element i takes draws 2i and 2i+1 -> u1, u2 = (draw >> 11) * 2^-53 in
    [0, 1), then the Box-Muller transform in float64:
    z = sqrt(-2 ln(1 - u1)) * cos(2 pi u2).
  * value = mean + std * z in float64 -> float32 (round to nearest even) ->
    bf16 / fp16 (round to nearest even).

Tensor streams: x = 0, w = 1, bias = 2, residual = 3, cached previous frames = 4.
Distributions (the workloads' recipe): x, residual ~ N(0, 1);
w ~ N(0, std = 1/sqrt(Cin*kt*kh*kw)); bias ~ N(0, std = 0.1).
"""
from __future__ import annotations

import math

import torch

GAMMA = 0x9E3779B97F4A7C15
MUL1 = 0xBF58476D1CE4E5B9
MUL2 = 0x94D049BB133111EB

STREAM_X = 0
STREAM_W = 1
STREAM_BIAS = 2
STREAM_RESIDUAL = 3
STREAM_PREV = 4


def _s64(v: int) -> int:
    """Reinterpret an unsigned 64-bit constant as a signed int64 value."""
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


def _shr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 tensors holding uint64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _finalise(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _shr(z, 30)) * _s64(MUL1)
    z = (z ^ _shr(z, 27)) * _s64(MUL2)
    return z ^ _shr(z, 31)


def finalise_int(v: int) -> int:
    """Scalar SplitMix64 finaliser on Python ints (exact, for keys and tests)."""
    m = (1 << 64) - 1
    z = v & m
    z = ((z ^ (z >> 30)) * MUL1) & m
    z = ((z ^ (z >> 27)) * MUL2) & m
    return z ^ (z >> 31)


def splitmix64_sequence(state: int, n: int) -> list[int]:
    """The classic sequential SplitMix64 stream (state += gamma; output = finalise)."""
    out = []
    m = (1 << 64) - 1
    for _ in range(n):
        state = (state + GAMMA) & m
        out.append(finalise_int(state))
    return out


def stream_base(seed: int, stream: int) -> int:
    return finalise_int((seed << 32) + stream)


def draws(seed: int, stream: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Draws start..start+count-1 of the (seed, stream) sequence as int64 bit patterns."""
    base = _s64(stream_base(seed, stream))
    j = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    return _finalise(j * _s64(GAMMA) + base)


def normal(seed: int, stream: int, numel: int, device="cpu") -> torch.Tensor:
    """numel standard-normal float64 values; element i uses draws 2i and 2i+1."""
    return _normal_range(seed, stream, 0, numel, device)


def tensor(shape, seed: int, stream: int, std: float = 1.0, dtype=torch.bfloat16,
           device="cpu") -> torch.Tensor:
    """A seeded N(0, std^2) tensor of ``shape`` rounded f64 -> f32 -> dtype (RNE)."""
    numel = 1
    for s in shape:
        numel *= int(s)
    out = torch.empty(numel, dtype=dtype, device=device)
    chunk = 1 << 24
    for s in range(0, numel, chunk):
        c = min(chunk, numel - s)
        z = _normal_range(seed, stream, s, c, device)
        out[s:s + c] = (z * std).to(torch.float32).to(dtype)
    return out.view(*shape)


def _normal_range(seed, stream, start, count, device):
    d = draws(seed, stream, 2 * start, 2 * count, device).view(count, 2)
    scale = 2.0 ** -53
    u1 = _shr(d[:, 0], 11).to(torch.float64) * scale
    u2 = _shr(d[:, 1], 11).to(torch.float64) * scale
    return torch.sqrt(-2.0 * torch.log1p(-u1)) * torch.cos((2.0 * math.pi) * u2)


def conv3d_problem(N, Cin, D, H, W, Cout, kernel, out_dhw, seed, dtype=torch.bfloat16,
                   bias=True, residual=False, device="cpu", prev_frames=0):
    """x, w, bias, residual (and cached previous frames) for one convolution,
    following the workload recipe.

    Returns a dict of torch tensors (NDHWC x, [Cout,kt,kh,kw,Cin] w, [Cout] bias,
    [N,Do,Ho,Wo,Cout] residual, [N,prev_frames,H,W,Cin] prev ~ N(0,1)); absent
    ones are None.
    """
    kt, kh, kw = kernel
    fan_in = Cin * kt * kh * kw
    x = tensor((N, D, H, W, Cin), seed, STREAM_X, 1.0, dtype, device)
    w = tensor((Cout, kt, kh, kw, Cin), seed, STREAM_W, 1.0 / math.sqrt(fan_in), dtype, device)
    b = tensor((Cout,), seed, STREAM_BIAS, 0.1, dtype, device) if bias else None
    r = None
    if residual:
        Do, Ho, Wo = out_dhw
        r = tensor((N, Do, Ho, Wo, Cout), seed, STREAM_RESIDUAL, 1.0, dtype, device)
    pv = None
    if prev_frames > 0:
        pv = tensor((N, prev_frames, H, W, Cin), seed, STREAM_PREV, 1.0, dtype, device)
    return {"x": x, "w": w, "bias": b, "residual": r, "prev": pv}


def bits(t: torch.Tensor):
    """The raw 16-bit patterns of a bf16/fp16 tensor as a numpy uint16 array (host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")

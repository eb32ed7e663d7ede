"""The synthetic workloads: shapes, padding, dtype, seed and residual flag.

Data only.  These stand in for the video-VAE decoder layers the pages discuss
(LTX-2.x and Wan 2.x decoder convolutions); no weights or real latents exist
here, so every tensor is drawn by ``seeded_inputs.conv3d_problem``.
Temporal modes: 0 zero, 1 causal replicate-first-frame, 2 causal zero,
3 causal with the previous chunk's last kt-1 frames cached in front.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str          # "bf16" or "f16"
    N: int
    Cin: int
    Cout: int
    D: int
    H: int
    W: int
    kernel: tuple
    pad: tuple          # (pt, ph, pw); pt only for the zero temporal mode
    tpad: int
    seed: int
    residual: bool
    note: str
    stride: tuple = (1, 1, 1)


WORKLOADS = {
    "cfg1": Workload("cfg1", "f16", 1, 32, 32, 5, 32, 32, (3, 3, 3), (1, 1, 1), 0, 0, False,
                     "fp16 32->32, 5x32x32, zero pad 1 on all dims (small correctness case)"),
    "cfg2": Workload("cfg2", "bf16", 1, 256, 256, 9, 128, 128, (3, 3, 3), (0, 1, 1), 1, 1, True,
                     "bf16 256->256, 9x128x128, causal replicate pad, fused residual"),
    "cfg2c": Workload("cfg2c", "bf16", 1, 256, 256, 9, 128, 128, (3, 3, 3), (0, 1, 1), 3, 10, True,
                      "bf16 256->256, a 9-frame chunk of 128x128 with 2 cached previous frames, "
                      "fused residual (chunked decoding)"),
    "cfg2s": Workload("cfg2s", "bf16", 1, 256, 256, 9, 256, 256, (3, 3, 3), (0, 1, 1), 1, 11, False,
                      "bf16 256->256, 9x256x256 -> 9x128x128, stride (1,2,2), causal replicate pad "
                      "(spatial downsampling, as in video-VAE encoders)", (1, 2, 2)),
    "cfg3": Workload("cfg3", "bf16", 1, 512, 512, 17, 64, 96, (3, 3, 3), (0, 1, 1), 1, 2, False,
                     "bf16 512->512, 17x64x96, causal replicate pad (deep mid-block)"),
    "cfg4": Workload("cfg4", "bf16", 1, 128, 128, 121, 256, 256, (3, 3, 3), (0, 1, 1), 1, 3, False,
                     "bf16 128->128, 121x256x256, causal replicate pad (late decoder stage)"),
    "cfg5a": Workload("cfg5a", "bf16", 1, 128, 512, 9, 64, 64, (3, 3, 3), (0, 1, 1), 1, 5, False,
                      "bf16 128->512, 9x64x64, causal replicate pad"),
    "cfg5b": Workload("cfg5b", "bf16", 1, 512, 256, 33, 128, 128, (3, 3, 3), (0, 1, 1), 1, 6, False,
                      "bf16 512->256, 33x128x128, causal replicate pad"),
    "cfg5c": Workload("cfg5c", "bf16", 1, 512, 256, 33, 128, 128, (1, 1, 1), (0, 0, 0), 0, 7, False,
                      "bf16 1x1x1 shortcut 512->256, 33x128x128"),
    "cfg4s": Workload("cfg4s", "bf16", 1, 128, 128, 9, 256, 256, (3, 3, 3), (0, 1, 1), 1, 9, False,
                      "bf16 128->128, 9x256x256, causal replicate pad (a 9-frame slice of the late "
                      "decoder stage, small enough for ncu replays)"),
    "cfg5d": Workload("cfg5d", "bf16", 1, 256, 256, 1, 256, 256, (3, 3, 3), (0, 1, 1), 1, 8, False,
                      "bf16 first frame T=1 256->256, 256x256, causal replicate pad (a 2D conv)"),
}


@dataclass(frozen=True)
class NormWorkload:
    name: str
    dtype: str
    shape: tuple        # [N, D, H, W, C]
    groups: int
    per_frame: bool
    seed: int
    note: str


NORM_WORKLOADS = {
    "gn_cfg2": NormWorkload("gn_cfg2", "bf16", (1, 9, 128, 128, 256), 32, False, 12,
                            "GroupNorm(32) + SiLU of the 256-channel 9x128x128 activation"),
    "gn_cfg4": NormWorkload("gn_cfg4", "bf16", (1, 121, 256, 256, 128), 32, True, 13,
                            "per-frame GroupNorm(32) + SiLU of the 128-channel 121x256x256 "
                            "activation"),
}

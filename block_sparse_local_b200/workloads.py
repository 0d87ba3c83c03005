"""Seeded synthetic workloads shared by the tests, the oracle checks and bench.py.

This module only describes shapes and draws random numbers; it holds none of
the attention arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it without sharing any of the method's code.

The shapes follow the STA README's Usage example (a (30, 48, 80) video cut
into (6, 8, 8) tiles, 256 padded text tokens, window (3, 3, 3) tiles) and the
sliding-window page's 4096-token causal window with grouped-query attention.
All values are synthetic: q, k, v are drawn i.i.d. normal in fp32 from a
seeded generator and rounded to bf16.
"""
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class StaWorkload:
    name: str
    B: int
    heads: int
    d: int
    T: int
    H: int
    W: int
    tile: tuple
    windows: tuple          # one (wt, wh, ww) per head
    text_len: int
    has_text: bool
    std: float
    seed: int
    note: str = ""

    @property
    def S(self):
        return self.T * self.H * self.W + (256 if self.has_text else 0)

    @property
    def L_v(self):
        return self.T * self.H * self.W


@dataclass(frozen=True)
class SwaWorkload:
    name: str
    B: int
    hq: int
    hkv: int
    d: int
    S: int
    window: int
    causal: bool
    std: float
    seed: int


def per_head_windows_video_only(heads=48, seed=3):
    """Per-head window draw of the video-only workload (logged by bench/tests)."""
    choices = ((3, 3, 3), (3, 5, 5), (5, 6, 6))
    idx = np.random.default_rng(seed).integers(0, 3, size=heads)
    return tuple(choices[i] for i in idx)


TINY = StaWorkload("tiny_18x24x32_w133", 1, 1, 64, 18, 24, 32, (6, 8, 8),
                   ((1, 3, 3),), 0, False, 1.0, 1,
                   "tile grid (3,3,4), 13,824 tokens, no text")
VIDEO_TEXT = StaWorkload("video_text_30x48x80_w333", 1, 24, 128, 30, 48, 80,
                         (6, 8, 8), ((3, 3, 3),) * 24, 200, True, 1.0, 2,
                         "tile grid (5,6,10) = 115,200 video + 256 text tokens")
VIDEO_ONLY = StaWorkload("video_only_36x48x48_perhead", 2, 48, 128, 36, 48, 48,
                         (6, 8, 8), per_head_windows_video_only(), 0, False,
                         0.5, 3, "tile grid (6,6,6), per-head windows")
IMAGE_2D = StaWorkload("image2d_256x256_w55", 8, 16, 64, 1, 256, 256,
                       (1, 16, 16), ((1, 5, 5),) * 16, 0, False, 1.0, 4,
                       "2-D, 16x16 tiles of 16x16 tokens")
IMAGE_2D_FULL = StaWorkload("image2d_256x256_w1616", 8, 16, 64, 1, 256, 256,
                            (1, 16, 16), ((1, 16, 16),) * 16, 0, False, 1.0, 4,
                            "window covers the grid: equals dense attention")
SWA_GQA = SwaWorkload("swa_causal_gqa_32k_w4096", 1, 32, 8, 128, 32768, 4096,
                      True, 1.0, 5)

STA_WORKLOADS = {w.name: w for w in (TINY, VIDEO_TEXT, VIDEO_ONLY, IMAGE_2D,
                                     IMAGE_2D_FULL)}


def randn_bf16(shape, seed, std=1.0, device="cpu"):
    """i.i.d. N(0, std^2) drawn in fp32 from ``seed`` and rounded to bf16."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def sta_inputs(w: StaWorkload, device="cpu", B=None):
    """q, k, v as [B, heads, S, d] bf16 in raster token order."""
    B = w.B if B is None else B
    shape = (B, w.heads, w.S, w.d)
    return tuple(randn_bf16(shape, w.seed * 1000 + i, w.std, device)
                 for i in range(3))


def swa_inputs(w: SwaWorkload, device="cpu"):
    q = randn_bf16((w.B, w.hq, w.S, w.d), w.seed * 1000 + 0, w.std, device)
    k = randn_bf16((w.B, w.hkv, w.S, w.d), w.seed * 1000 + 1, w.std, device)
    v = randn_bf16((w.B, w.hkv, w.S, w.d), w.seed * 1000 + 2, w.std, device)
    return q, k, v


def small_sta_case(T, H, W, tile, windows, text_len, has_text, d=64, B=1,
                   seed=0, std=1.0):
    """Ad-hoc small workload for parity tests (several tiles + ragged text)."""
    return StaWorkload(f"small_{T}x{H}x{W}", B, len(windows), d, T, H, W,
                       tuple(tile), tuple(tuple(x) for x in windows), text_len,
                       has_text, std, seed)

"""Seeded synthetic workloads: the five stream configurations and their inputs.

This module holds no arithmetic of the method.  It only names the configurations (sizes,
retention parameters, keyframe schedule, value distributions) and draws their q/k/v inputs
from seeded generators.  The tests, ``bench.py`` and the oracle-side checks all take their
inputs from here, so the CUDA path and the oracle see the same numbers.

Recipe, per (config c, frame f, tensor t in {q:0, k:1, v:2}, region r in {special:0,
patch:1}): ``numpy.random.default_rng([c, f, t, r])`` draws float32 standard normals (or
uniforms on [-1, 1) for v where the config says so) of shape [rows, heads, head_dim]; the
special rows (6) come first, then the patch rows (pph * ppw), giving [T, heads, head_dim].
bf16 configurations round the float32 draws to bf16 with round-to-nearest-even.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class StreamConfig:
    cid: int
    name: str
    heads: int
    head_dim: int
    dtype: str                  # "f32" or "bf16"
    pph: int
    ppw: int
    n_frames: int
    keyframe_interval: int
    scale_frames: int
    sliding_window: int
    v_dist: str = "normal"      # "normal" or "uniform"
    specials: int = 6

    @property
    def patches(self) -> int:
        return self.pph * self.ppw

    @property
    def tokens(self) -> int:
        return self.specials + self.patches

    @property
    def keyframes(self) -> list:
        return [(f % self.keyframe_interval) == 0 for f in range(self.n_frames)]

    @property
    def n_keyframes(self) -> int:
        return sum(self.keyframes)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def describe(self) -> str:
        return (f"{self.name}: {self.heads} heads x head_dim {self.head_dim}, {self.dtype}; "
                f"frame = {self.specials} special + {self.pph}x{self.ppw} patches; "
                f"{self.n_frames} frames, keyframe every {self.keyframe_interval}; "
                f"scale_frames={self.scale_frames}, sliding_window={self.sliding_window}")


CONFIGS = [
    StreamConfig(0, "tiny", 2, 64, "f32", 4, 4, 8, 1, 1, 3),
    StreamConfig(1, "stream-768", 16, 64, "bf16", 24, 32, 64, 1, 8, 16),
    StreamConfig(2, "keyframe5-999", 16, 64, "bf16", 37, 27, 320, 5, 8, 64),
    StreamConfig(3, "long-2000", 16, 64, "bf16", 37, 27, 2000, 1, 8, 128),
    StreamConfig(4, "large-4096", 8, 128, "bf16", 64, 64, 96, 1, 4, 32, v_dist="uniform"),
]


def custom_config(cid: int, heads: int, head_dim: int, dtype: str, pph: int, ppw: int,
                  n_frames: int, keyframe_interval: int, scale_frames: int,
                  sliding_window: int, v_dist: str = "normal") -> StreamConfig:
    """A test-sized stream with the same recipe (cid keeps its seeds apart from CONFIGS)."""
    return StreamConfig(cid, f"custom{cid}", heads, head_dim, dtype, pph, ppw, n_frames,
                        keyframe_interval, scale_frames, sliding_window, v_dist)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 (ties to even), returned as float32 holding the bf16 value."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    rounded = (bits + (np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))))
    return (rounded & np.uint32(0xFFFF0000)).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are exactly bf16 (as uint16)."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float32 values."""
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def _draw(cfg: StreamConfig, frame: int, tensor: int, region: int) -> np.ndarray:
    rows = cfg.specials if region == 0 else cfg.patches
    rng = np.random.default_rng([cfg.cid, frame, tensor, region])
    shape = (rows, cfg.heads, cfg.head_dim)
    if tensor == 2 and cfg.v_dist == "uniform":
        x = rng.random(shape, dtype=np.float32) * np.float32(2.0) - np.float32(1.0)
    else:
        x = rng.standard_normal(shape, dtype=np.float32)
    return x


def frame_tensor(cfg: StreamConfig, frame: int, tensor: int) -> np.ndarray:
    """One of q (0), k (1), v (2) of one frame: float32 [T, heads, head_dim]."""
    x = np.concatenate([_draw(cfg, frame, tensor, 0), _draw(cfg, frame, tensor, 1)], axis=0)
    return round_bf16(x) if cfg.dtype == "bf16" else x


def frame_qkv(cfg: StreamConfig, frame: int):
    """(q, k, v) of one frame, float32 [T, heads, head_dim] each (bf16 values for bf16)."""
    return tuple(frame_tensor(cfg, frame, t) for t in range(3))


def frame_specials(cfg: StreamConfig, frame: int, tensor: int) -> np.ndarray:
    """The 6 special rows of one tensor of one frame (cheap: no patch draws)."""
    x = _draw(cfg, frame, tensor, 0)
    return round_bf16(x) if cfg.dtype == "bf16" else x

"""3D (frame t, row h, column w) rotary position embedding, float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

What the pages fix
------------------
* [3DRoPE-KV] "Multi-Axis Frequency Generation": one independent 1D RoPE frequency table
  per axis (t, h, w), concatenated along ``head_dim // 2`` into one complex table that is
  expanded to every token of ``ppf`` frames, special tokens included:
  shape ``[ppf * (patch_start_idx + pph * ppw), head_dim // 2]``.
* [3DRoPE-KV] "Complex-Valued Tensor Application": the table is applied as a complex
  multiplication written in real arithmetic.
* [VideoRoPE] "The Three Rotary Dimensions" and "NTK-Aware Frequency Scaling": the 1D
  table of an axis is built from ``theta`` (10000) and an ``ntk_factor`` that multiplies
  theta (1 unless given).
* [3DRoPE-KV] "Implementation Example" and [VideoRoPE] "Enabling 3D RoPE for Video Heads"
  print explicit (t, h, w) feature splits ``fhw_dim`` = [20, 22, 22] (head_dim 64) and
  [40, 44, 44] (head_dim 128); every function below takes such a ``split`` instead of the
  default one.
* [VideoRoPE] "Temporal Consistency in KV-Cache Streaming": the t coordinate is the
  absolute (global) frame index of the stream.

Readings where the pages leave a step open:

* inv_freq of axis a with ``d_a`` features: ``theta ** (-(2 i) / d_a)``, ``i < d_a / 2``.
* Split of ``head_dim``: ``d_h = d_w = 2 * (head_dim // 6)``, ``d_t = head_dim - 2 d_h``
  (64 -> 24/20/20, 128 -> 44/42/42).  Pairs are concatenated in the order t, h, w.
* Feature pairs are adjacent: pair ``i`` is (x[2i], x[2i+1]) viewed as x[2i] + 1j x[2i+1].
* Token positions inside frame t: the ``patch_start_idx`` special tokens come first and sit
  at (t, 0, 0); patch (r, c) of the ``pph x ppw`` grid (row-major) sits at (t, 1+r, 1+c).
"""

from __future__ import annotations

import numpy as np

THETA = 10000.0


def axis_split(head_dim: int, split=None) -> tuple[int, int, int]:
    """Feature counts (d_t, d_h, d_w) of the three axes; all even, summing to head_dim.

    ``split`` gives them explicitly (the pages' ``fhw_dim``); otherwise the default reading.
    """
    if head_dim % 2 != 0 or head_dim < 6:
        raise ValueError("head_dim must be even and >= 6")
    if split is not None:
        d_t, d_h, d_w = (int(x) for x in split)
        if d_t + d_h + d_w != head_dim or min(d_t, d_h, d_w) < 2 or d_t % 2 or d_h % 2 or d_w % 2:
            raise ValueError("split must be three even sizes >= 2 summing to head_dim")
        return d_t, d_h, d_w
    d_h = 2 * (head_dim // 6)
    d_w = d_h
    d_t = head_dim - d_h - d_w
    return d_t, d_h, d_w


def inv_freq(d_axis: int, theta: float = THETA, ntk_factor: float = 1.0) -> np.ndarray:
    """1D RoPE inverse frequencies of one axis: (theta * ntk) ** (-(2 i) / d_axis), fp64.

    [VideoRoPE] "NTK-Aware Frequency Scaling" multiplies theta by ntk_factor before use.
    """
    base = float(theta) * float(ntk_factor)
    i = np.arange(d_axis // 2, dtype=np.float64)
    return base ** (-(2.0 * i) / float(d_axis))


def token_positions(frame_idx: int, patch_start_idx: int, pph: int, ppw: int) -> np.ndarray:
    """(t, h, w) of every token of one frame, shape [patch_start_idx + pph*ppw, 3], int64.

    Specials first at (t, 0, 0); patches row-major at (t, 1 + r, 1 + c).
    """
    n_patch = pph * ppw
    pos = np.zeros((patch_start_idx + n_patch, 3), dtype=np.int64)
    pos[:, 0] = frame_idx
    j = np.arange(n_patch)
    pos[patch_start_idx:, 1] = 1 + j // ppw
    pos[patch_start_idx:, 2] = 1 + j % ppw
    return pos


def angles_for_positions(pos: np.ndarray, head_dim: int, theta: float = THETA, split=None,
                         ntk_factor: float = 1.0) -> np.ndarray:
    """Rotation angle of every (token, pair): [N, head_dim/2] fp64, pairs ordered t, h, w."""
    d_t, d_h, d_w = axis_split(head_dim, split)
    pos = np.asarray(pos, dtype=np.float64)
    return np.concatenate(
        [
            np.outer(pos[:, 0], inv_freq(d_t, theta, ntk_factor)),
            np.outer(pos[:, 1], inv_freq(d_h, theta, ntk_factor)),
            np.outer(pos[:, 2], inv_freq(d_w, theta, ntk_factor)),
        ],
        axis=1,
    )


def expanded_table(head_dim: int, ppf: int, pph: int, ppw: int, patch_start_idx: int,
                   theta: float = THETA, f_start: int = 0, split=None, ntk_factor: float = 1.0):
    """The concatenated, expanded table as (cos, sin), each [ppf*(psi+pph*ppw), head_dim/2].

    Frames f_start .. f_start+ppf-1, each frame's tokens in the order of token_positions.
    [3DRoPE-KV] "Multi-Axis Frequency Generation" prints this shape.
    """
    pos = np.concatenate(
        [token_positions(f_start + f, patch_start_idx, pph, ppw) for f in range(ppf)], axis=0
    )
    ang = angles_for_positions(pos, head_dim, theta, split, ntk_factor)
    return np.cos(ang), np.sin(ang)


def rotate(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate feature pairs of x [N, H, D] by angles [N, D/2] (same angle for every head).

    Pair (x0, x1) = (x[2i], x[2i+1]) becomes (x0 c - x1 s, x0 s + x1 c): the complex
    product (x0 + 1j x1) * exp(1j * angle) written in real arithmetic, in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def rotate_frame(x: np.ndarray, frame_idx: int, patch_start_idx: int, pph: int, ppw: int,
                 theta: float = THETA, split=None, ntk_factor: float = 1.0) -> np.ndarray:
    """Rotate one frame's tokens x [psi + pph*ppw, H, D] at their 3D positions."""
    head_dim = x.shape[-1]
    pos = token_positions(frame_idx, patch_start_idx, pph, ppw)
    return rotate(x, angles_for_positions(pos, head_dim, theta, split, ntk_factor))

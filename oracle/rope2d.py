"""2D (row y, column x) rotary position embedding, float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

What the page fixes ("How to Handle Sequences Exceeding the RoPE Training Range in
LingBot-Map"):

* "Spatial Position Encoding": a position getter gives every patch of the grid its (y, x)
  coordinates; the features of a token are split into two halves, the first rotated by a 1D
  rotary embedding of y, the second by one of x, and the halves are concatenated back.
* "Automatic Cache Generation During Forward Pass": the module is built with
  ``frequency=100.0`` (the base of the 1D embeddings) and ``scaling_factor=1.0``; head_dim
  must be divisible by 4 (two halves, each of whole feature pairs); a 64 x 64 grid gives
  4096 tokens.
* "Deriving Size from Token Count" and "Pre-populating Frequency Tables": the frequency
  table of a half (``dim // 2`` features) has as many rows as there are tokens (positions
  0 .. n_tokens - 1), not max position + 1.

Readings where the page leaves a step open:

* inv_freq of a half with ``d = head_dim / 2`` features: ``frequency ** (-(2 i) / d)``,
  ``i < d / 2`` (the same 1D form as the 3D embedding's axes).
* Feature pairs are adjacent, (x[2i], x[2i+1]), as in the 3D embedding; pairs
  ``[0, head_dim/4)`` take y, pairs ``[head_dim/4, head_dim/2)`` take x.
* In a stream the special tokens sit at (0, 0) and patch (r, c) at (1 + r, 1 + c), the
  spatial part of the 3D positions; the frame index plays no part.  A bare image grid (no
  special tokens) uses the position getter's (r, c).
* ``scaling_factor`` is given only as 1.0 and never defined, so it is not modelled.
"""

from __future__ import annotations

import numpy as np

from . import rope3d

FREQUENCY = 100.0


def half_dim(head_dim: int) -> int:
    """Features per half (y or x); head_dim must be divisible by 4."""
    if head_dim % 4 != 0 or head_dim < 4:
        raise ValueError("head_dim must be a positive multiple of 4")
    return head_dim // 2


def inv_freq(d_half: int, frequency: float = FREQUENCY) -> np.ndarray:
    """1D inverse frequencies of one half: frequency ** (-(2 i) / d_half), fp64."""
    i = np.arange(d_half // 2, dtype=np.float64)
    return float(frequency) ** (-(2.0 * i) / float(d_half))


def frequency_components(d_half: int, seq_len: int, frequency: float = FREQUENCY):
    """(cos, sin) of one half's table: [seq_len, d_half / 2], rows = positions 0..seq_len-1."""
    ang = np.outer(np.arange(seq_len, dtype=np.float64), inv_freq(d_half, frequency))
    return np.cos(ang), np.sin(ang)


def position_getter(pph: int, ppw: int) -> np.ndarray:
    """(y, x) of every patch of a pph x ppw grid, row-major: [pph * ppw, 2], int64."""
    j = np.arange(pph * ppw)
    return np.stack([j // ppw, j % ppw], axis=1).astype(np.int64)


def token_positions(patch_start_idx: int, pph: int, ppw: int) -> np.ndarray:
    """(y, x) of every token of a frame in a stream: specials (0, 0), patches (1+r, 1+c)."""
    pos = np.zeros((patch_start_idx + pph * ppw, 2), dtype=np.int64)
    pos[patch_start_idx:] = 1 + position_getter(pph, ppw)
    return pos


def angles_for_positions(pos: np.ndarray, head_dim: int, frequency: float = FREQUENCY,
                         seq_len: int | None = None) -> np.ndarray:
    """Rotation angle of every (token, pair): [N, head_dim / 2], y pairs then x pairs.

    The angles are read from a table of ``seq_len`` rows (default: one per token, as the page
    sizes it); every coordinate must be below it.
    """
    pos = np.asarray(pos, dtype=np.int64)
    d = half_dim(head_dim)
    rows = len(pos) if seq_len is None else int(seq_len)
    if pos.size and pos.max() >= rows:
        raise ValueError("a coordinate lies beyond the table sized from the token count")
    table = np.outer(np.arange(rows, dtype=np.float64), inv_freq(d, frequency))
    return np.concatenate([table[pos[:, 0]], table[pos[:, 1]]], axis=1)


def expanded_table(head_dim: int, ppf: int, pph: int, ppw: int, patch_start_idx: int,
                   frequency: float = FREQUENCY):
    """(cos, sin) per token of ``ppf`` frames of a stream, each [ppf * T, head_dim / 2]."""
    ang = angles_for_positions(token_positions(patch_start_idx, pph, ppw), head_dim, frequency)
    ang = np.tile(ang, (ppf, 1))
    return np.cos(ang), np.sin(ang)


def rotate_frame(x: np.ndarray, patch_start_idx: int, pph: int, ppw: int,
                 frequency: float = FREQUENCY) -> np.ndarray:
    """Rotate one frame's tokens x [psi + pph*ppw, H, D] at their (y, x) positions."""
    pos = token_positions(patch_start_idx, pph, ppw)
    return rope3d.rotate(x, angles_for_positions(pos, x.shape[-1], frequency))


def rotate_grid(tokens: np.ndarray, positions: np.ndarray,
                frequency: float = FREQUENCY) -> np.ndarray:
    """The page's module call on a bare grid: tokens [B, heads, N, D], positions [B, N, 2]
    (from position_getter); returns the rotated tokens, same shape."""
    tokens = np.asarray(tokens, dtype=np.float64)
    out = np.empty_like(tokens)
    for b in range(tokens.shape[0]):
        ang = angles_for_positions(positions[b], tokens.shape[-1], frequency)
        # rope3d.rotate takes [N, H, D]
        out[b] = rope3d.rotate(tokens[b].transpose(1, 0, 2), ang).transpose(1, 0, 2)
    return out

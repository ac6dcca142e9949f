"""Attention of one frame's queries over the keys the cache retains, float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

[3DRoPE-KV] "Attention Computation with Cached RoPE": the frame's queries attend over the
visible pages with K/V that already carry their rotation.  [RealTime3D] "Per-Frame
Processing and Causal Attention": a frame sees cached past tokens and special tokens, no
future frame.  Reading where the pages are loose: a frame's own tokens are all visible to each other
(bidirectional inside the frame); scale is 1/sqrt(head_dim).

Two formulations, which must agree:

* ``attend``         plain softmax over an explicit key list (the retained keys, in
                     visible-page-table order);
* ``attend_masked``  softmax over the whole history of the stream with masked-out keys set
                     to -inf, the mask built from the closed form of the retained set.
"""

from __future__ import annotations

import numpy as np


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None,
           return_lse: bool = False):
    """out[t, h] = sum_n softmax_n(q[t,h] . k[n,h] * scale) v[n,h].

    q [T, H, D], k and v [N, H, D]; fp64; max-subtracted softmax.
    With return_lse, also the natural-log sum of exp of the scaled scores, [T, H].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    s = np.matmul(q.transpose(1, 0, 2), k.transpose(1, 2, 0)) * scale   # [H, T, N]
    m = s.max(axis=-1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=-1, keepdims=True)
    out = np.matmul(p / l, v.transpose(1, 0, 2)).transpose(1, 0, 2)      # [T, H, D]
    if return_lse:
        return out, (m[..., 0] + np.log(l[..., 0])).T
    return out


def attend_masked(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                  scale: float | None = None) -> np.ndarray:
    """Like ``attend`` over all N keys, with keys where mask is False set to -inf."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    s = np.matmul(q.transpose(1, 0, 2), k.transpose(1, 2, 0)) * scale
    s = np.where(np.asarray(mask, dtype=bool)[None, None, :], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    p = np.exp(s - m)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.matmul(p, v.transpose(1, 0, 2)).transpose(1, 0, 2)


def history_mask(frames: list, current: int, committed_before: list, retained_before: list,
                 specials_per_frame: int, tokens_per_frame: int) -> np.ndarray:
    """Visibility of every token of ``frames`` (the whole stream up to ``current``).

    A token of frame f at index j is visible to frame ``current`` iff f is the current
    frame, or j is a patch (j >= specials_per_frame) of a retained frame, or j is a special
    token of a committed keyframe.
    """
    committed = set(committed_before)
    retained = set(retained_before)
    mask = np.zeros(len(frames) * tokens_per_frame, dtype=bool)
    for n, f in enumerate(frames):
        base = n * tokens_per_frame
        if f == current:
            mask[base:base + tokens_per_frame] = True
            continue
        if f in committed:
            mask[base:base + specials_per_frame] = True
        if f in retained:
            mask[base + specials_per_frame:base + tokens_per_frame] = True
    return mask

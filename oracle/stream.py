"""A stream of frames through rotate -> append -> attend -> commit/rollback, float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Per frame ([3DRoPE-KV] "Frame Appending and Position Encoding Integration" and
"Attention Computation with Cached RoPE"; [KVBenefits] "Dynamic Keyframe Selection"):

1. rotate the frame's q and k at their 3D positions (``rope3d``), v unrotated;
2. append: the patch keys/values take a page popped from the free list, the 6 special
   tokens take the next slots of the special stream (``retention``);
3. attend: the frame's queries over scale pages -> window pages -> own page -> specials
   (``attention.attend``);
4. commit (keyframe: deferred eviction) or roll back (non-keyframe).

Only the K/V of frames still retained are kept, so long streams stay bounded in memory,
unless ``keep_history`` is set (small streams; enables the masked whole-history check).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import attention, retention, rope2d, rope3d

ROW_CHUNK = 64


@dataclass
class FrameResult:
    frame_idx: int
    is_keyframe: bool
    page: int
    special_slot: int
    visible: retention.Visible
    visible_frames: list       # frames whose patch pages are visible, visible order
    q_rot: np.ndarray          # [T, H, D] fp64
    k_rot: np.ndarray          # [T, H, D] fp64
    rows: np.ndarray           # query rows computed
    out: np.ndarray            # [len(rows), H, D] fp64
    lse: np.ndarray            # [len(rows), H] natural-log sum-exp of scaled scores
    evicted: int | None
    state: dict                # retention snapshot after commit / rollback


class StreamOracle:
    def __init__(self, heads: int, head_dim: int, pph: int, ppw: int, scale_frames: int,
                 sliding_window: int, max_frames: int, specials_per_frame: int = 6,
                 theta: float = rope3d.THETA, keep_history: bool = False, kv_source=None,
                 split=None, ntk_factor: float = 1.0, rope2d_frequency: float | None = None):
        """split / ntk_factor: an explicit (t, h, w) feature split and NTK factor of the 3D
        RoPE (``rope3d.axis_split``, ``rope3d.inv_freq``).  rope2d_frequency: rotate with the
        2D (y, x) embedding of that base frequency instead (``rope2d``; the frame index then
        plays no part in the rotation).  kv_source, if given, is a callable
        (frame, region) -> (k, v) returning a past frame's unrotated inputs (region "patch":
        [pph*ppw, H, D], "special": [6, H, D]); the oracle then keeps no K/V of its own and
        re-creates retained keys when a frame attends, which keeps long streams small in
        memory."""
        self.heads = heads
        self.head_dim = head_dim
        self.pph = pph
        self.ppw = ppw
        self.psi = specials_per_frame
        self.theta = theta
        self.split = split
        self.ntk_factor = ntk_factor
        self.rope2d_frequency = rope2d_frequency
        self.ret = retention.PagedRetention(scale_frames, sliding_window, max_frames,
                                            specials_per_frame)
        self.patch_kv: dict = {}      # frame -> (k [Pf,H,D], v [Pf,H,D]) of retained frames
        self.special_kv: list = []    # [(frame, k [6,H,D], v [6,H,D])] committed, in order
        self.keep_history = keep_history
        self.history: list = []       # [(frame, k [T,H,D], v [T,H,D])] every frame seen
        self.kv_source = kv_source

    @property
    def tokens_per_frame(self) -> int:
        return self.psi + self.pph * self.ppw

    def reset(self) -> None:
        self.ret.reset()
        self.patch_kv = {}
        self.special_kv = []
        self.history = []

    def _retained_kv(self, frame: int, region: str):
        """Rotated k and plain v of a retained frame's patches or specials (fp64)."""
        if self.kv_source is None:
            if region == "patch":
                return self.patch_kv[frame]
            for f, ks, vs in self.special_kv:
                if f == frame:
                    return ks, vs
            raise KeyError(frame)
        k, v = self.kv_source(frame, region)
        ang = self.angles(frame)
        ang = ang[self.psi:] if region == "patch" else ang[:self.psi]
        return rope3d.rotate(k, ang), np.asarray(v, dtype=np.float64)

    def angles(self, frame: int) -> np.ndarray:
        """Rotation angles of every token of frame ``frame``: [T, head_dim / 2]."""
        if self.rope2d_frequency is not None:
            pos = rope2d.token_positions(self.psi, self.pph, self.ppw)
            return rope2d.angles_for_positions(pos, self.head_dim, self.rope2d_frequency)
        pos = rope3d.token_positions(frame, self.psi, self.pph, self.ppw)
        return rope3d.angles_for_positions(pos, self.head_dim, self.theta, self.split,
                                           self.ntk_factor)

    def step(self, frame_idx: int, is_keyframe: bool, q: np.ndarray, k: np.ndarray,
             v: np.ndarray, rows=None, attend: bool = True) -> FrameResult:
        T = self.tokens_per_frame
        assert q.shape == (T, self.heads, self.head_dim), q.shape
        page, slot = self.ret.append(frame_idx, is_keyframe)
        ang = self.angles(frame_idx)
        qr = rope3d.rotate(q, ang)
        kr = rope3d.rotate(k, ang)
        v64 = np.asarray(v, dtype=np.float64)
        vis = self.ret.visible()

        frames = self.ret.retained_frames()
        rows = np.arange(T) if rows is None else np.asarray(rows)
        if attend and len(rows):
            ks, vs = [], []
            for f in frames:
                kf, vf = self._retained_kv(f, "patch")
                ks.append(kf)
                vs.append(vf)
            ks.append(kr[self.psi:])
            vs.append(v64[self.psi:])
            for f in self.committed_frames():
                kf, vf = self._retained_kv(f, "special")
                ks.append(kf)
                vs.append(vf)
            ks.append(kr[:self.psi])
            vs.append(v64[:self.psi])
            K = np.concatenate(ks, axis=0)
            V = np.concatenate(vs, axis=0)
            assert K.shape[0] == len(vis.patch_pages) * self.pph * self.ppw + vis.n_special
            # rows are independent, so the query rows are taken in chunks to bound memory
            outs, lses = [], []
            for c in range(0, len(rows), ROW_CHUNK):
                o, e = attention.attend(qr[rows[c:c + ROW_CHUNK]], K, V, return_lse=True)
                outs.append(o)
                lses.append(e)
            out = np.concatenate(outs, axis=0)
            lse = np.concatenate(lses, axis=0)
        else:
            rows = rows[:0]
            out = np.zeros((0, self.heads, self.head_dim))
            lse = np.zeros((0, self.heads))

        if self.keep_history:
            self.history.append((frame_idx, kr, v64))
        evicted_frame = None
        if is_keyframe and len(self.ret.scale) >= self.ret.scale_frames \
                and len(self.ret.window) >= self.ret.sliding_window:
            evicted_frame = self.ret.window[0][1] if self.ret.sliding_window > 0 else frame_idx
        evicted = self.ret.finish()
        if is_keyframe and self.kv_source is None:
            self.patch_kv[frame_idx] = (kr[self.psi:], v64[self.psi:])
            self.special_kv.append((frame_idx, kr[:self.psi], v64[:self.psi]))
            if evicted is not None:
                del self.patch_kv[evicted_frame]
        return FrameResult(frame_idx, is_keyframe, page, slot, vis, frames + [frame_idx],
                           qr, kr, rows, out, lse, evicted, self.ret.snapshot())

    def committed_frames(self) -> list:
        """Committed keyframes in commit order (their specials are all visible)."""
        return list(self.ret.committed)

    def attend_history_masked(self, q_rot: np.ndarray, frame_idx: int,
                              committed_before: list) -> np.ndarray:
        """Whole-history masked attention for the frame just stepped (keep_history only)."""
        assert self.keep_history
        frames = [h[0] for h in self.history]
        K = np.concatenate([h[1] for h in self.history], axis=0)
        V = np.concatenate([h[2] for h in self.history], axis=0)
        retained = retention.retained_closed_form(committed_before, self.ret.scale_frames,
                                                  self.ret.sliding_window)
        mask = attention.history_mask(frames, frame_idx, committed_before, retained,
                                      self.psi, self.tokens_per_frame)
        return attention.attend_masked(q_rot, K, V, mask)

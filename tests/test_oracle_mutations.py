"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case swaps one oracle function for a plausibly wrong version (a flipped sign, a dropped
factor, a transposed index, the wrong page evicted) and checks that at least one pin test
of tests/test_oracle_*.py then fails.  The mistakes are planted in the oracle, on the CPU,
through monkeypatch; nothing here touches the CUDA path.
"""

import numpy as np
import pytest

from oracle import attention, retention, rope3d

import test_oracle_attention as ta
import test_oracle_retention as tr
import test_oracle_rope as tp


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_flipped_sin_sign_is_caught(monkeypatch):
    def bad_rotate(x, angles):
        x = np.asarray(x, dtype=np.float64)
        c = np.cos(angles)[:, None, :]
        s = np.sin(angles)[:, None, :]
        out = np.empty_like(x)
        out[..., 0::2] = x[..., 0::2] * c + x[..., 1::2] * s
        out[..., 1::2] = -x[..., 0::2] * s + x[..., 1::2] * c
        return out
    monkeypatch.setattr(rope3d, "rotate", bad_rotate)
    _fails(tp.test_rotation_is_complex_multiplication)


def test_frequency_exponent_without_factor_two_is_caught(monkeypatch):
    def bad_inv_freq(d_axis, theta=rope3d.THETA, ntk_factor=1.0):
        i = np.arange(d_axis // 2, dtype=np.float64)
        return (theta * ntk_factor) ** (-i / d_axis)
    monkeypatch.setattr(rope3d, "inv_freq", bad_inv_freq)
    _fails(tp.test_inv_freq_matches_library_1d_rope, 64)


def test_rotate_half_pairing_is_caught(monkeypatch):
    def bad_rotate(x, angles):
        x = np.asarray(x, dtype=np.float64)
        h = x.shape[-1] // 2
        c = np.cos(angles)[:, None, :]
        s = np.sin(angles)[:, None, :]
        out = np.empty_like(x)
        out[..., :h] = x[..., :h] * c - x[..., h:] * s
        out[..., h:] = x[..., :h] * s + x[..., h:] * c
        return out
    monkeypatch.setattr(rope3d, "rotate", bad_rotate)
    _fails(tp.test_each_axis_is_library_1d_rope, 64, None, 1.0)


def test_transposed_patch_grid_is_caught(monkeypatch):
    def bad_positions(frame_idx, patch_start_idx, pph, ppw):
        n_patch = pph * ppw
        pos = np.zeros((patch_start_idx + n_patch, 3), dtype=np.int64)
        pos[:, 0] = frame_idx
        j = np.arange(n_patch)
        pos[patch_start_idx:, 1] = 1 + j % pph
        pos[patch_start_idx:, 2] = 1 + j // pph
        return pos
    monkeypatch.setattr(rope3d, "token_positions", bad_positions)
    _fails(tp.test_positions_and_identity_at_origin)


def test_evicting_the_newest_window_page_is_caught(monkeypatch):
    orig = retention.PagedRetention.finish

    def bad_finish(self):
        page, frame, key = self.pending
        if key and len(self.scale) >= self.scale_frames and \
                len(self.window) >= self.sliding_window > 0:
            self.pending = None
            self.free.append(page)               # drops the new frame instead of the oldest
            self.n_special += self.specials_per_frame
            self.committed.append(frame)
            return page
        return orig(self)
    monkeypatch.setattr(retention.PagedRetention, "finish", bad_finish)
    _fails(tr.test_replay_matches_closed_form, 1, 3, 1, 8)


def test_missing_softmax_scale_is_caught(monkeypatch):
    orig = attention.attend

    def bad_attend(q, k, v, scale=None, return_lse=False):
        return orig(q, k, v, scale=1.0, return_lse=return_lse)
    monkeypatch.setattr(attention, "attend", bad_attend)
    _fails(ta.test_attend_matches_torch_sdpa_and_brute_force)


def test_specials_not_kept_is_caught(monkeypatch):
    orig = attention.history_mask

    def bad_mask(frames, current, committed_before, retained_before, spf, tpf):
        return orig(frames, current, [], retained_before, spf, tpf)
    monkeypatch.setattr(attention, "history_mask", bad_mask)
    _fails(ta.test_stream_two_formulations_agree, ta.CONFIGS[0])


def test_ntk_factor_ignored_is_caught(monkeypatch):
    orig = rope3d.inv_freq

    def bad_inv_freq(d_axis, theta=rope3d.THETA, ntk_factor=1.0):
        return orig(d_axis, theta, 1.0)
    monkeypatch.setattr(rope3d, "inv_freq", bad_inv_freq)
    _fails(tp.test_each_axis_is_library_1d_rope, 64, "example_fhw_dim", 4.0)


def test_split_axes_swapped_is_caught(monkeypatch):
    orig = rope3d.axis_split

    def bad_split(head_dim, split=None):
        d_t, d_h, d_w = orig(head_dim, split)
        return d_h, d_t, d_w
    monkeypatch.setattr(rope3d, "axis_split", bad_split)
    _fails(tp.test_each_axis_is_library_1d_rope, 64, "example_fhw_dim", 1.0)


# ---- the 2D variant ("How to Handle Sequences Exceeding the RoPE Training Range in
# LingBot-Map") ----

import test_oracle_rope2d as t2  # noqa: E402
from oracle import rope2d  # noqa: E402


def test_rope2d_halves_swapped_is_caught(monkeypatch):
    orig = rope2d.angles_for_positions

    def bad(pos, head_dim, frequency=rope2d.FREQUENCY, seq_len=None):
        return orig(np.asarray(pos)[:, ::-1], head_dim, frequency, seq_len)   # x half first
    monkeypatch.setattr(rope2d, "angles_for_positions", bad)
    _fails(t2.test_each_half_is_library_1d_rope, 64)


def test_rope2d_base_of_the_3d_axes_is_caught(monkeypatch):
    orig = rope2d.inv_freq

    def bad(d_half, frequency=rope2d.FREQUENCY):
        return orig(d_half, 10000.0)                   # the 3D embedding's theta
    monkeypatch.setattr(rope2d, "inv_freq", bad)
    _fails(t2.test_each_half_is_library_1d_rope, 128)


def test_rope2d_table_sized_by_max_position_is_caught(monkeypatch):
    def bad(d_half, seq_len, frequency=rope2d.FREQUENCY):
        ang = np.outer(np.arange(65, dtype=np.float64), rope2d.inv_freq(d_half, frequency))
        return np.cos(ang), np.sin(ang)                # max position + 1 rows (64x64 grid)
    monkeypatch.setattr(rope2d, "frequency_components", bad)
    _fails(t2.test_page_example_shapes)

"""Pins of the oracle's 3D RoPE (CPU only).

Each test ties ``oracle.rope3d`` to something other than itself: the table shape printed on
"How 3D RoPE Positional Encoding Works with the Paged KV Cache in LingBot-Map"
(section "Implementation Example"), the 1D RoPE of a library (transformers' LLaMA rotary
embedding: frequencies and rotation), numpy's complex exponential, and invariants every
rotary embedding has (norm preservation, dependence on position offsets only).
"""

import os

import numpy as np
import pytest
import torch

from oracle import rope3d

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.txt")


def _facts():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if "=" in line:
            k, v = (s.strip() for s in line.split("=", 1))
            out[k] = v
    return out


def test_expanded_table_shape_matches_page_example():
    f = _facts()
    cos, sin = rope3d.expanded_table(int(f["example_head_dim"]), int(f["example_ppf"]),
                                     int(f["example_pph"]), int(f["example_ppw"]),
                                     int(f["example_patch_start_idx"]))
    assert cos.shape == (int(f["example_table_rows"]), int(f["example_table_pairs"]))
    assert sin.shape == cos.shape


def test_page_splits_are_accepted_and_bad_splits_refused():
    assert rope3d.axis_split(64, _fhw("example_fhw_dim")) == (20, 22, 22)
    assert rope3d.axis_split(128, _fhw("video_head_fhw_dim")) == (40, 44, 44)
    for bad in [(20, 22, 20), (21, 21, 22), (0, 32, 32)]:
        with pytest.raises(ValueError):
            rope3d.axis_split(64, bad)


def test_axis_split_reading():
    # The stated reading: d_h = d_w = 2 * (head_dim // 6), d_t takes the rest.
    assert rope3d.axis_split(64) == (24, 20, 20)
    assert rope3d.axis_split(128) == (44, 42, 42)
    for d in range(6, 258, 2):
        dt, dh, dw = rope3d.axis_split(d)
        assert dt + dh + dw == d and dt % 2 == dh % 2 == dw % 2 == 0 and dh == dw


def _llama_rope(d_axis, positions, x_half, theta=10000.0):
    """transformers' LLaMA rotary embedding of dimension d_axis (rotate-half layout)."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    cfg = LlamaConfig(hidden_size=d_axis * 2, num_attention_heads=2, head_dim=d_axis,
                      rope_parameters={"rope_type": "default", "rope_theta": theta})
    emb = LlamaRotaryEmbedding(cfg)
    xt = torch.tensor(x_half[None], dtype=torch.float32)        # [1, N, d] -> as [B, H=1?]
    xt = xt[:, None]                                             # [1, 1, N, d]
    pos = torch.tensor(positions, dtype=torch.long)[None]
    cos, sin = emb(xt, pos)
    q, _ = apply_rotary_pos_emb(xt, xt, cos, sin)
    return q[0, 0].numpy().astype(np.float64)


@pytest.mark.parametrize("head_dim", [64, 128])
def test_inv_freq_matches_library_1d_rope(head_dim):
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    for d in rope3d.axis_split(head_dim):
        cfg = LlamaConfig(hidden_size=d * 2, num_attention_heads=2, head_dim=d,
                          rope_parameters={"rope_type": "default", "rope_theta": 10000.0})
        lib, _ = LlamaRotaryEmbedding.compute_default_rope_parameters(cfg)
        ours = rope3d.inv_freq(d)
        assert ours[0] == 1.0
        np.testing.assert_allclose(ours, lib.double().numpy(), rtol=6e-7, atol=0)   # the library computes in float32


def _fhw(key):
    return tuple(int(v) for v in _facts()[key].split(","))


@pytest.mark.parametrize("head_dim,split,ntk", [(64, None, 1.0), (128, None, 1.0),
                                                (64, "example_fhw_dim", 1.0),
                                                (128, "video_head_fhw_dim", 1.0),
                                                (64, "example_fhw_dim", 4.0),
                                                (128, None, 2.5)])
def test_each_axis_is_library_1d_rope(head_dim, split, ntk):
    """Features of axis a rotate exactly as a 1D RoPE of dimension d_a at that coordinate,
    with the default split or the pages' explicit fhw_dim splits, and with theta multiplied
    by ntk_factor ("NTK-Aware Frequency Scaling")."""
    rng = np.random.default_rng(7)
    pph, ppw, psi = 5, 7, 6
    frame = 37
    split = _fhw(split) if split else None
    x = rng.standard_normal((psi + pph * ppw, 1, head_dim))
    out = rope3d.rotate_frame(x, frame, psi, pph, ppw, split=split, ntk_factor=ntk)
    pos = rope3d.token_positions(frame, psi, pph, ppw)
    # the axis sizes come from the pages (explicit split) or the stated default reading
    d_t, d_h, d_w = split if split else {64: (24, 20, 20), 128: (44, 42, 42)}[head_dim]
    assert sum((d_t, d_h, d_w)) == head_dim
    lo = 0
    for axis, d in enumerate((d_t, d_h, d_w)):
        seg = x[:, 0, lo:lo + d]
        half = np.concatenate([seg[:, 0::2], seg[:, 1::2]], axis=1)   # adjacent -> rotate-half
        lib = _llama_rope(d, pos[:, axis], half, theta=10000.0 * ntk)
        back = np.empty_like(seg)
        back[:, 0::2] = lib[:, :d // 2]
        back[:, 1::2] = lib[:, d // 2:]
        np.testing.assert_allclose(out[:, 0, lo:lo + d], back, atol=2e-5, rtol=0)
        lo += d


def test_rotation_is_complex_multiplication():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 3, 64))
    ang = rng.uniform(-50, 50, (50, 32))
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * ang)[:, None, :]
    out = rope3d.rotate(x, ang)
    np.testing.assert_allclose(out[..., 0::2], z.real, atol=1e-13)
    np.testing.assert_allclose(out[..., 1::2], z.imag, atol=1e-13)


def test_rotation_preserves_pair_norms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3 * 4 * 5 + 6, 4, 128))
    y = rope3d.rotate_frame(x, 1234, 6, 6, 10)
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("head_dim", [64, 128])
def test_scores_depend_only_on_position_offsets(head_dim):
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, head_dim))
    k = rng.standard_normal((1, 1, head_dim))
    for _ in range(20):
        p = rng.integers(0, 500, 3)
        pk = rng.integers(0, 500, 3)
        delta = rng.integers(-200, 200, 3)
        a = rope3d.angles_for_positions(p[None], head_dim)
        b = rope3d.angles_for_positions(pk[None], head_dim)
        a2 = rope3d.angles_for_positions((p + delta)[None], head_dim)
        b2 = rope3d.angles_for_positions((pk + delta)[None], head_dim)
        s1 = float(np.sum(rope3d.rotate(q, a) * rope3d.rotate(k, b)))
        s2 = float(np.sum(rope3d.rotate(q, a2) * rope3d.rotate(k, b2)))
        assert abs(s1 - s2) < 1e-9 * (1 + abs(s1))
    # a change of one axis alone changes the score (no axis is silently dropped)
    base = rope3d.angles_for_positions(np.array([[10, 3, 4]]), head_dim)
    for axis in range(3):
        pp = np.array([[10, 3, 4]])
        pp[0, axis] += 1
        s1 = float(np.sum(rope3d.rotate(q, base) * k))
        s2 = float(np.sum(rope3d.rotate(q, rope3d.angles_for_positions(pp, head_dim)) * k))
        assert abs(s1 - s2) > 1e-6


def test_positions_and_identity_at_origin():
    pos = rope3d.token_positions(0, 6, 3, 4)
    assert pos.shape == (18, 3)
    # brute force over the grid: specials at (0,0,0), patches row-major at (1+r, 1+c)
    for j in range(6):
        assert tuple(pos[j]) == (0, 0, 0)
    j = 6
    for r in range(3):
        for c in range(4):
            assert tuple(pos[j]) == (0, 1 + r, 1 + c)
            j += 1
    x = np.random.default_rng(4).standard_normal((18, 2, 64))
    y = rope3d.rotate_frame(x, 0, 6, 3, 4)
    np.testing.assert_array_equal(y[:6], x[:6])          # frame-0 specials: identity
    assert np.abs(y[6:] - x[6:]).max() > 0.1
    # t only enters through frame_idx
    pos7 = rope3d.token_positions(7, 6, 3, 4)
    assert (pos7[:, 0] == 7).all() and (pos7[:, 1:] == pos[:, 1:]).all()


def test_expanded_table_rows_follow_token_order():
    cos, sin = rope3d.expanded_table(64, 3, 2, 3, 6, f_start=5)
    T = 6 + 6
    for f in range(3):
        ang = rope3d.angles_for_positions(rope3d.token_positions(5 + f, 6, 2, 3), 64)
        np.testing.assert_array_equal(cos[f * T:(f + 1) * T], np.cos(ang))
        np.testing.assert_array_equal(sin[f * T:(f + 1) * T], np.sin(ang))

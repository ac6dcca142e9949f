"""Pins of the oracle's 2D RoPE (CPU only).

"How to Handle Sequences Exceeding the RoPE Training Range in LingBot-Map": sections
"Spatial Position Encoding" (a (y, x) position per patch; the features split into a y half and
an x half, each rotated by a 1D rotary embedding), "Automatic Cache Generation During Forward
Pass" (frequency 100, dim divisible by 4, the 64 x 64 example and its output shape) and
"Deriving Size from Token Count" (a table row per token).  Each test ties ``oracle.rope2d`` to
something other than itself: the values the page prints (``tests/golden/page_facts.txt``),
transformers' LLaMA 1D rotary embedding per half, and invariants of rotary embeddings.
"""

import numpy as np
import pytest
import torch

from oracle import rope2d, rope3d

from test_oracle_rope import _facts, _llama_rope


def test_page_example_shapes():
    f = _facts()
    gh, gw = (int(v) for v in f["rope2d_example_grid"].split(","))
    n = int(f["rope2d_example_tokens"])
    assert gh * gw == n
    b, heads, dim = (int(f[k]) for k in ("rope2d_example_batch", "rope2d_example_heads",
                                         "rope2d_example_dim"))
    pos = np.stack([rope2d.position_getter(gh, gw)] * b)
    assert pos.shape == (b, n, 2)
    x = np.random.default_rng(0).standard_normal((b, heads, n, dim))
    out = rope2d.rotate_grid(x, pos, float(f["rope2d_example_frequency"]))
    assert out.shape == (b, heads, n, dim)
    # the table of a half: dim // 2 features, a row per token (not max position + 1 = 64)
    cos, sin = rope2d.frequency_components(dim // 2, n, float(f["rope2d_example_frequency"]))
    assert cos.shape == sin.shape == (n, dim // 4)
    cos, _ = rope2d.frequency_components(int(f["rope2d_prepopulate_features"]),
                                         int(f["rope2d_prepopulate_seq_len"]))
    assert cos.shape == (int(f["rope2d_prepopulate_seq_len"]),
                         int(f["rope2d_prepopulate_features"]) // 2)
    assert float(f["rope2d_example_scaling_factor"]) == 1.0    # the only value given


def test_dim_must_split_into_two_halves_of_pairs():
    for bad in (2, 6, 66, 130):
        with pytest.raises(ValueError):
            rope2d.half_dim(bad)
    assert rope2d.half_dim(64) == 32 and rope2d.half_dim(128) == 64


@pytest.mark.parametrize("head_dim", [64, 128])
def test_each_half_is_library_1d_rope(head_dim):
    """The y half rotates as a 1D RoPE of dimension head_dim/2 with base 100 at y, the x half
    as one at x (transformers' LLaMA rotary embedding, re-paired from rotate-half)."""
    f = _facts()
    freq = float(f["rope2d_example_frequency"])
    rng = np.random.default_rng(3)
    pph, ppw, psi = 6, 9, 6
    x = rng.standard_normal((psi + pph * ppw, 1, head_dim))
    out = rope2d.rotate_frame(x, psi, pph, ppw, freq)
    pos = rope2d.token_positions(psi, pph, ppw)
    d = head_dim // 2
    for axis in range(2):
        seg = x[:, 0, axis * d:(axis + 1) * d]
        half = np.concatenate([seg[:, 0::2], seg[:, 1::2]], axis=1)
        lib = _llama_rope(d, pos[:, axis], half, theta=freq)
        back = np.empty_like(seg)
        back[:, 0::2] = lib[:, :d // 2]
        back[:, 1::2] = lib[:, d // 2:]
        np.testing.assert_allclose(out[:, 0, axis * d:(axis + 1) * d], back, atol=2e-5, rtol=0)


def test_inv_freq_matches_library():
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    for d in (32, 64):
        cfg = LlamaConfig(hidden_size=d * 2, num_attention_heads=2, head_dim=d,
                          rope_parameters={"rope_type": "default", "rope_theta": 100.0})
        lib, _ = LlamaRotaryEmbedding.compute_default_rope_parameters(cfg)
        np.testing.assert_allclose(rope2d.inv_freq(d, 100.0), lib.double().numpy(), rtol=6e-7)


def test_scores_depend_on_the_spatial_offset_only():
    """<R(p) q, R(p') k> is unchanged by moving both positions by the same (dy, dx), changes
    with either coordinate, and does not see the frame index at all."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 64))
    k = rng.standard_normal((1, 1, 64))

    def score(pq, pk):
        aq = rope2d.angles_for_positions(np.array([pq]), 64, seq_len=64)
        ak = rope2d.angles_for_positions(np.array([pk]), 64, seq_len=64)
        return float((rope3d.rotate(q, aq) * rope3d.rotate(k, ak)).sum())

    base = score((3, 5), (7, 2))
    assert abs(score((13, 25), (17, 22)) - base) < 1e-12
    assert abs(score((4, 5), (7, 2)) - base) > 1e-6          # y matters
    assert abs(score((3, 6), (7, 2)) - base) > 1e-6          # x matters
    # rotation preserves each pair's norm; specials at (0, 0) are left unchanged
    x = rng.standard_normal((6 + 12, 2, 64))
    r = rope2d.rotate_frame(x, 6, 3, 4)
    np.testing.assert_allclose(np.hypot(r[..., 0::2], r[..., 1::2]),
                               np.hypot(x[..., 0::2], x[..., 1::2]), rtol=1e-12)
    np.testing.assert_array_equal(r[:6], x[:6])


def test_table_rows_follow_the_token_count():
    """Positions are looked up in a table of one row per token; a coordinate past it is an
    error, not a silent extrapolation."""
    pos = rope2d.token_positions(6, 4, 5)
    assert pos.max() < len(pos)
    with pytest.raises(ValueError):
        rope2d.angles_for_positions(np.array([[0, 9]]), 64, seq_len=9)


def test_stream_oracle_2d_mode_rotates_with_rope2d():
    from oracle import stream
    rng = np.random.default_rng(9)
    so = stream.StreamOracle(2, 64, 3, 4, 1, 1, 4, rope2d_frequency=100.0)
    q, k, v = (rng.standard_normal((18, 2, 64)) for _ in range(3))
    for f in (0, 7):                                    # the frame index does not matter
        r = so.step(f, True, q, k, v)
        np.testing.assert_allclose(r.q_rot, rope2d.rotate_frame(q, 6, 3, 4), rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.k_rot, rope2d.rotate_frame(k, 6, 3, 4), rtol=0, atol=1e-12)

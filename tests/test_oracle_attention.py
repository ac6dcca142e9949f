"""Pins of the oracle's attention and of the whole-stream driver (CPU only).

Ties ``oracle.attention`` / ``oracle.stream`` to torch's scaled_dot_product_attention on the
CPU in float64 (a library routine), to brute-force Python loops on tiny inputs, and to
properties every softmax attention has.  The key set follows "How 3D RoPE Positional
Encoding Works with the Paged KV Cache in LingBot-Map" (section "Attention Computation
with Cached RoPE") and "How LingBot-Map Achieves Real-Time 3D Reconstruction" (section
"Per-Frame Processing and Causal Attention").
"""

import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import attention, retention, rope3d, stream
from rope_paged_kv_02_b200.workloads import CONFIGS, custom_config, frame_qkv


def _sdpa(q, k, v, mask=None):
    qt = torch.tensor(q, dtype=torch.float64).permute(1, 0, 2)
    kt = torch.tensor(k, dtype=torch.float64).permute(1, 0, 2)
    vt = torch.tensor(v, dtype=torch.float64).permute(1, 0, 2)
    m = None if mask is None else torch.tensor(mask, dtype=torch.bool)[None, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], attn_mask=m)
    return o[0].permute(1, 0, 2).numpy()


def test_attend_matches_torch_sdpa_and_brute_force():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((5, 2, 8))
    k = rng.standard_normal((11, 2, 8))
    v = rng.standard_normal((11, 2, 8))
    out, lse = attention.attend(q, k, v, return_lse=True)
    np.testing.assert_allclose(out, _sdpa(q, k, v), atol=1e-13)
    for t in range(5):
        for h in range(2):
            s = [sum(q[t, h, d] * k[n, h, d] for d in range(8)) / math.sqrt(8) for n in range(11)]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            z = sum(e)
            for d in range(8):
                ref = sum(e[n] * v[n, h, d] for n in range(11)) / z
                assert abs(out[t, h, d] - ref) < 1e-12
            assert abs(lse[t, h] - logsumexp(np.array(s))) < 1e-12
    mask = rng.random(11) < 0.5
    mask[3] = True
    np.testing.assert_allclose(attention.attend_masked(q, k, v, mask),
                               _sdpa(q, k, v, mask), atol=1e-13)
    np.testing.assert_allclose(attention.attend_masked(q, k, v, mask),
                               attention.attend(q, k[mask], v[mask]), atol=1e-13)


def test_attention_properties():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((7, 3, 16))
    k = rng.standard_normal((40, 3, 16))
    v = np.broadcast_to(rng.standard_normal((1, 3, 16)), (40, 3, 16)).copy()
    np.testing.assert_allclose(attention.attend(q, k, v), np.broadcast_to(v[:1], (7, 3, 16)),
                               atol=1e-14)                                   # constant V
    v = rng.standard_normal((40, 3, 16))
    one = attention.attend(q, k[5:6], v[5:6])
    np.testing.assert_allclose(one, np.broadcast_to(v[5:6], (7, 3, 16)), atol=1e-15)
    perm = rng.permutation(40)
    np.testing.assert_allclose(attention.attend(q, k[perm], v[perm]), attention.attend(q, k, v),
                               atol=1e-13)                                   # key order
    rows = [0, 3, 6]
    np.testing.assert_allclose(attention.attend(q[rows], k, v), attention.attend(q, k, v)[rows],
                               atol=1e-14, rtol=0)                           # rows independent


@pytest.mark.parametrize("cfg", [CONFIGS[0],
                                 custom_config(100, 2, 64, "bf16", 3, 5, 12, 2, 1, 2),
                                 custom_config(101, 1, 128, "bf16", 2, 3, 9, 3, 0, 1)])
def test_stream_two_formulations_agree(cfg):
    """Retained-keys attention == whole-history masked attention (closed-form mask)."""
    so = stream.StreamOracle(cfg.heads, cfg.head_dim, cfg.pph, cfg.ppw, cfg.scale_frames,
                             cfg.sliding_window, cfg.n_keyframes, keep_history=True)
    committed = []
    for f, key in enumerate(cfg.keyframes):
        q, k, v = frame_qkv(cfg, f)
        r = so.step(f, key, q, k, v)
        masked = so.attend_history_masked(r.q_rot, f, committed)
        np.testing.assert_allclose(r.out, masked, atol=1e-12, rtol=0)
        if key:
            committed.append(f)


def test_full_window_equals_frame_causal_attention():
    """With a window longer than the stream and all keyframes, every earlier token is seen."""
    cfg = custom_config(102, 2, 64, "f32", 2, 3, 7, 1, 2, 10)
    so = stream.StreamOracle(cfg.heads, cfg.head_dim, cfg.pph, cfg.ppw, cfg.scale_frames,
                             cfg.sliding_window, cfg.n_keyframes)
    ks, vs = [], []
    for f in range(cfg.n_frames):
        q, k, v = frame_qkv(cfg, f)
        r = so.step(f, True, q, k, v)
        qr = rope3d.rotate_frame(q, f, 6, cfg.pph, cfg.ppw)
        ks.append(rope3d.rotate_frame(k, f, 6, cfg.pph, cfg.ppw))
        vs.append(v.astype(np.float64))
        ref = _sdpa(qr, np.concatenate(ks), np.concatenate(vs))
        np.testing.assert_allclose(r.out, ref, atol=1e-12)


def _needle_stream(W):
    cfg = custom_config(103, 1, 64, "f32", 2, 4, 6, 1, 1, W)
    q5, _, _ = frame_qkv(cfg, 5)
    q5r = rope3d.rotate_frame(q5, 5, 6, 2, 4)
    ang = rope3d.angles_for_positions(rope3d.token_positions(2, 6, 2, 4)[9:10], 64)
    so = stream.StreamOracle(1, 64, 2, 4, 1, W, 6)
    needle_v = None
    for f in range(6):
        q, k, v = frame_qkv(cfg, f)
        if f == 2:
            # a key whose rotated form is 4 * (rotated query 0 of frame 5)
            k = k.astype(np.float64)
            k[9] = rope3d.rotate(4.0 * q5r[0:1], -ang)[0]
            needle_v = v[9, 0].astype(np.float64)
        r = so.step(f, True, q, k, v)
    return r, needle_v


def test_needle_key_is_found_in_its_page():
    """A planted key equal to 4*q in a retained page dominates that query's output."""
    r, needle_v = _needle_stream(3)
    assert r.visible_frames == [0, 2, 3, 4, 5]
    np.testing.assert_allclose(r.out[0, 0], needle_v, atol=1e-3)
    r, needle_v = _needle_stream(2)           # frame 2 evicted before frame 5
    assert r.visible_frames == [0, 3, 4, 5]
    assert np.abs(r.out[0, 0] - needle_v).max() > 0.1


def test_regenerated_kv_source_matches_stored_kv():
    """The long-stream mode (retained keys re-created from the seeded inputs) agrees exactly."""
    cfg = custom_config(104, 2, 64, "bf16", 3, 4, 15, 2, 1, 3)

    def source(frame, region):
        q, k, v = frame_qkv(cfg, frame)
        sl = slice(6, None) if region == "patch" else slice(0, 6)
        return k[sl], v[sl]

    a = stream.StreamOracle(2, 64, 3, 4, 1, 3, cfg.n_keyframes)
    b = stream.StreamOracle(2, 64, 3, 4, 1, 3, cfg.n_keyframes, kv_source=source)
    for f, key in enumerate(cfg.keyframes):
        q, k, v = frame_qkv(cfg, f)
        ra = a.step(f, key, q, k, v)
        rb = b.step(f, key, q, k, v, rows=[0, 5, 7, 17])
        np.testing.assert_allclose(rb.out, ra.out[[0, 5, 7, 17]], atol=1e-13, rtol=0)
        assert ra.state == rb.state

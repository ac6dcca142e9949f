"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on seeded inputs.

Steps checked per frame (tolerances in ``tests/stream_check.py``): the 3D RoPE of q (in
place) and of k, the pages and special slots written by the fused rotate+append kernel,
the page table / free list / retained frames (bit-exact) and the paged attention output.
"""

import os

import numpy as np
import pytest

from oracle import rope3d
from rope_paged_kv_02_b200 import _lib
from rope_paged_kv_02_b200.workloads import CONFIGS, custom_config

from stream_check import run_stream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rope_paged_kv_02_b200.build import build
    build()
    _lib.load()


@pytest.mark.parametrize("head_dim,ppf,pph,ppw", [(64, 30, 14, 14), (128, 5, 64, 64),
                                                  (64, 2000, 37, 27)])
def test_rope_tables_match_oracle(head_dim, ppf, pph, ppw):
    import torch
    rope = _lib.Rope3D(head_dim, ppf, pph, ppw, 6)
    rows = ppf * (6 + pph * ppw)
    cos = torch.empty(rows, head_dim // 2, device="cuda")
    sin = torch.empty_like(cos)
    rope.expand(cos, sin)
    torch.cuda.synchronize()
    ec, es = rope3d.expanded_table(head_dim, ppf, pph, ppw, 6)
    assert np.abs(cos.cpu().numpy() - ec).max() <= 1e-5
    assert np.abs(sin.cpu().numpy() - es).max() <= 1e-5
    rope.close()


@pytest.mark.parametrize("head_dim,split,ntk", [(64, (20, 22, 22), 1.0), (128, (40, 44, 44), 4.0),
                                                (64, None, 2.0)])
def test_rope_variant_tables_match_oracle(head_dim, split, ntk):
    """Explicit (t, h, w) splits as printed on the pages, and the NTK factor."""
    import torch
    rope = _lib.Rope3D(head_dim, 12, 9, 11, 6, split=split, ntk_factor=ntk)
    rows = 12 * (6 + 9 * 11)
    cos = torch.empty(rows, head_dim // 2, device="cuda")
    sin = torch.empty_like(cos)
    rope.expand(cos, sin)
    torch.cuda.synchronize()
    ec, es = rope3d.expanded_table(head_dim, 12, 9, 11, 6, split=split, ntk_factor=ntk)
    assert np.abs(cos.cpu().numpy() - ec).max() <= 1e-5
    assert np.abs(sin.cpu().numpy() - es).max() <= 1e-5
    rope.close()


@pytest.mark.parametrize("head_dim,split,ntk", [(64, (20, 22, 22), 1.0), (128, (40, 44, 44), 4.0)])
def test_rope_variant_stream(head_dim, split, ntk):
    """Fused rotate + append and attention with a RoPE variant: q, pages and outputs match
    the oracle rotating with the same split and NTK factor."""
    run_stream(custom_config(211 + head_dim // 64, 2, head_dim, "bf16", 5, 8, 7, 2, 1, 2),
               split=split, ntk_factor=ntk)


@pytest.mark.parametrize("head_dim,ppf,pph,ppw", [(64, 4, 9, 11), (128, 3, 64, 64)])
def test_rope2d_tables_match_oracle(head_dim, ppf, pph, ppw):
    """The 2D (y, x) variant ("How to Handle Sequences Exceeding the RoPE Training Range in
    LingBot-Map"): the tables the library builds, expanded per token, equal the oracle's."""
    import torch
    from oracle import rope2d
    rope = _lib.Rope2D(head_dim, ppf, pph, ppw, 6, frequency=100.0)
    rows = ppf * (6 + pph * ppw)
    cos = torch.empty(rows, head_dim // 2, device="cuda")
    sin = torch.empty_like(cos)
    rope.expand(cos, sin)
    torch.cuda.synchronize()
    ec, es = rope2d.expanded_table(head_dim, ppf, pph, ppw, 6, 100.0)
    assert np.abs(cos.cpu().numpy() - ec).max() <= 1e-5
    assert np.abs(sin.cpu().numpy() - es).max() <= 1e-5
    rope.close()


@pytest.mark.parametrize("head_dim", [64, 128])
def test_rope2d_stream_all_frames_all_rows(head_dim):
    """Fused rotate + append and attention with the 2D variant: q, pages, page table and
    outputs match the oracle rotating by (y, x) with base frequency 100."""
    cfg = custom_config(222 + head_dim // 64, 2, head_dim, "bf16", 7, 9, 8, 2, 1, 2)
    run_stream(cfg, rope2d_frequency=100.0)
    run_stream(cfg, rope2d_frequency=100.0, fold_q=True)


def test_rope2d_64x64_grid_sampled():
    """The page's high-resolution case: a 64 x 64 grid (4096 patch tokens), 8 heads x 128;
    135 sampled query rows (all specials, the last row, 128 random) at every frame."""
    cfg = custom_config(225, 8, 128, "bf16", 64, 64, 5, 1, 1, 2, v_dist="uniform")
    rng = np.random.default_rng(225)
    rows = np.unique(np.concatenate([np.arange(6), [cfg.tokens - 1],
                                     rng.choice(np.arange(6, cfg.tokens - 1), 128,
                                                replace=False)]))
    run_stream(cfg, rows=rows, rope2d_frequency=100.0)


def test_tiny_fp32_config_all_frames():
    run_stream(CONFIGS[0])


SMALL = [
    # two query tiles with a ragged tail, two key tiles per page (130 patches), keyframe
    # every 2nd frame (rollbacks)
    custom_config(200, 2, 64, "bf16", 10, 13, 9, 2, 1, 2),
    # head_dim 128, odd patch count, keyframe every 3rd frame
    custom_config(201, 2, 128, "bf16", 9, 15, 12, 3, 2, 1),
    # T = 22 < 128; no scale frames; specials cross the 128-token special page at frame 21
    custom_config(202, 3, 64, "bf16", 4, 4, 40, 1, 0, 3),
    # no sliding window: every frame after the scale frames is evicted right after attending
    custom_config(203, 1, 64, "bf16", 6, 6, 6, 1, 2, 0),
    # fp32 cache, head_dim 128
    custom_config(204, 2, 128, "f32", 3, 5, 7, 2, 1, 2),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_streams_all_frames_all_rows(cfg):
    run_stream(cfg)


@pytest.mark.parametrize("cfg", [c for c in SMALL if c.dtype == "bf16"], ids=lambda c: c.name)
def test_small_streams_rotation_folded_into_attention(cfg):
    """The folded path: the append moves k and v only, the attention kernel rotates the raw q
    in shared memory after its TMA load; the rotated q it used is checked like the in-place
    rotation (1/2 bf16 ulp), outputs, pages and page table like every stream."""
    run_stream(cfg, fold_q=True)


def test_folded_rotation_argument_checks():
    """lbm_attend_frame_qrot only for frames whose append left q to the attention; a float32
    cache cannot fold the rotation (its attention is the SIMT kernel)."""
    import torch
    rope = _lib.Rope3D(64, 4, 4, 4, 6)
    cache = _lib.PagedKVCache(rope, 2, 64, 16, 1, 1, 4, _lib.LBM_BF16)
    q = torch.randn(22, 2, 64, device="cuda").to(torch.bfloat16)
    k, v, out, qr = torch.randn_like(q), torch.randn_like(q), torch.empty_like(q), torch.empty_like(q)
    cache.append_frame(q, k, v, 0, True)                  # q rotated here
    with pytest.raises(_lib.LbmError) as e:
        cache.attend_frame(q, out, q_rot_out=qr)
    assert e.value.status == _lib.LBM_ERR_INVALID
    cache.attend_frame(q, out)
    cache.append_frame(None, k, v, 1, True)               # q left to the attention
    cache.attend_frame(q, out, q_rot_out=qr)
    cache.check()
    cache.close()
    rope32 = _lib.Rope3D(64, 4, 4, 4, 6)
    c32 = _lib.PagedKVCache(rope32, 2, 64, 16, 1, 1, 4, _lib.LBM_F32)
    q32 = torch.randn(22, 2, 64, device="cuda")
    with pytest.raises(_lib.LbmError) as e:
        c32.append_frame(None, q32, q32, 0, True)
    assert e.value.status == _lib.LBM_ERR_UNSUPPORTED
    c32.close()
    rope32.close()
    rope.close()


@pytest.mark.parametrize("grid", ["1", "3", "16", "148"])
def test_forced_grid_sizes_agree(grid, monkeypatch):
    monkeypatch.setenv("LBM_ATTN_GRID", grid)
    cfg = custom_config(205, 2, 64, "bf16", 12, 12, 8, 1, 2, 3)
    run_stream(cfg)
    run_stream(cfg, fold_q=True)          # the folded kernel walks the same segments


def test_keyframes_decided_after_attention():
    """[KVBenefits] "Dynamic Keyframe Selection": each frame is appended undecided, attends,
    and is then kept or dropped (every 3rd kept); outputs, pages and page table match the
    oracle that took the same decisions at append."""
    run_stream(custom_config(210, 2, 64, "bf16", 6, 9, 14, 3, 1, 2), decide_after=True)


def test_windowed_stream_resets_between_windows():
    """[KVBenefits] "Cross-Window Alignment for Long Videos": a long video processed in
    windows, the cache cleaned (lbm_cache_reset) before each window and frame indices
    starting again at 0: every window matches a fresh oracle, so nothing of an earlier window
    (pages, special tokens) stays visible."""
    cfg = custom_config(214, 2, 64, "bf16", 6, 7, 21, 2, 1, 2)
    run_stream(cfg, frame_ids=list(range(7)) * 3, reset_at=(7, 14))


def test_non_contiguous_frame_indices():
    cfg = custom_config(206, 2, 64, "bf16", 5, 7, 8, 2, 1, 2)
    run_stream(cfg, frame_ids=[0, 3, 4, 10, 11, 20, 57, 58])


def _needle(cfg, n_needle_frame, target_frame, row, boost, page_pos=5):
    """Tamper hook: plant at frame n_needle_frame, page position page_pos, a key equal to
    boost * (rotated q of target_frame, row), and scale every q by 4 (peaked softmax: scores
    of std 4, the needle's about 25)."""
    from rope_paged_kv_02_b200.workloads import frame_qkv, round_bf16
    q_t, _, _ = frame_qkv(cfg, target_frame)
    q_rot = rope3d.rotate_frame(q_t.astype(np.float64) * 4.0, target_frame, 6, cfg.pph, cfg.ppw)
    slot = 6 + page_pos
    pos = rope3d.token_positions(n_needle_frame, 6, cfg.pph, cfg.ppw)[slot:slot + 1]
    kneedle = rope3d.rotate(boost * q_rot[row:row + 1],
                            -rope3d.angles_for_positions(pos, cfg.head_dim))[0]

    def tamper(n, q, k, v):
        q = q * np.float32(4.0)       # exact in bf16 and fp32
        if n == n_needle_frame:
            k = k.copy()
            k[slot] = round_bf16(kneedle.astype(np.float32)) if cfg.dtype == "bf16" else kneedle
        return q, k, v

    return tamper


def test_peaked_softmax_with_needle_key():
    cfg = custom_config(207, 2, 64, "bf16", 10, 13, 6, 1, 1, 3)
    tamper = _needle(cfg, 2, 5, 0, 0.2)
    run_stream(cfg, tamper=tamper)


@pytest.mark.parametrize("page_pos", [40, 70, 100, 129])
def test_needle_key_past_the_first_score_chunk(page_pos):
    """head_dim 64 reads a 128-key tile in four 32-key chunks and may move its reference max
    at any chunk: a needle at key 40, 70 or 100 of its page's first tile (chunks 1, 2, 3) or
    at key 129 (second tile) makes the max jump after P of earlier chunks was produced, so
    those are scaled again; the output must still match the oracle."""
    cfg = custom_config(207, 2, 64, "bf16", 10, 13, 6, 1, 1, 3)
    tamper = _needle(cfg, 2, 5, 0, 0.2, page_pos=page_pos)
    run_stream(cfg, tamper=tamper)


@pytest.mark.parametrize("cid,frames", [
    (1, [0, 1, 8, 24, 25, 63]),
    (2, [0, 4, 5, 315, 316, 319]),
    (4, [0, 36, 37, 95]),
])
def test_full_size_config_sampled(cid, frames):
    cfg = CONFIGS[cid]
    rng = np.random.default_rng(cid)
    rows = np.unique(np.concatenate([np.arange(6), [cfg.tokens - 1],
                                     rng.choice(np.arange(6, cfg.tokens - 1), 128,
                                                replace=False)]))
    assert len(rows) == 128 + 7
    run_stream(cfg, check_frames=frames, rows=rows, regenerate=True)


def test_full_size_768_folded_sampled():
    """The folded rotation at full size (768-patch stream, frames around the window fill)."""
    cfg = CONFIGS[1]
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([np.arange(6), [cfg.tokens - 1],
                                     rng.choice(np.arange(6, cfg.tokens - 1), 128,
                                                replace=False)]))
    run_stream(cfg, check_frames=[0, 24, 25, 63], rows=rows, regenerate=True, fold_q=True)


@pytest.mark.slow
def test_long_stream_2000_keyframes_sampled():
    cfg = CONFIGS[3]
    rng = np.random.default_rng(3)
    # every special row, the last row and 128 random rows (>= 128 query rows, all heads);
    # pools (K rotated at t up to 1999, V copied) checked at every sampled frame
    rows = np.unique(np.concatenate([np.arange(6), [cfg.tokens - 1],
                                     rng.choice(np.arange(6, cfg.tokens - 1), 128,
                                                replace=False)]))
    assert len(rows) >= 128 + 7
    run_stream(cfg, check_frames=[0, 135, 136, 137, 1000, 1999], rows=rows, regenerate=True,
               check_pools=True)


@pytest.mark.parametrize("head_dim", [64, 128])
def test_single_patch_frames(head_dim):
    """The smallest frame: 6 special tokens and one patch (T = 7, one mostly padded query
    tile, one-key patch pages)."""
    run_stream(custom_config(218 + head_dim // 64, 1, head_dim, "bf16", 1, 1, 9, 2, 1, 2))


@pytest.mark.slow
def test_maximum_page_count():
    """The largest page table the cache takes (scale_frames + sliding_window + 1 = 1024 =
    LBM_MAX_PAGES) over a stream long enough to fill and roll it: the kernel's visible page
    list is full, and each unit's ~1000 key tiles are spread over every CTA, so the combine
    merges ~70 partials a row."""
    cfg = custom_config(221, 2, 64, "bf16", 4, 4, 1030, 1, 8, 1015)
    run_stream(cfg, check_frames=[0, 1, 1022, 1023, 1024, 1029], regenerate=True)


def test_sequence_errors_leave_state_unchanged():
    import torch
    cfg = custom_config(208, 2, 64, "bf16", 4, 4, 4, 1, 1, 1)
    rope = _lib.Rope3D(64, 4, 4, 4, 6)
    cache = _lib.PagedKVCache(rope, 2, 64, 16, 1, 1, 2, _lib.LBM_BF16)
    q = torch.randn(22, 2, 64, device="cuda").to(torch.bfloat16)
    k, v, out = torch.randn_like(q), torch.randn_like(q), torch.empty_like(q)
    with pytest.raises(_lib.LbmError) as e:
        cache.attend_frame(q, out)                        # nothing appended
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    cache.append_frame(q, k, v, 0, True)
    s0 = cache.state()
    with pytest.raises(_lib.LbmError) as e:
        cache.append_frame(q, k, v, 1, True)              # append twice
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    assert cache.state() == s0
    cache.attend_frame(q, out)
    with pytest.raises(_lib.LbmError) as e:
        cache.append_frame(q, k, v, 4, True)              # beyond the t table (ppf = 4)
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    with pytest.raises(_lib.LbmError) as e:
        cache.append_frame(q, k, v, 0, True)              # frame index must increase
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    bad = q.view(-1)[1:].view(-1)                         # 2-byte offset: misaligned
    with pytest.raises(_lib.LbmError) as e:
        cache.append_frame(bad, k, v, 1, True)
    assert e.value.status == _lib.LBM_ERR_INVALID
    cache.append_frame(q, k, v, 1, True)
    cache.attend_frame(q, out)
    s1 = cache.state()
    with pytest.raises(_lib.LbmError) as e:
        cache.append_frame(q, k, v, 2, True)              # max_frames = 2 keyframes held
    assert e.value.status == _lib.LBM_ERR_CAPACITY
    assert cache.state() == s1
    cache.append_frame(q, k, v, 2, False)                 # a non-keyframe still fits
    cache.attend_frame(q, out)
    cache.check()
    cache.reset()
    st = cache.state()
    assert st["free"] == [2, 1, 0] and st["n_special"] == 0 and not st["pending"]
    cache.append_frame(q, k, v, 0, None)                  # decided after attention
    with pytest.raises(_lib.LbmError) as e:
        cache.commit_frame(True)                          # not attended yet
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    cache.attend_frame(q, out)
    with pytest.raises(_lib.LbmError) as e:
        cache.attend_frame(q, out)                        # attended, still undecided
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    cache.commit_frame(True)
    assert cache.state()["scale_frames"] == [0] and not cache.state()["pending"]
    cache.check()
    with pytest.raises(_lib.LbmError) as e:
        _lib.PagedKVCache(rope, 2, 96, 16, 1, 1, 2, _lib.LBM_BF16)
    assert e.value.status == _lib.LBM_ERR_UNSUPPORTED
    with pytest.raises(_lib.LbmError) as e:
        _lib.PagedKVCache(rope, 2, 64, 15, 1, 1, 2, _lib.LBM_BF16)   # != pph * ppw
    assert e.value.status == _lib.LBM_ERR_INVALID
    cache.close()
    rope.close()


def test_calls_on_two_streams_are_ordered():
    """append on one stream, attend on another: the library orders them with its event."""
    import torch
    cfg = custom_config(209, 2, 64, "bf16", 8, 8, 6, 1, 1, 2)
    from rope_paged_kv_02_b200.workloads import frame_qkv
    from oracle import stream as ostream
    from stream_check import check_attn, dev, host
    rope = _lib.Rope3D(64, 6, 8, 8, 6)
    cache = _lib.PagedKVCache(rope, 2, 64, 64, 1, 2, 6, _lib.LBM_BF16)
    so = ostream.StreamOracle(2, 64, 8, 8, 1, 2, 6)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for f in range(6):
        q, k, v = frame_qkv(cfg, f)
        with torch.cuda.stream(s1):
            qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
            out = torch.empty_like(qd)
            cache.append_frame(qd, kd, vd, f, True, stream=s1)
        s2.wait_stream(s1)    # the caller orders its own buffers; the cache orders itself
        cache.attend_frame(qd, out, stream=s2)
        torch.cuda.synchronize()
        r = so.step(f, True, q, k, v)
        check_attn(host(out), r.out, f"frame {f}")
    cache.close()
    rope.close()


def test_multi_block_cache_shares_the_page_table():
    """[3DRoPE-KV] "Implementation Example": one cache manager for several transformer blocks
    (num_blocks, block_idx).  Three blocks with their own seeded inputs stream the same frames
    (append then attend per block, blocks in order); each block's outputs and pages match its
    own oracle, and the shared page table matches every oracle's."""
    import torch
    from oracle import stream as ostream
    from stream_check import check_attn, check_rope, dev, host, pool_values
    from rope_paged_kv_02_b200 import workloads
    nb = 3
    cfgs = [custom_config(215 + b, 2, 64, "bf16", 5, 6, 9, 2, 1, 2) for b in range(nb)]
    c0 = cfgs[0]
    rope = _lib.Rope3D(64, c0.n_frames, c0.pph, c0.ppw, 6)
    cache = _lib.PagedKVCache(rope, 2, 64, c0.patches, c0.scale_frames, c0.sliding_window,
                              c0.n_keyframes, _lib.LBM_BF16, num_blocks=nb)
    oracles = [ostream.StreamOracle(2, 64, c0.pph, c0.ppw, c0.scale_frames, c0.sliding_window,
                                    c0.n_keyframes) for _ in range(nb)]
    for f in range(c0.n_frames):
        key = c0.keyframes[f]
        for b in range(nb):
            q, k, v = workloads.frame_qkv(cfgs[b], f)
            qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
            out = torch.empty_like(qd)
            cache.append_frame_block(b, qd, kd, vd, f, key)
            cache.attend_frame_block(b, qd, out)
            r = oracles[b].step(f, key, q, k, v)
            torch.cuda.synchronize()
            check_rope(host(qd), r.q_rot, "bf16", f"block {b} frame {f} q")
            check_attn(host(out), r.out, f"block {b} frame {f} attention")
            kp = pool_values(cache.read_kv(_lib.LBM_K_PATCH, r.page, block=b), "bf16")
            check_rope(kp.transpose(1, 0, 2), r.k_rot[6:], "bf16", f"block {b} K page")
            vp = pool_values(cache.read_kv(_lib.LBM_V_PATCH, r.page, block=b), "bf16")
            np.testing.assert_array_equal(vp.transpose(1, 0, 2), v[6:])
            st = cache.state()
            assert st["pending"] == (b < nb - 1)       # committed after the last block
        for b in range(nb):
            snap = oracles[b].ret.snapshot()
            for k_ in ("scale_pages", "scale_frames", "window_pages", "window_frames", "free",
                       "n_special"):
                assert st[k_] == snap[k_], (f, b, k_)
    cache.check()
    cache.close()
    rope.close()


def test_multi_block_sequence_errors():
    import torch
    rope = _lib.Rope3D(64, 4, 4, 4, 6)
    cache = _lib.PagedKVCache(rope, 2, 64, 16, 1, 1, 4, _lib.LBM_BF16, num_blocks=2)
    q = torch.randn(22, 2, 64, device="cuda").to(torch.bfloat16)
    k, v, out = torch.randn_like(q), torch.randn_like(q), torch.empty_like(q)

    def status(fn, *a):
        with pytest.raises(_lib.LbmError) as e:
            fn(*a)
        return e.value.status

    assert status(cache.append_frame_block, 1, q, k, v, 0, True) == _lib.LBM_ERR_SEQUENCE
    assert status(cache.append_frame_block, 2, q, k, v, 0, True) == _lib.LBM_ERR_INVALID
    cache.append_frame_block(0, q, k, v, 0, True)
    assert status(cache.append_frame_block, 1, q, k, v, 0, True) == _lib.LBM_ERR_SEQUENCE
    assert status(cache.attend_frame_block, 1, q, out) == _lib.LBM_ERR_SEQUENCE
    cache.attend_frame_block(0, q, out)
    assert status(cache.attend_frame_block, 0, q, out) == _lib.LBM_ERR_SEQUENCE
    assert status(cache.append_frame_block, 1, q, k, v, 1, True) == _lib.LBM_ERR_SEQUENCE
    assert status(cache.append_frame_block, 1, q, k, v, 0, False) == _lib.LBM_ERR_INVALID
    s0 = cache.state()
    assert s0["pending"]
    cache.append_frame(q, k, v, 0, True)                  # the next block in order: block 1
    cache.attend_frame(q, out)
    assert not cache.state()["pending"] and cache.state()["scale_frames"] == [0]
    cache.check()
    cache.close()
    rope.close()


@pytest.mark.parametrize("head_dim,fold", [(64, False), (64, True), (128, False), (128, True)])
def test_wait_that_runs_out_is_reported_and_the_cache_recovers(head_dim, fold):
    """Failure detection without a fault: with a wait limit of 1 ns the attention kernel's first
    wait that is not already satisfied runs out; every role leaves the kernel (copies and
    tensor-core operations already issued are drained under the full bound before tensor
    memory is freed), lbm_cache_check reports LBM_ERR_TIMEOUT once and clears it.  With the
    default limit restored and the cache reset, the same cache then streams frames that match
    the oracle, so the context stays usable."""
    import torch
    from oracle import stream as ostream
    from rope_paged_kv_02_b200.workloads import frame_qkv
    from stream_check import check_attn, dev, host
    cfg = custom_config(226 + head_dim // 64, 2, head_dim, "bf16", 10, 13, 4, 1, 1, 2)
    rope = _lib.Rope3D(head_dim, cfg.n_frames, cfg.pph, cfg.ppw, 6)
    cache = _lib.PagedKVCache(rope, 2, head_dim, cfg.patches, 1, 2, cfg.n_frames, _lib.LBM_BF16)
    q, k, v = frame_qkv(cfg, 0)
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    out = torch.empty_like(qd)
    cache.set_wait_limit(1)
    cache.append_frame(None if fold else qd, kd, vd, 0, True)
    cache.attend_frame(qd, out)
    with pytest.raises(_lib.LbmError) as e:
        cache.check()
    assert e.value.status == _lib.LBM_ERR_TIMEOUT
    cache.check()                                         # reported once, then cleared
    with pytest.raises(_lib.LbmError) as e:
        cache.set_wait_limit(3_000_000_000)               # above the 2 s default
    assert e.value.status == _lib.LBM_ERR_INVALID
    cache.set_wait_limit(0)
    cache.reset()
    so = ostream.StreamOracle(2, head_dim, cfg.pph, cfg.ppw, 1, 2, cfg.n_frames)
    for f in range(cfg.n_frames):
        q, k, v = frame_qkv(cfg, f)
        qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
        out = torch.empty_like(qd)
        cache.append_frame(None if fold else qd, kd, vd, f, True)
        cache.attend_frame(qd, out)
        r = so.step(f, True, q, k, v)
        torch.cuda.synchronize()
        check_attn(host(out), r.out, f"frame {f} after the timeout")
    cache.check()
    cache.close()
    rope.close()


@pytest.mark.parametrize("head_dim", [64, 128])
def test_more_units_than_the_rotation_table(head_dim):
    """1100 heads of a 22-token frame: 1100 (query-tile pair, head) units, more than the
    1024 whose key order the planner rotates, so units 1024..1099 read their keys in the
    natural order; every head must still match the oracle."""
    cfg = custom_config(222, 1100, head_dim, "bf16", 4, 4, 6, 1, 1, 3)
    run_stream(cfg, check_frames=[0, 3, 5])

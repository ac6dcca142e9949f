"""Pins of the oracle's retention state machine (CPU only).

Ties ``oracle.retention`` to closed forms and to the numbers the pages print:
"How 3D RoPE Positional Encoding Works with the Paged KV Cache in LingBot-Map"
(sections "Dual-Stream Memory Layout", "Attention Computation with Cached RoPE") and
"KV Caching Benefits in Ling Bot-Map" (sections "Reduced KV Growth via Keyframe
Streaming": 80 % cut at interval 5; "Dynamic Keyframe Selection": rollback).
"""

import os

import numpy as np
import pytest

from oracle import retention
from rope_paged_kv_02_b200.workloads import CONFIGS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.txt")


def _facts():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if "=" in line:
            k, v = (s.strip() for s in line.split("=", 1))
            out[k] = v
    return out


def _replay(S, W, schedule, max_frames=None):
    r = retention.PagedRetention(S, W, max_frames or max(1, sum(schedule)))
    log = []
    for f, key in enumerate(schedule):
        page, slot = r.append(f, key)
        vis = r.visible()
        ev = r.finish()
        log.append((f, key, page, slot, vis, ev, r.snapshot()))
    return r, log


@pytest.mark.parametrize("S,W,interval,n", [(1, 3, 1, 8), (8, 16, 1, 64), (8, 64, 5, 320),
                                            (0, 4, 1, 20), (3, 0, 2, 15), (0, 0, 1, 5),
                                            (2, 5, 3, 100), (4, 32, 1, 96)])
def test_replay_matches_closed_form(S, W, interval, n):
    sched = retention.keyframe_schedule(n, interval)
    r, log = _replay(S, W, sched)
    committed = []
    for f, key, page, slot, vis, ev, snap in log:
        # the frame's attention saw the retained set as of before it, plus itself
        expect = retention.retained_closed_form(committed, S, W)
        assert snap is not None
        assert len(vis.scale_pages) + len(vis.window_pages) == len(expect)
        if key:
            committed.append(f)
        got = snap["scale_frames"] + snap["window_frames"]
        assert got == retention.retained_closed_form(committed, S, W)
        # conservation and uniqueness of pages
        used = snap["scale_pages"] + snap["window_pages"]
        assert sorted(used + snap["free"]) == list(range(S + W + 1))
        assert snap["n_special"] == 6 * len(committed)
        assert len(vis.patch_pages) <= S + W + 1


def test_non_keyframes_leave_state_unchanged():
    r = retention.PagedRetention(2, 3, 100)
    rng = np.random.default_rng(0)
    for f in range(200):
        key = bool(rng.random() < 0.3)
        before = r.snapshot()
        r.append(f, key)
        r.visible()
        r.finish()
        after = r.snapshot()
        if not key:
            before["last_frame"] = after["last_frame"]
            assert before == after


def test_visible_order_and_last_page_len():
    f = _facts()
    assert f["visible_order"] == "scale,window,special"
    r = retention.PagedRetention(2, 2, 1000)
    for fr in range(60):
        page, slot = r.append(fr, True)
        vis = r.visible()
        assert vis.patch_pages == [p for p, _ in r.scale] + [p for p, _ in r.window] + [page]
        assert slot == 6 * fr
        n_sp = 6 * (fr + 1)
        # brute force: count tokens page by page
        left, pages, last = n_sp, 0, 0
        while left > 0:
            last = min(128, left)
            left -= last
            pages += 1
        assert (vis.n_special, vis.special_pages, vis.last_page_len) == (n_sp, pages, last)
        r.finish()


def test_keyframe_interval_five_stores_twenty_percent():
    f = _facts()
    interval = int(f["keyframe_interval"])
    cut = int(f["kv_storage_cut_percent"])
    cfg2 = CONFIGS[2]
    assert cfg2.keyframe_interval == interval
    r, _ = _replay(cfg2.scale_frames, cfg2.sliding_window, cfg2.keyframes)
    stored = len(r.committed)
    assert stored * 100 == (100 - cut) * cfg2.n_frames          # 64 of 320
    # the API example on the same page: 200 frames, window 64, 8 scale frames
    n = int(f["api_example_frames"])
    r2, _ = _replay(int(f["api_example_scale_frames"]), int(f["api_example_sliding_window"]),
                    retention.keyframe_schedule(n, interval))
    assert len(r2.committed) * 100 == (100 - cut) * n
    assert len(r2.retained_frames()) == len(r2.committed)      # 40 <= 72: nothing evicted


def test_long_stream_final_retained_set():
    cfg3 = CONFIGS[3]
    r, _ = _replay(cfg3.scale_frames, cfg3.sliding_window, cfg3.keyframes)
    assert r.retained_frames() == list(range(8)) + list(range(1872, 2000))
    assert r.n_special == 12000


def test_deferred_eviction_and_lifo_pages():
    # S=1, W=2: P = 4 pages; fresh pops 0,1,2,3; frame 3 overflows the window
    r = retention.PagedRetention(1, 2, 100)
    pages = []
    for f in range(4):
        p, _ = r.append(f, True)
        pages.append(p)
        vis = r.visible()
        ev = r.finish()
        if f < 3:
            assert ev is None
    assert pages == [0, 1, 2, 3]
    assert ev == 1                                  # oldest window page, after frame 3's attention
    assert vis.window_pages == [1, 2]               # frame 3 still saw frame 1
    p, _ = r.append(4, True)
    assert p == 1                                   # LIFO: the evicted page is reused first
    assert r.visible().window_pages == [2, 3]
    r.finish()
    # rollback pushes the page back on top
    p, _ = r.append(5, False)
    r.visible()
    r.finish()
    p2, _ = r.append(6, True)
    assert p2 == p


def test_sequence_and_capacity_errors():
    r = retention.PagedRetention(1, 1, 2)
    with pytest.raises(retention.SequenceError):
        r.visible()
    r.append(0, True)
    with pytest.raises(retention.SequenceError):
        r.append(1, True)
    r.finish()
    with pytest.raises(retention.SequenceError):
        r.append(0, True)
    r.append(3, True)
    r.finish()
    with pytest.raises(retention.CapacityError):
        r.append(4, True)
    r.append(4, False)          # non-keyframes still fit
    r.finish()


@pytest.mark.parametrize("seed", range(6))
def test_decision_after_attention_equals_decision_at_append(seed):
    """"Dynamic Keyframe Selection": keeping or dropping a frame after its attention gives
    the state the same decision taken at append gives, frame by frame, and the retained set
    of the closed form."""
    rng = np.random.default_rng(seed)
    S, W = int(rng.integers(0, 5)), int(rng.integers(0, 7))
    n = int(rng.integers(5, 80))
    sched = [bool(x) for x in rng.random(n) < rng.uniform(0.2, 0.9)]
    up_front = retention.PagedRetention(S, W, max(1, sum(sched)))
    deferred = retention.PagedRetention(S, W, max(1, sum(sched)))
    committed = []
    for f, key in enumerate(sched):
        assert up_front.append(f, key) == deferred.append(f, None)
        assert up_front.visible() == deferred.visible()
        assert up_front.finish() == deferred.finish(keep=key)
        assert up_front.snapshot() == deferred.snapshot()
        if key:
            committed.append(f)
        assert deferred.retained_frames() == retention.retained_closed_form(committed, S, W)


def test_decision_after_attention_errors():
    r = retention.PagedRetention(1, 1, 1)
    r.append(0, None)
    with pytest.raises(retention.SequenceError):
        r.finish()                              # undecided frame needs keep
    r.finish(keep=True)
    r.append(1, False)
    with pytest.raises(retention.SequenceError):
        r.finish(keep=True)                     # decided at append: no second decision
    r.finish()
    r.append(2, None)
    before = r.snapshot()
    with pytest.raises(retention.CapacityError):
        r.finish(keep=True)                     # max_frames = 1 keyframe already kept
    assert r.snapshot() == before               # still pending, unchanged
    r.finish(keep=False)
    assert r.snapshot()["pending"] is None


def test_reset_gives_a_fresh_cache():
    """"Cross-Window Alignment for Long Videos" (clean_kv_cache between windows): after any
    stream, reset() leaves the state of a new cache, and a second window replays exactly as
    on a new cache, frame indices starting again at 0."""
    rng = np.random.default_rng(9)
    for _ in range(10):
        S, W = int(rng.integers(0, 4)), int(rng.integers(0, 6))
        first = [bool(x) for x in rng.random(int(rng.integers(1, 40))) < 0.6]
        second = [bool(x) for x in rng.random(int(rng.integers(1, 40))) < 0.6]
        m = max(1, sum(first), sum(second))
        r = retention.PagedRetention(S, W, m)
        for f, key in enumerate(first):
            r.append(f, key)
            r.finish()
        r.reset()
        fresh = retention.PagedRetention(S, W, m)
        assert r.snapshot() == fresh.snapshot()
        for f, key in enumerate(second):
            assert r.append(f, key) == fresh.append(f, key)
            assert r.visible() == fresh.visible()
            assert r.finish() == fresh.finish()
            assert r.snapshot() == fresh.snapshot()

"""The C ABI on the host (no GPU): symbols, the page manager against the oracle, errors.

The page manager (lbm_pager_*) is the integer state machine the cache drives; it is compared
bit for bit with ``oracle.retention`` over every stream configuration's keyframe schedule
and over random schedules ("How 3D RoPE Positional Encoding Works with the Paged KV Cache in
LingBot-Map", section "Dual-Stream Memory Layout"; "KV Caching Benefits in Ling Bot-Map",
section "Dynamic Keyframe Selection").
"""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import retention
from rope_paged_kv_02_b200 import _lib
from rope_paged_kv_02_b200.build import build
from rope_paged_kv_02_b200.workloads import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "lbm.h")).read()
    return sorted(set(re.findall(r"^LBM_API\s+[\w\s\*]+?\b(lbm_\w+)\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 19
    assert sorted(_lib.SYMBOLS) == names
    for n in names:
        assert hasattr(lib, n), n
    assert _lib.status_string(_lib.LBM_ERR_SEQUENCE) == "call out of sequence"


def _replay_both(S, W, schedule, max_frames):
    pg = _lib.Pager(S, W, max_frames)
    orc = retention.PagedRetention(S, W, max_frames)
    for f, key in enumerate(schedule):
        got = pg.append(f, key)
        exp = orc.append(f, key)
        assert got == exp, (f, got, exp)
        pages, n_sp, last = pg.visible()
        vis = orc.visible()
        assert pages == vis.patch_pages
        assert (n_sp, last) == (vis.n_special, vis.last_page_len)
        ev = pg.finish()
        oev = orc.finish()
        assert ev == (-1 if oev is None else oev)
        st = pg.state()
        snap = orc.snapshot()
        for k in ("scale_pages", "scale_frames", "window_pages", "window_frames"):
            assert st[k] == snap[k], (f, k)
        assert st["free"] == snap["free"]
        assert st["n_special"] == snap["n_special"]
        assert not st["pending"]
    pg.close()


@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_pager_replays_config_schedules_bit_exactly(lib, cfg):
    _replay_both(cfg.scale_frames, cfg.sliding_window, cfg.keyframes, cfg.n_keyframes)


def test_pager_replays_random_schedules_bit_exactly(lib):
    rng = np.random.default_rng(11)
    for _ in range(40):
        S = int(rng.integers(0, 6))
        W = int(rng.integers(0, 9))
        n = int(rng.integers(1, 120))
        sched = list(rng.random(n) < rng.uniform(0.1, 1.0))
        _replay_both(S, W, sched, max(1, sum(sched)))


def test_pager_errors_leave_state_unchanged(lib):
    pg = _lib.Pager(1, 2, 2)
    with pytest.raises(_lib.LbmError) as e:
        pg.visible()
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    with pytest.raises(_lib.LbmError) as e:
        pg.finish()
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    pg.append(0, True)
    before = pg.state()
    with pytest.raises(_lib.LbmError) as e:
        pg.append(1, True)                       # append twice
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    assert pg.state() == before
    pg.finish()
    with pytest.raises(_lib.LbmError) as e:
        pg.append(0, True)                       # frame index must increase
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    pg.append(5, True)
    pg.finish()
    before = pg.state()
    with pytest.raises(_lib.LbmError) as e:
        pg.append(6, True)                       # 2 keyframes committed = max_frames
    assert e.value.status == _lib.LBM_ERR_CAPACITY
    assert pg.state() == before
    pg.append(6, False)                          # a non-keyframe still fits
    pg.finish()
    pg.reset()
    assert pg.state()["free"] == [3, 2, 1, 0]


def test_pager_decisions_after_attention_replay_bit_exactly(lib):
    """Frames appended undecided (LBM_KEYFRAME_DEFERRED), attended, then kept or dropped
    give the page table the oracle gives for the same decisions."""
    rng = np.random.default_rng(5)
    for _ in range(20):
        S, W = int(rng.integers(0, 5)), int(rng.integers(0, 7))
        n = int(rng.integers(1, 90))
        sched = [bool(x) for x in rng.random(n) < rng.uniform(0.1, 1.0)]
        pg = _lib.Pager(S, W, max(1, sum(sched)))
        orc = retention.PagedRetention(S, W, max(1, sum(sched)))
        for f, key in enumerate(sched):
            assert pg.append(f, None) == orc.append(f, None)
            pages, n_sp, last = pg.visible()
            assert pages == orc.visible().patch_pages
            assert pg.finish() == -1                    # attended, still undecided
            st = pg.state()
            assert st["pending"] and st["pending_is_keyframe"] is None
            oev = orc.finish(keep=key)
            assert pg.commit(key) == (-1 if oev is None else oev)
            st, snap = pg.state(), orc.snapshot()
            for k in ("scale_pages", "scale_frames", "window_pages", "window_frames", "free",
                      "n_special"):
                assert st[k] == snap[k], (f, k)
            assert not st["pending"]
        pg.close()


def test_pager_decision_after_attention_errors(lib):
    pg = _lib.Pager(1, 1, 2)
    page, slot = ctypes.c_int(), ctypes.c_int()
    assert lib.lbm_pager_append(pg.handle, 0, 3, ctypes.byref(page),
                                ctypes.byref(slot)) == _lib.LBM_ERR_INVALID  # not 0, 1, 2
    pg.append(0, None)
    with pytest.raises(_lib.LbmError) as e:
        pg.commit(True)                             # not attended yet
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    pg.finish()
    with pytest.raises(_lib.LbmError) as e:
        pg.finish()                                 # attended twice
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    pg.commit(True)
    pg.append(1, True)
    pg.finish()
    with pytest.raises(_lib.LbmError) as e:
        pg.commit(True)                             # decided at append, already settled
    assert e.value.status == _lib.LBM_ERR_SEQUENCE
    pg.append(2, None)
    pg.finish()
    before = pg.state()
    with pytest.raises(_lib.LbmError) as e:
        pg.commit(True)                             # max_frames = 2 keyframes already kept
    assert e.value.status == _lib.LBM_ERR_CAPACITY
    assert pg.state() == before                     # still pending
    pg.commit(False)
    assert not pg.state()["pending"]
    pg.close()


def test_rope_variant_argument_checks_without_gpu(lib):
    h = ctypes.c_void_p()
    for args in [(64, 20, 22, 21), (64, 0, 32, 32), (64, 21, 21, 22),   # odd or empty axes
                 (64, 20, 22, 24), (4, 0, 0, 0), (63, 0, 0, 0)]:       # wrong sum, bad head_dim
        assert lib.lbm_rope3d_tables_fhw(*args, 4, 3, 3, 6, 10000.0, 1.0,
                                         ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    assert lib.lbm_rope3d_tables_fhw(64, 20, 22, 22, 4, 3, 3, 6, 10000.0, 0.0,
                                     ctypes.byref(h)) == _lib.LBM_ERR_INVALID   # ntk <= 0
    assert lib.lbm_rope3d_tables_fhw(64, 20, 22, 22, 4, 3, 3, 6, 1.0, 0.5,
                                     ctypes.byref(h)) == _lib.LBM_ERR_INVALID   # theta*ntk <= 1
    assert lib.lbm_rope3d_tables_fhw(64, 0, 0, 0, 4, 3, 3, 6, 1.0, 0.5,
                                     ctypes.byref(h)) == _lib.LBM_ERR_INVALID   # default split too
    # the 2D variant: head_dim a multiple of 4, frequency > 1
    for hd, freq in [(66, 100.0), (2, 100.0), (64, 1.0), (64, 0.0)]:
        assert lib.lbm_rope2d_tables(hd, 4, 3, 3, 6, freq, ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    assert lib.lbm_rope2d_tables(64, 4, 3, 3, 6, 100.0, None) == _lib.LBM_ERR_INVALID


def test_create_argument_checks_without_gpu(lib):
    h = ctypes.c_void_p()
    # pager: bad sizes
    assert lib.lbm_pager_create(-1, 2, 4, 6, ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    assert lib.lbm_pager_create(600, 600, 4, 6, ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    assert lib.lbm_pager_create(1, 1, 0, 6, ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    # rope tables: odd head_dim / bad theta are rejected before any device call
    assert lib.lbm_rope3d_tables(63, 4, 2, 2, 6, 10000.0, ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    assert lib.lbm_rope3d_tables(64, 4, 2, 2, 6, 0.5, ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    # cache: null rope, null out
    assert lib.lbm_cache_create(2, 64, 16, 6, 1, 3, 8, _lib.LBM_BF16, None,
                                ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    assert lib.lbm_cache_create(2, 64, 16, 6, 1, 3, 8, _lib.LBM_BF16, None,
                                None) == _lib.LBM_ERR_INVALID
    # per-frame calls on a null cache
    assert lib.lbm_append_frame(None, None, None, None, 0, 1, None) == _lib.LBM_ERR_INVALID
    assert lib.lbm_attend_frame(None, None, None, None) == _lib.LBM_ERR_INVALID
    assert lib.lbm_cache_reset(None) == _lib.LBM_ERR_INVALID
    assert lib.lbm_cache_check(None) == _lib.LBM_ERR_INVALID
    assert lib.lbm_commit_frame(None, 1) == _lib.LBM_ERR_INVALID
    assert lib.lbm_cache_set_wait_limit(None, 1000) == _lib.LBM_ERR_INVALID
    # multi-block caches: block count checked first; block calls on a null cache
    for nb in (0, -1, 1025):
        assert lib.lbm_cache_create_blocks(nb, 2, 64, 16, 6, 1, 3, 8, _lib.LBM_BF16, None,
                                           ctypes.byref(h)) == _lib.LBM_ERR_INVALID
    assert lib.lbm_append_frame_block(None, 0, None, None, None, 0, 1,
                                      None) == _lib.LBM_ERR_INVALID
    assert lib.lbm_attend_frame_block(None, 0, None, None, None) == _lib.LBM_ERR_INVALID
    buf = ctypes.create_string_buffer(16)
    assert lib.lbm_cache_read_kv_block(None, 0, 0, 0, 0, buf) == _lib.LBM_ERR_INVALID

"""lbm_attend_frame_noalloc (GPU, through the C ABI).

Some callers cannot allocate device memory once frames are streaming: a serving runtime that
hands every byte of the GPU to its own pool and budget, or a real-time frame loop in which a
cudaMalloc / cudaFree would synchronise the device and stall the stream.  The no-allocation
entry point serves them: it gives the same attention output and the same page-table update
as lbm_attend_frame, but its stream-K partial results go to the library's file-scope device
array instead of memory the cache allocated.

Checked here:
* frame by frame against the regular call on an identical second cache, and against the
  fp64 oracle, with the tolerances of the parity tests, several calls in a row, on frames
  whose keys are split between CTAs (so the array really carries partial results);
* a two-block cache attended block by block through the no-allocation call;
* a frame whose partial results need more than the array holds is refused with
  LBM_ERR_CAPACITY, leaves the cache as it was (state and launch count), and the regular call
  then attends the same frame correctly.

This file is collected last on purpose: a run that stops at the first failure has then
already run every other test.
"""

import ctypes

import numpy as np
import pytest

from rope_paged_kv_02_b200 import _lib
from rope_paged_kv_02_b200.workloads import custom_config, frame_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rope_paged_kv_02_b200.build import build
    build()
    return _lib.load()


def _noalloc(lib, cache, q, out):
    import torch
    stream = torch.cuda.current_stream().cuda_stream
    return lib.lbm_attend_frame_noalloc(cache.handle, ctypes.c_void_p(q.data_ptr()),
                                        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(stream))


def test_noalloc_attend_matches_regular_attend_and_oracle(lib):
    import torch
    from oracle import stream as ostream
    from stream_check import check_attn, dev, host

    # one query tile per head and many key tiles: the planner splits the keys, so the
    # static array really carries the partial results
    cfg = custom_config(300, 2, 64, "bf16", 4, 4, 10, 1, 2, 6)
    ropes = [_lib.Rope3D(64, cfg.n_frames, 4, 4, 6) for _ in range(2)]
    caches = [_lib.PagedKVCache(r, 2, 64, 16, 2, 6, cfg.n_frames, _lib.LBM_BF16) for r in ropes]
    so = ostream.StreamOracle(2, 64, 4, 4, 2, 6, cfg.n_frames)
    split_frames = 0
    for f in range(cfg.n_frames):
        q, k, v = frame_qkv(cfg, f)
        outs = []
        for which, cache in enumerate(caches):
            qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
            out = torch.empty_like(qd)
            cache.append_frame(qd, kd, vd, f, True)
            before = cache.state()["kernel_launches"]
            if which == 0:
                cache.attend_frame(qd, out)
            else:
                st = _noalloc(lib, cache, qd, out)
                assert st == _lib.LBM_OK, _lib.status_string(st)
                if cache.state()["kernel_launches"] - before == 2:
                    split_frames += 1           # attention + combine: the array was used
            outs.append(out)
        r = so.step(f, True, q, k, v)
        torch.cuda.synchronize()
        check_attn(host(outs[1]), host(outs[0]).astype(np.float64), f"frame {f} vs regular")
        check_attn(host(outs[1]), r.out, f"frame {f} vs oracle")
        s0, s1 = caches[0].state(), caches[1].state()
        for key in ("scale_pages", "scale_frames", "window_pages", "window_frames", "free",
                    "n_special"):
            assert s0[key] == s1[key] == r.state[key], (f, key)
    assert split_frames >= 2
    for c in caches:
        c.check()
        c.close()
    for r in ropes:
        r.close()


def test_noalloc_two_block_cache(lib):
    import torch
    from oracle import stream as ostream
    from stream_check import check_attn, dev, host
    nb = 2
    cfgs = [custom_config(301 + b, 2, 64, "bf16", 4, 4, 7, 2, 1, 3) for b in range(nb)]
    rope = _lib.Rope3D(64, 7, 4, 4, 6)
    cache = _lib.PagedKVCache(rope, 2, 64, 16, 1, 3, 7, _lib.LBM_BF16, num_blocks=nb)
    oracles = [ostream.StreamOracle(2, 64, 4, 4, 1, 3, 7) for _ in range(nb)]
    for f in range(7):
        key = cfgs[0].keyframes[f]
        for b in range(nb):
            q, k, v = frame_qkv(cfgs[b], f)
            qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
            out = torch.empty_like(qd)
            cache.append_frame_block(b, qd, kd, vd, f, key)
            st = _noalloc(lib, cache, qd, out)             # attends block b, the next in order
            assert st == _lib.LBM_OK, _lib.status_string(st)
            r = oracles[b].step(f, key, q, k, v)
            torch.cuda.synchronize()
            check_attn(host(out), r.out, f"block {b} frame {f}")
            assert cache.state()["pending"] == (b < nb - 1)
    cache.check()
    cache.close()
    rope.close()


def test_noalloc_refuses_frames_beyond_the_array(lib):
    """48 heads x head_dim 128 on one CTA per SM: (48 units + up to 148 CTAs) x 256 rows x 129
    floats is far above the array's LBM_NOALLOC_SCRATCH_BYTES, so the call must refuse the
    frame before launching anything and leave the cache untouched."""
    import torch
    from oracle import stream as ostream
    from stream_check import check_attn, dev, host
    cfg = custom_config(303, 48, 128, "bf16", 9, 15, 3, 1, 1, 1)
    rope = _lib.Rope3D(128, 3, 9, 15, 6)
    cache = _lib.PagedKVCache(rope, 48, 128, 135, 1, 1, 3, _lib.LBM_BF16)
    so = ostream.StreamOracle(48, 128, 9, 15, 1, 1, 3)
    rows = np.array([0, 5, 6, 70, 140])
    for f in range(3):
        q, k, v = frame_qkv(cfg, f)
        qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
        out = torch.empty_like(qd)
        cache.append_frame(qd, kd, vd, f, True)
        before = cache.state()
        assert _noalloc(lib, cache, qd, out) == _lib.LBM_ERR_CAPACITY
        assert cache.state() == before                    # page table and launch count
        cache.attend_frame(qd, out)                       # the regular call still works
        r = so.step(f, True, q, k, v, rows=rows)
        torch.cuda.synchronize()
        check_attn(host(out)[rows], r.out, f"frame {f} after a refused call")
    cache.check()
    cache.close()
    rope.close()

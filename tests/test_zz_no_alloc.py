"""lbm_attend_frame_noalloc against lbm_attend_frame (GPU, through the C ABI).

The no-allocation entry point exists for callers that may not allocate device memory while
frames stream (a runtime that owns the GPU through its own pool, a real-time loop where
cudaMalloc would synchronise the device).  It must give the same attention output and the
same page-table update as the regular call while taking its stream-K scratch from the
library's file-scope device array.  Two caches receive the identical seeded stream; frame
by frame, one is attended with each entry point (several calls in a row), and the outputs
are compared with the tolerance the parity tests use.  This file is collected last on
purpose.
"""

import ctypes

import numpy as np
import pytest

from rope_paged_kv_02_b200 import _lib
from rope_paged_kv_02_b200.workloads import custom_config, frame_qkv

pytestmark = pytest.mark.gpu


def test_noalloc_attend_matches_regular_attend():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rope_paged_kv_02_b200.build import build
    build()
    lib = _lib.load()
    from stream_check import check_attn, host

    # one query tile per head and many key tiles: the planner splits the keys, so the
    # static scratch really carries the partial results
    cfg = custom_config(300, 2, 64, "bf16", 4, 4, 10, 1, 2, 6)
    ropes = [_lib.Rope3D(64, cfg.n_frames, 4, 4, 6) for _ in range(2)]
    caches = [_lib.PagedKVCache(r, 2, 64, 16, 2, 6, cfg.n_frames, _lib.LBM_BF16) for r in ropes]
    stream = torch.cuda.current_stream().cuda_stream
    split_frames = 0
    for f in range(cfg.n_frames):
        q, k, v = frame_qkv(cfg, f)
        outs = []
        for which, cache in enumerate(caches):
            qd = torch.from_numpy(q).cuda().to(torch.bfloat16)
            kd = torch.from_numpy(k).cuda().to(torch.bfloat16)
            vd = torch.from_numpy(v).cuda().to(torch.bfloat16)
            out = torch.empty_like(qd)
            cache.append_frame(qd, kd, vd, f, True)
            before = cache.state()["kernel_launches"]
            if which == 0:
                cache.attend_frame(qd, out)
            else:
                st = lib.lbm_attend_frame_noalloc(cache.handle, ctypes.c_void_p(qd.data_ptr()),
                                                  ctypes.c_void_p(out.data_ptr()),
                                                  ctypes.c_void_p(stream))
                assert st == _lib.LBM_OK, _lib.status_string(st)
                if cache.state()["kernel_launches"] - before == 2:
                    split_frames += 1           # attention + combine: scratch was used
            outs.append(out)
        torch.cuda.synchronize()
        check_attn(host(outs[1]), host(outs[0]).astype(np.float64), f"frame {f}")
        s0, s1 = caches[0].state(), caches[1].state()
        for key in ("scale_pages", "window_pages", "free", "n_special"):
            assert s0[key] == s1[key]
    assert split_frames >= 2
    for c in caches:
        c.check()
        c.close()
    for r in ropes:
        r.close()

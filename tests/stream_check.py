"""Streams a seeded configuration through the CUDA path and the oracle side by side.

Used by the GPU parity tests, ``__graft_entry__.smoke()`` and ``bench.py``'s correctness
probe.  Inputs come from ``rope_paged_kv_02_b200.workloads`` only; expected values come from
``oracle`` only.  Tolerances (from the arithmetic of each step):

* RoPE, float32 caches: max |gpu - oracle| <= 1e-5.
* RoPE, bf16 caches: |gpu - y| <= 2^-8 |y| + 2e-6 per element, y the fp64 oracle value: the
  kernel rotates in fp32 and rounds once to bf16 (round-to-nearest-even is within half an
  ulp, i.e. 2^-8 |y|); 2e-6 covers the fp32 table and product rounding.
* V written to the pools: bit-exact copies of the inputs.
* Page tables, free lists, retained frames, special counts: bit-exact.
* Attention: relative L2 <= 1e-2 and max |gpu - oracle| <= 3e-2 over the compared rows,
  against fp64.
"""

from __future__ import annotations

import numpy as np

from oracle import stream as ostream
from rope_paged_kv_02_b200 import _lib, workloads

ATTN_REL_L2 = 1e-2
ATTN_MAX_ABS = 3e-2


def dev(x: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def host(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy()


def pool_values(raw: np.ndarray, dtype: str) -> np.ndarray:
    return workloads.bits_to_f32(raw) if dtype == "bf16" else raw


def check_rope(got: np.ndarray, exact: np.ndarray, dtype: str, what: str) -> float:
    err = np.abs(got.astype(np.float64) - exact)
    if dtype == "f32":
        bound = np.full_like(err, 1e-5)
    else:
        bound = 2.0 ** -8 * np.abs(exact) + 2e-6
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements out of bound, "
                           f"worst {float((err - bound).max()):.3e}")
    return float(err.max())


def attn_errors(got: np.ndarray, exact: np.ndarray) -> tuple[float, float]:
    d = got.astype(np.float64) - exact
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(exact), 1e-300))
    return rel, float(np.abs(d).max())


def check_attn(got: np.ndarray, exact: np.ndarray, what: str) -> tuple[float, float]:
    rel, mx = attn_errors(got, exact)
    assert rel <= ATTN_REL_L2 and mx <= ATTN_MAX_ABS, f"{what}: rel-L2 {rel:.3e}, max {mx:.3e}"
    return rel, mx


def make_cache(cfg: workloads.StreamConfig, max_frame_idx: int | None = None, split=None,
               ntk_factor: float = 1.0, rope2d_frequency: float | None = None):
    ppf = (max_frame_idx + 1) if max_frame_idx is not None else cfg.n_frames
    if rope2d_frequency is not None:
        rope = _lib.Rope2D(cfg.head_dim, ppf, cfg.pph, cfg.ppw, 6, frequency=rope2d_frequency)
    else:
        rope = _lib.Rope3D(cfg.head_dim, ppf, cfg.pph, cfg.ppw, 6, split=split,
                           ntk_factor=ntk_factor)
    cache = _lib.PagedKVCache(rope, cfg.heads, cfg.head_dim, cfg.patches, cfg.scale_frames,
                              cfg.sliding_window, max(1, cfg.n_keyframes),
                              _lib.LBM_BF16 if cfg.dtype == "bf16" else _lib.LBM_F32)
    return rope, cache


def regen_source(cfg: workloads.StreamConfig, frame_ids: list):
    """kv_source for the oracle: re-creates a past frame's inputs from its seed."""
    index = {fid: n for n, fid in enumerate(frame_ids)}

    def source(frame, region):
        n = index[frame]
        if region == "special":
            return (workloads.frame_specials(cfg, n, 1), workloads.frame_specials(cfg, n, 2))
        k = workloads.frame_tensor(cfg, n, 1)[6:]
        v = workloads.frame_tensor(cfg, n, 2)[6:]
        return k, v

    return source


def run_stream(cfg: workloads.StreamConfig, check_frames=None, rows=None, frame_ids=None,
               tamper=None, check_pools=True, regenerate=False, report=None, decide_after=False,
               split=None, ntk_factor: float = 1.0, reset_at=(),
               rope2d_frequency: float | None = None, fold_q: bool | None = None):
    """Streams every frame of cfg through the cache; checks the frames in check_frames.

    split, ntk_factor: RoPE variant (explicit (t, h, w) split, NTK factor), for both sides.
    rope2d_frequency: rotate with the 2D (y, x) variant of that base frequency instead.
    fold_q: append with q = None, so the attention kernel rotates q as it loads it (it also
    writes the rotated q it used, which is checked like the in-place rotation; bf16 only).
    Default False: the append rotates q in place, as bench.py streams.
    reset_at: stream positions before which cache and oracle are reset (windowed streaming;
    frame_ids may then start again).
    decide_after: append every frame undecided and keep / drop it after its attention
    (lbm_commit_frame) by the schedule; the oracle takes the same decision at append.

    frame_ids: absolute frame index of each streamed frame (default 0..n-1).
    tamper(n, q, k, v) -> (q, k, v): changes the seeded inputs of frame n (stress tests).
    rows: query rows compared at checked frames (default: all).
    Returns a list of per-checked-frame error summaries.
    """
    import torch
    frame_ids = list(range(cfg.n_frames)) if frame_ids is None else list(frame_ids)
    check = set(range(cfg.n_frames)) if check_frames is None else set(check_frames)
    rope, cache = make_cache(cfg, max(frame_ids), split, ntk_factor, rope2d_frequency)
    so = ostream.StreamOracle(cfg.heads, cfg.head_dim, cfg.pph, cfg.ppw, cfg.scale_frames,
                              cfg.sliding_window, max(1, cfg.n_keyframes),
                              kv_source=regen_source(cfg, frame_ids) if regenerate else None,
                              split=split, ntk_factor=ntk_factor,
                              rope2d_frequency=rope2d_frequency)
    fold_q = bool(fold_q)
    summary = []
    T = cfg.tokens
    keys = cfg.keyframes
    for n, fid in enumerate(frame_ids):
        if n in reset_at:
            cache.reset()
            so.reset()
        q, k, v = workloads.frame_qkv(cfg, n)
        if tamper is not None:
            q, k, v = tamper(n, q, k, v)
        qd, kd, vd = dev(q, cfg.dtype), dev(k, cfg.dtype), dev(v, cfg.dtype)
        out = torch.empty_like(qd)
        q_rot = torch.empty_like(qd) if fold_q else None
        cache.append_frame(None if fold_q else qd, kd, vd, fid, None if decide_after else keys[n])
        cache.attend_frame(qd, out, q_rot_out=q_rot)
        if decide_after:
            st = cache.state()
            assert st["pending"] and st["pending_is_keyframe"] is None, fid
            cache.commit_frame(keys[n])
        checking = n in check
        r = so.step(fid, keys[n], q, k, v, rows=rows if checking else [], attend=checking)
        if not checking:
            continue
        torch.cuda.synchronize()
        st = cache.state()
        for key in ("scale_pages", "scale_frames", "window_pages", "window_frames", "free",
                    "n_special"):
            assert st[key] == r.state[key], (fid, key, st[key], r.state[key])
        if fold_q:
            # the raw q is left as it was; the rotated q is what the attention kernel used
            np.testing.assert_array_equal(host(qd), q)
            q_err = check_rope(host(q_rot), r.q_rot, cfg.dtype, f"frame {fid} q (in attention)")
        else:
            q_err = check_rope(host(qd), r.q_rot, cfg.dtype, f"frame {fid} q")
        o = host(out)[r.rows]
        rel, mx = check_attn(o, r.out, f"frame {fid} attention")
        item = {"frame": fid, "q_err": q_err, "attn_rel_l2": rel, "attn_max_abs": mx}
        if check_pools:
            kp = pool_values(cache.read_kv(_lib.LBM_K_PATCH, r.page), cfg.dtype)
            vp = pool_values(cache.read_kv(_lib.LBM_V_PATCH, r.page), cfg.dtype)
            ks = pool_values(cache.read_kv(_lib.LBM_K_SPECIAL, r.special_slot, 6), cfg.dtype)
            vs = pool_values(cache.read_kv(_lib.LBM_V_SPECIAL, r.special_slot, 6), cfg.dtype)
            item["k_err"] = check_rope(kp.transpose(1, 0, 2), r.k_rot[6:], cfg.dtype,
                                       f"frame {fid} K page")
            check_rope(ks.transpose(1, 0, 2), r.k_rot[:6], cfg.dtype, f"frame {fid} K special")
            np.testing.assert_array_equal(vp.transpose(1, 0, 2), v[6:])
            np.testing.assert_array_equal(vs.transpose(1, 0, 2), v[:6])
        summary.append(item)
        if report is not None:
            report(item)
    cache.check()
    cache.close()
    rope.close()
    return summary

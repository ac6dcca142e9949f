"""ctypes binding of liblbm.so: argument marshalling only.

Every function of ``include/lbm.h`` is bound under its own name.  The classes below hold a
handle and turn torch tensors into (device pointer, current stream) pairs; no step of the
streaming-frame computation runs in Python.  If the library is missing this module raises:
there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblbm.so")

LBM_OK = 0
LBM_ERR_INVALID = -1
LBM_ERR_UNSUPPORTED = -2
LBM_ERR_SEQUENCE = -3
LBM_ERR_CAPACITY = -4
LBM_ERR_NOMEM = -5
LBM_ERR_CUDA = -6
LBM_ERR_TIMEOUT = -7
LBM_F32 = 0
LBM_BF16 = 1
LBM_K_PATCH, LBM_V_PATCH, LBM_K_SPECIAL, LBM_V_SPECIAL = 0, 1, 2, 3
LBM_SPECIAL_PAGE = 128
LBM_MAX_PAGES = 1024

# every symbol include/lbm.h declares
SYMBOLS = [
    "lbm_rope3d_tables", "lbm_rope3d_tables_fhw", "lbm_rope2d_tables", "lbm_rope3d_expand",
    "lbm_rope_destroy",
    "lbm_cache_create", "lbm_cache_create_blocks", "lbm_append_frame", "lbm_append_frame_block",
    "lbm_attend_frame", "lbm_attend_frame_block", "lbm_attend_frame_qrot",
    "lbm_attend_frame_noalloc",
    "lbm_commit_frame", "lbm_cache_reset", "lbm_cache_read_kv_block",
    "lbm_cache_set_wait_limit",
    "lbm_cache_state", "lbm_cache_read_kv", "lbm_cache_check", "lbm_cache_destroy",
    "lbm_status_string",
    "lbm_pager_create", "lbm_pager_append", "lbm_pager_visible", "lbm_pager_finish",
    "lbm_pager_commit", "lbm_pager_reset", "lbm_pager_state", "lbm_pager_destroy",
]


LBM_KEYFRAME_DEFERRED = 2


def _keyframe_mode(is_keyframe) -> int:
    """True -> 1, False -> 0, None -> LBM_KEYFRAME_DEFERRED (decided after attention)."""
    if is_keyframe is None:
        return LBM_KEYFRAME_DEFERRED
    return 1 if is_keyframe else 0


class LbmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class CacheState(ctypes.Structure):
    _fields_ = [
        ("num_pages", ctypes.c_int), ("n_scale", ctypes.c_int), ("n_window", ctypes.c_int),
        ("n_free", ctypes.c_int), ("n_special", ctypes.c_int), ("special_pages", ctypes.c_int),
        ("last_page_len", ctypes.c_int), ("pending", ctypes.c_int),
        ("pending_page", ctypes.c_int), ("pending_is_keyframe", ctypes.c_int),
        ("pending_frame", ctypes.c_longlong), ("last_frame", ctypes.c_longlong),
        ("device_bytes", ctypes.c_longlong), ("kernel_launches", ctypes.c_longlong),
        ("capacity", ctypes.c_int),
        ("scale_pages", ctypes.POINTER(ctypes.c_int)),
        ("scale_frames", ctypes.POINTER(ctypes.c_longlong)),
        ("window_pages", ctypes.POINTER(ctypes.c_int)),
        ("window_frames", ctypes.POINTER(ctypes.c_longlong)),
        ("free_pages", ctypes.POINTER(ctypes.c_int)),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """The library, loaded once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m rope_paged_kv_02_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    c_int, c_ll, c_void, c_d = ctypes.c_int, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_double
    pint = ctypes.POINTER(c_int)
    lib.lbm_rope3d_tables.argtypes = [c_int] * 5 + [c_d, ctypes.POINTER(c_void)]
    lib.lbm_rope3d_tables_fhw.argtypes = [c_int] * 8 + [c_d, c_d, ctypes.POINTER(c_void)]
    lib.lbm_rope2d_tables.argtypes = [c_int] * 5 + [c_d, ctypes.POINTER(c_void)]
    lib.lbm_rope3d_expand.argtypes = [c_void, c_void, c_void, c_void]
    lib.lbm_rope_destroy.argtypes = [c_void]
    lib.lbm_rope_destroy.restype = None
    lib.lbm_cache_create.argtypes = [c_int] * 8 + [c_void, ctypes.POINTER(c_void)]
    lib.lbm_cache_create_blocks.argtypes = [c_int] * 9 + [c_void, ctypes.POINTER(c_void)]
    lib.lbm_append_frame_block.argtypes = [c_void, c_int, c_void, c_void, c_void, c_ll, c_int,
                                           c_void]
    lib.lbm_attend_frame_block.argtypes = [c_void, c_int, c_void, c_void, c_void]
    lib.lbm_cache_read_kv_block.argtypes = [c_void, c_int, c_int, c_int, c_int, c_void]
    lib.lbm_append_frame.argtypes = [c_void, c_void, c_void, c_void, c_ll, c_int, c_void]
    lib.lbm_attend_frame.argtypes = [c_void, c_void, c_void, c_void]
    lib.lbm_attend_frame_noalloc.argtypes = [c_void, c_void, c_void, c_void]
    lib.lbm_attend_frame_qrot.argtypes = [c_void, c_void, c_void, c_void, c_void]
    lib.lbm_commit_frame.argtypes = [c_void, c_int]
    lib.lbm_cache_reset.argtypes = [c_void]
    lib.lbm_cache_state.argtypes = [c_void, ctypes.POINTER(CacheState)]
    lib.lbm_cache_read_kv.argtypes = [c_void, c_int, c_int, c_int, c_void]
    lib.lbm_cache_check.argtypes = [c_void]
    lib.lbm_cache_set_wait_limit.argtypes = [c_void, ctypes.c_ulonglong]
    lib.lbm_cache_destroy.argtypes = [c_void]
    lib.lbm_cache_destroy.restype = None
    lib.lbm_status_string.argtypes = [c_int]
    lib.lbm_status_string.restype = ctypes.c_char_p
    lib.lbm_pager_create.argtypes = [c_int] * 4 + [ctypes.POINTER(c_void)]
    lib.lbm_pager_append.argtypes = [c_void, c_ll, c_int, pint, pint]
    lib.lbm_pager_visible.argtypes = [c_void, pint, c_int, pint, pint, pint]
    lib.lbm_pager_finish.argtypes = [c_void, pint]
    lib.lbm_pager_commit.argtypes = [c_void, c_int, pint]
    lib.lbm_pager_reset.argtypes = [c_void]
    lib.lbm_pager_state.argtypes = [c_void, ctypes.POINTER(CacheState)]
    lib.lbm_pager_destroy.argtypes = [c_void]
    lib.lbm_pager_destroy.restype = None
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().lbm_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != LBM_OK:
        raise LbmError(status, where)


def _ptr(x) -> int:
    """Device address of a torch tensor (or an int address passed through)."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _state_dict(fill, capacity: int) -> dict:
    st = CacheState()
    st.capacity = capacity
    sp = (ctypes.c_int * capacity)()
    sf = (ctypes.c_longlong * capacity)()
    wp = (ctypes.c_int * capacity)()
    wf = (ctypes.c_longlong * capacity)()
    fp = (ctypes.c_int * capacity)()
    st.scale_pages, st.scale_frames = sp, sf
    st.window_pages, st.window_frames = wp, wf
    st.free_pages = fp
    _check(fill(ctypes.byref(st)), "state")
    return {
        "num_pages": st.num_pages,
        "scale_pages": list(sp[:st.n_scale]), "scale_frames": list(sf[:st.n_scale]),
        "window_pages": list(wp[:st.n_window]), "window_frames": list(wf[:st.n_window]),
        "free": list(fp[:st.n_free]),
        "n_special": st.n_special, "special_pages": st.special_pages,
        "last_page_len": st.last_page_len, "pending": bool(st.pending),
        "pending_page": st.pending_page,
        "pending_is_keyframe": (None if st.pending_is_keyframe == LBM_KEYFRAME_DEFERRED
                                else bool(st.pending_is_keyframe)),
        "pending_frame": st.pending_frame, "last_frame": st.last_frame,
        "device_bytes": st.device_bytes, "kernel_launches": st.kernel_launches,
    }


class Rope3D:
    """lbm_rope3d_tables: the per-axis cos/sin tables (device), built once."""

    def __init__(self, head_dim: int, ppf: int, pph: int, ppw: int, patch_start_idx: int = 6,
                 theta: float = 10000.0, split=None, ntk_factor: float = 1.0):
        """split: explicit (d_t, d_h, d_w) summing to head_dim (lbm_rope3d_tables_fhw);
        None leaves the split to the library's default."""
        lib = load()
        h = ctypes.c_void_p()
        if split is None and ntk_factor == 1.0:
            _check(lib.lbm_rope3d_tables(head_dim, ppf, pph, ppw, patch_start_idx, theta,
                                         ctypes.byref(h)), "lbm_rope3d_tables")
        else:
            d_t, d_h, d_w = (0, 0, 0) if split is None else (int(x) for x in split)
            _check(lib.lbm_rope3d_tables_fhw(head_dim, d_t, d_h, d_w, ppf, pph, ppw,
                                             patch_start_idx, theta, float(ntk_factor),
                                             ctypes.byref(h)), "lbm_rope3d_tables_fhw")
        self.handle = h
        self.head_dim, self.ppf, self.pph, self.ppw = head_dim, ppf, pph, ppw
        self.patch_start_idx = patch_start_idx

    def expand(self, cos_out, sin_out, stream=None) -> None:
        """lbm_rope3d_expand into float32 device tensors [ppf*(psi+pph*ppw), head_dim/2]."""
        _check(load().lbm_rope3d_expand(self.handle, _ptr(cos_out), _ptr(sin_out),
                                        _stream(stream)), "lbm_rope3d_expand")

    def close(self) -> None:
        if self.handle:
            load().lbm_rope_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Rope2D(Rope3D):
    """lbm_rope2d_tables: the 2D (y, x) variant's tables (device), built once; used like
    Rope3D by caches."""

    def __init__(self, head_dim: int, ppf: int, pph: int, ppw: int, patch_start_idx: int = 6,
                 frequency: float = 100.0):
        h = ctypes.c_void_p()
        _check(load().lbm_rope2d_tables(head_dim, ppf, pph, ppw, patch_start_idx,
                                        float(frequency), ctypes.byref(h)), "lbm_rope2d_tables")
        self.handle = h
        self.head_dim, self.ppf, self.pph, self.ppw = head_dim, ppf, pph, ppw
        self.patch_start_idx = patch_start_idx


class PagedKVCache:
    """lbm_cache_*: the dual-stream paged KV cache of one layer, or of num_blocks layers
    sharing one page table, on the current device."""

    def __init__(self, rope: Rope3D, heads: int, head_dim: int, patches_per_frame: int,
                 scale_frames: int, sliding_window: int, max_frames: int, dtype: int,
                 specials_per_frame: int = 6, num_blocks: int = 1):
        lib = load()
        h = ctypes.c_void_p()
        if num_blocks == 1:
            _check(lib.lbm_cache_create(heads, head_dim, patches_per_frame, specials_per_frame,
                                        scale_frames, sliding_window, max_frames, dtype,
                                        rope.handle, ctypes.byref(h)), "lbm_cache_create")
        else:
            _check(lib.lbm_cache_create_blocks(num_blocks, heads, head_dim, patches_per_frame,
                                               specials_per_frame, scale_frames, sliding_window,
                                               max_frames, dtype, rope.handle, ctypes.byref(h)),
                   "lbm_cache_create_blocks")
        self.num_blocks = num_blocks
        self.handle = h
        self.rope = rope                      # the tables must outlive the cache
        self.heads, self.head_dim = heads, head_dim
        self.patches, self.psi = patches_per_frame, specials_per_frame
        self.dtype = dtype
        self.num_pages = scale_frames + sliding_window + 1

    @property
    def tokens(self) -> int:
        return self.psi + self.patches

    def append_frame(self, q, k, v, frame_idx: int, is_keyframe, stream=None) -> None:
        """is_keyframe: True / False, or None to decide after attention (commit_frame).
        q: rotated in place here, or None to leave its rotation to attend_frame."""
        _check(load().lbm_append_frame(self.handle, _ptr(q), _ptr(k), _ptr(v), int(frame_idx),
                                       _keyframe_mode(is_keyframe), _stream(stream)),
               "lbm_append_frame")

    def append_frame_block(self, block: int, q, k, v, frame_idx: int, is_keyframe,
                           stream=None) -> None:
        _check(load().lbm_append_frame_block(self.handle, int(block), _ptr(q), _ptr(k), _ptr(v),
                                             int(frame_idx), _keyframe_mode(is_keyframe),
                                             _stream(stream)), "lbm_append_frame_block")

    def attend_frame_block(self, block: int, q, out, stream=None) -> None:
        _check(load().lbm_attend_frame_block(self.handle, int(block), _ptr(q), _ptr(out),
                                             _stream(stream)), "lbm_attend_frame_block")

    def commit_frame(self, keep: bool) -> None:
        _check(load().lbm_commit_frame(self.handle, 1 if keep else 0), "lbm_commit_frame")

    def attend_frame(self, q, out, stream=None, q_rot_out=None) -> None:
        """q_rot_out: also receive the rotated q the kernel used (frames appended with
        q = None only; lbm_attend_frame_qrot)."""
        if q_rot_out is None:
            _check(load().lbm_attend_frame(self.handle, _ptr(q), _ptr(out), _stream(stream)),
                   "lbm_attend_frame")
        else:
            _check(load().lbm_attend_frame_qrot(self.handle, _ptr(q), _ptr(out), _ptr(q_rot_out),
                                                _stream(stream)), "lbm_attend_frame_qrot")

    def reset(self) -> None:
        _check(load().lbm_cache_reset(self.handle), "lbm_cache_reset")

    def state(self) -> dict:
        return _state_dict(lambda p: load().lbm_cache_state(self.handle, p),
                           max(self.num_pages, 1))

    def read_kv(self, which: int, index: int, count: int = 0, block: int = 0) -> np.ndarray:
        """Pool contents on the host: [heads, patches or count, head_dim], raw dtype."""
        rows = self.patches if which in (LBM_K_PATCH, LBM_V_PATCH) else count
        dt = np.uint16 if self.dtype == LBM_BF16 else np.float32
        out = np.empty((self.heads, rows, self.head_dim), dtype=dt)
        _check(load().lbm_cache_read_kv_block(self.handle, int(block), which, index, count,
                                              out.ctypes.data_as(ctypes.c_void_p)),
               "lbm_cache_read_kv_block")
        return out

    def check(self) -> None:
        _check(load().lbm_cache_check(self.handle), "lbm_cache_check")

    def set_wait_limit(self, ns: int) -> None:
        """lbm_cache_set_wait_limit: bound of each wait of the attention kernel's roles
        (0: the default, 2 s)."""
        _check(load().lbm_cache_set_wait_limit(self.handle, int(ns)), "lbm_cache_set_wait_limit")

    def close(self) -> None:
        if self.handle:
            load().lbm_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Pager:
    """lbm_pager_*: the host-only page manager (no GPU needed)."""

    def __init__(self, scale_frames: int, sliding_window: int, max_frames: int,
                 specials_per_frame: int = 6):
        h = ctypes.c_void_p()
        _check(load().lbm_pager_create(scale_frames, sliding_window, max_frames,
                                       specials_per_frame, ctypes.byref(h)), "lbm_pager_create")
        self.handle = h
        self.num_pages = scale_frames + sliding_window + 1

    def append(self, frame_idx: int, is_keyframe) -> tuple[int, int]:
        page, slot = ctypes.c_int(), ctypes.c_int()
        _check(load().lbm_pager_append(self.handle, int(frame_idx), _keyframe_mode(is_keyframe),
                                       ctypes.byref(page), ctypes.byref(slot)),
               "lbm_pager_append")
        return page.value, slot.value

    def commit(self, keep: bool) -> int:
        ev = ctypes.c_int()
        _check(load().lbm_pager_commit(self.handle, 1 if keep else 0, ctypes.byref(ev)),
               "lbm_pager_commit")
        return ev.value

    def visible(self) -> tuple[list, int, int]:
        cap = self.num_pages
        pages = (ctypes.c_int * cap)()
        n, n_sp, last = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        _check(load().lbm_pager_visible(self.handle, pages, cap, ctypes.byref(n),
                                        ctypes.byref(n_sp), ctypes.byref(last)),
               "lbm_pager_visible")
        return list(pages[:n.value]), n_sp.value, last.value

    def finish(self) -> int:
        ev = ctypes.c_int()
        _check(load().lbm_pager_finish(self.handle, ctypes.byref(ev)), "lbm_pager_finish")
        return ev.value

    def reset(self) -> None:
        _check(load().lbm_pager_reset(self.handle), "lbm_pager_reset")

    def state(self) -> dict:
        return _state_dict(lambda p: load().lbm_pager_state(self.handle, p), self.num_pages)

    def close(self) -> None:
        if self.handle:
            load().lbm_pager_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

"""B200-native streaming-frame step: 3D RoPE + dual-stream paged KV cache + paged attention.

The computation lives in ``liblbm.so`` (hand-written CUDA for sm_100a behind the C ABI of
``include/lbm.h``); ``_lib`` binds it with ctypes, ``workloads`` holds the seeded synthetic
stream configurations.  Build the library with ``python -m rope_paged_kv_02_b200.build``.
"""

from ._lib import (  # noqa: F401
    LBM_BF16, LBM_F32, LBM_K_PATCH, LBM_K_SPECIAL, LBM_V_PATCH, LBM_V_SPECIAL, LbmError,
    PagedKVCache, Pager, Rope3D, load, status_string,
)

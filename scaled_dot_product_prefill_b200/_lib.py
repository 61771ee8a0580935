"""ctypes loader for libattn_b200.so.  Fails loudly: there is no fallback path."""
from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn_b200.so")
_lib = None

ATTN_STATUS = {
    0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_CUDA",
    4: "ATTN_ERR_TIMEOUT", 5: "ATTN_ERR_BAD_PAGE", 6: "ATTN_ERR_WORKSPACE", 7: "ATTN_ERR_OUT_OF_PAGES",
}

# name -> (restype, argtypes); mirrors include/attn_b200.h
_c_int, _c_float, _c_size, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
PROTOTYPES = {
    "attn_status_string": (ctypes.c_char_p, [_c_int]),
    "attn_version": (_c_int, []),
    "attn_prefill": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 6 + [_c_float, _c_int, _c_int, _vp]),
    "attn_prefill_f32": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 6 + [_c_float, _c_int, _c_int, _vp]),
    "attn_prefill_lse": (_c_int, [_vp] * 5 + [_c_int] * 6 + [_c_float, _c_int, _c_int, _vp]),
    "attn_prefill_f32_lse": (_c_int, [_vp] * 5 + [_c_int] * 6 + [_c_float, _c_int, _c_int, _vp]),
    "attn_prefill_paged": (_c_int, [_vp] * 5 + [_c_int] * 9 + [_c_float, _c_int, _c_int, _vp, _vp, _vp]),
    "attn_prefill_host": (_c_int, [_vp] * 8 + [_c_int] * 6 + [_c_float, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "attn_decode_paged": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 8 + [_c_float, _c_int, _vp, _c_size,
                                                                          _vp, _vp]),
    "attn_decode_paged_fp8": (_c_int, [_vp] * 5 + [_c_int] * 8 + [_c_float] * 3 + [_c_int, _vp, _c_size, _vp, _vp]),
    "attn_decode_step_host": (_c_int, [_vp] * 12 + [_c_int] * 8 + [_c_float, _c_int, _vp, _c_size, _vp]),
    "attn_decode_paged_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 8 + [_c_float, _c_int, _vp, _vp]),
    "attn_decode_paged_workspace_size": (_c_size, [_c_int] * 5),
    "attn_device_status": (_c_int, [_c_int]),
    "attn_selftest_wait_timeout": (_c_int, [_c_int, _vp]),
    "attn_kv_append": (_c_int, [_vp] * 6 + [_c_int] * 7 + [_vp]),
    "attn_kv_append_fp8": (_c_int, [_vp] * 6 + [_c_int] * 7 + [_c_float, _c_float, _vp]),
    "attn_page_pool_create": (_c_int, [_c_int] * 4 + [ctypes.POINTER(_vp)]),
    "attn_page_pool_destroy": (None, [_vp]),
    "attn_page_pool_resize": (_c_int, [_vp, _c_int, _c_int]),
    "attn_page_pool_release": (_c_int, [_vp, _c_int]),
    "attn_page_pool_free_pages": (_c_int, [_vp]),
    "attn_page_pool_seq_len": (_c_int, [_vp, _c_int]),
    "attn_page_pool_export": (_c_int, [_vp, _vp, _vp]),
    "attn_page_pool_upload": (_c_int, [_vp, _vp, _vp, _vp]),
}


class AttnError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} returned {ATTN_STATUS.get(status, status)}")


def lib_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load the shared library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m scaled_dot_product_prefill_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib

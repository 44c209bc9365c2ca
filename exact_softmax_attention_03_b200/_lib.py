"""ctypes loader for the C ABI in include/attn.h (libattn.so, built in-tree)."""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# ATTN_LIBRARY=debug selects the bounds-checking debug build (libattn_debug.so,
# see attn_debug_checks in include/attn.h); the default is the release build.
LIB_NAMES = {"release": "libattn.so", "debug": "libattn_debug.so"}
VARIANT = os.environ.get("ATTN_LIBRARY", "release")
if VARIANT not in LIB_NAMES:
    raise RuntimeError(f"ATTN_LIBRARY={VARIANT!r}: expected one of {sorted(LIB_NAMES)}")
LIB_PATH = os.path.join(_HERE, LIB_NAMES[VARIANT])

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4
ATTN_ERR_WORKSPACE = 5
ATTN_ERR_INTERNAL = 6

# Size of the fixed device scratch behind attn_decode_noalloc (include/attn.h).
ATTN_DECODE_NOALLOC_SCRATCH_BYTES = 8 << 20

STATUS_NAMES = {
    ATTN_OK: "ATTN_OK",
    ATTN_ERR_INVALID_ARG: "ATTN_ERR_INVALID_ARG",
    ATTN_ERR_UNSUPPORTED: "ATTN_ERR_UNSUPPORTED",
    ATTN_ERR_CUDA: "ATTN_ERR_CUDA",
    ATTN_ERR_TIMEOUT: "ATTN_ERR_TIMEOUT",
    ATTN_ERR_WORKSPACE: "ATTN_ERR_WORKSPACE",
    ATTN_ERR_INTERNAL: "ATTN_ERR_INTERNAL",
}

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

# name -> (restype, argtypes); mirrors include/attn.h
SIGNATURES = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_f32o": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                             _f, _i, _i, _vp]),
    "attn_bwd_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i]),
    "attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i,
                      _i, _vp, ctypes.c_size_t, _vp]),
    "attn_merge": (_i, [_vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _vp]),
    "attn_decode_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i, _i]),
    "attn_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _vp,
                         ctypes.c_size_t, _vp]),
    "attn_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i,
                                 _vp]),
    "attn_decode_paged": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                               _f, _i, _i, _vp, ctypes.c_size_t, _vp]),
    "attn_last_error": (ctypes.c_char_p, []),
    "attn_device_status": (_i, [_vp]),
    "attn_selftest_wait_timeout": (_i, [_vp]),
    "attn_launch_count": (ctypes.c_ulonglong, []),
    "attn_debug_checks": (_i, []),
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {message}")
        self.code = code


def load() -> ctypes.CDLL:
    """Load libattn.so; raise if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m exact_softmax_attention_03_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(code: int) -> None:
    if code != ATTN_OK:
        msg = load().attn_last_error()
        raise AttnError(code, msg.decode() if msg else "")

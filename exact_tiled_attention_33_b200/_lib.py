"""ctypes loader for libfattn.so (the C ABI declared in include/fattn.h).

The library is loaded from this package directory only.  There is no fallback: if the
shared object is missing or cannot be loaded, every attention call raises.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfattn.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_TIMEOUT = 4
FA_BF16 = 0
FA_FP16 = 1

# Every entry point the header declares, with its ctypes signature.
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "fa_varlen_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _i, _i,
                           _i, _vp]),
    "fa_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "fa_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz,
                    _i, _vp]),
    "fa_varlen_bwd_workspace_size": (_sz, [_i, _i, _i]),
    "fa_varlen_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                           _f, _i, _i, _i, _i, _vp, _sz, _i, _vp]),
    "fa_bwd_deterministic": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                  _f, _i, _i, _vp, _sz, _i, _vp]),
    "fa_varlen_bwd_deterministic": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                         _i, _i, _i, _i, _f, _i, _i, _i, _i, _i, _vp, _sz, _i,
                                         _vp]),
    "fa_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i,
                            _i, _vp]),
    "fa_fwd_local": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _i, _vp]),
    "fa_varlen_fwd_local": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i,
                                 _i, _i, _i, _i, _vp]),
    "fa_bwd_local": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i,
                          _i, _vp, _sz, _i, _vp]),
    "fa_varlen_bwd_local": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i,
                                 _i, _i, _f, _i, _i, _i, _i, _i, _vp, _sz, _i, _vp]),
    "fa_fwd_fp8": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _f, _f, _f, _i, _i, _vp]),
    "fa_varlen_fwd_fp8": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _f, _f, _f,
                               _i, _i, _i, _i, _i, _vp]),
    "fa_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "fa_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz, _i,
                       _vp]),
    "fa_decode_paged": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                             _f, _i, _vp, _sz, _i, _vp]),
    "fa_get_device_status": (_i, [_vp]),
    "fa_status_string": (ctypes.c_char_p, [_i]),
    "fa_last_error": (ctypes.c_char_p, []),
    "fa_selftest_wait_timeout": (_i, [ctypes.c_uint, _vp]),
    "fa_selftest_exp2": (_i, [_vp, _vp, _i, _vp]),
    "fa_selftest_fwd_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _i, _vp]),
}

_LIB = None


class FattnError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


def load():
    """Load libfattn.so and bind every declared entry point (raises if unavailable)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libfattn.so not found at {LIB_PATH}; build it with "
                          "`python -m exact_tiled_attention_33_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def check(status: int, where: str) -> None:
    if status != FA_OK:
        lib = load()
        detail = lib.fa_last_error().decode() or lib.fa_status_string(status).decode()
        raise FattnError(status, where, detail)

"""ctypes view of the C ABI declared in ``include/la.h``.

Loads the in-tree ``liblcl_b200.so``; there is no fallback: if the library
has not been built the import fails with an explanation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblcl_b200.so")

LA_OK = 0
LA_ERR_INVALID_ARG = 1
LA_ERR_UNSUPPORTED = 2
LA_ERR_CUDA = 3
LA_ERR_TIMEOUT = 4
LA_BF16 = 0
LA_FP32 = 1
LA_STATE_FP32 = 0
LA_STATE_BF16 = 1
LA_STATE_FP16 = 2
LA_STATE_FP8_E4M3 = 3
LA_STATE_FP8_E5M2 = 4
LA_PHI_IDENTITY = 0
LA_PHI_ELU1 = 1
LA_PHI_RELU = 2

# name -> (restype, argtypes), mirroring include/la.h
_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
SIGNATURES = {
    "la_status_string": (ctypes.c_char_p, [_i]),
    "la_last_error": (ctypes.c_char_p, []),
    "la_version": (_i, []),
    "la_prefill_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "la_prefill_workspace_size_ex": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "la_prefill_varlen_workspace_size_ex": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "la_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "la_prefill_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "la_prefill_varlen_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "la_prefill_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i,
                               _vp, _sz, _vp]),
    "la_prefill_varlen_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                  _vp, _sz, _vp]),
    "la_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "la_decode_step_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "la_decode_verify": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "la_decode_commit": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "la_prefill_host_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "la_prefill_host": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "la_prefill_backward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "la_prefill_backward_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "la_prefill_backward_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz,
                                    _vp]),
    "la_device_status": (_i, [ctypes.POINTER(_i), _i]),
    "la_selftest_wait_timeout": (_i, [_i, _vp]),
    "la_prefill_varlen_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
}

NOALLOC_MAX_SEQS = 4096  # LA_NOALLOC_MAX_SEQS in include/la.h
MAX_DRAFTS = 16  # largest m of la_decode_verify / la_decode_commit


class LAError(RuntimeError):
    """A non-LA_OK status returned by the library."""

    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


def load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"CUDA library {LIB_PATH} is not built; run `python long_context_linear_b200/build.py` "
            "(needs nvcc with sm_100a support). There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()


def check(status: int, where: str) -> None:
    if status != LA_OK:
        detail = lib.la_last_error().decode(errors="replace") or lib.la_status_string(status).decode()
        raise LAError(status, where, detail)

"""ctypes view of libaxr.so (include/axr.h).  Loads the in-tree library and declares every entry point.

There is no fallback: if the library is missing or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libaxr.so")

STATUS = {0: "AXR_OK", 1: "AXR_EINVAL", 2: "AXR_EUNSUPPORTED", 3: "AXR_ECUDA", 4: "AXR_EWORKSPACE"}
F32, F16 = 0, 1
V_F16, V_QUANT, V_QUANT_TILED = 0, 1, 2
GATHER_FACTORED, GATHER_TABLE, GATHER_TENSOR, GATHER_MMA, GATHER_DIRECT = 0, 1, 2, 3, 4
STATUS_WAIT_TIMEOUT = 1

_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_sz = ctypes.c_size_t

SIGNATURES = {
    "axr_last_error": (ctypes.c_char_p, []),
    "axr_version": (_i, []),
    "axr_codebook": (_i, [_i, _i, _p, _p]),
    "axr_write_keys": (_i, [_p, _i, _i64, _i, _i, _p, _p, _p, _p, _p]),
    "axr_write_values_tiled": (_i, [_p, _i, _i64, _i, _i, _p, _p, _i, _p, _p, _p]),
    "axr_score": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _f, _p, _p]),
    "axr_attend_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "axr_attend_decode": (_i, [_p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _f, _p, _p, _sz, _p]),
    "axr_decode_step": (_i, [_p, _p, _p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _f, _p, _p, _sz, _p]),
    "axr_attend_decode_paged": (_i, [_p, _p, _p, _i, _p, _p, _p, _i, _i, _p, _i, _i, _i, _i, _i, _i, _p, _f, _p, _p,
                                     _sz, _p]),
    "axr_decode_step_paged": (_i, [_p, _p, _p, _p, _p, _i, _p, _p, _p, _i, _i, _p, _i, _i, _i, _i, _i, _i, _p, _f, _p,
                                   _p, _sz, _p]),
    "axr_dense_decode": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _sz, _p]),
    "axr_select_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "axr_select_signs": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _i, _i, _p, _p, _p, _sz, _p]),
    "axr_select_signs_per_layer": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _i, _i, _p, _p, _p, _p, _sz,
                                        _p]),
    "axr_attend_decode_static": (_i, [_p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _f, _p, _p]),
    "axr_attend_static_scratch_bytes": (_sz, []),
    "axr_pq_train_workspace_bytes": (_sz, [_i, _i, _i]),
    "axr_pq_train": (_i, [_p, _i, _i64, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "axr_pq_encode": (_i, [_p, _i, _i64, _i, _i, _i, _p, _i, _i, _p, _p, _p]),
    "axr_pq_score": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p]),
    "axr_pq_attend_decode": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _sz, _p]),
    "axr_pot_write": (_i, [_p, _i64, _i, _i, _i, _p, _p, _p, _p]),
    "axr_pot_score": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p]),
    "axr_pot_attend_decode": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _sz, _p]),
    "axr_set_gather": (_i, [_i]),
    "axr_device_status": (_i, [_p, _i]),
    "axr_selftest_wait_timeout": (_i, [_i, _p]),
    "axr_get_gather": (_i, []),
}

_lock = threading.Lock()
_lib = None


class AxrError(RuntimeError):
    """A non-OK status from libaxr; .status holds the axr_status value."""

    def __init__(self, what: str, status: int, message: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is not built; run `python -m kv_cache_quantized_b200.build` (needs nvcc). "
                        "There is no CPU fallback.")
                L = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(L, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = L
    return _lib


def check(status: int, what: str) -> None:
    if status != 0:
        msg = lib().axr_last_error()
        raise AxrError(what, status, msg.decode() if msg else "")

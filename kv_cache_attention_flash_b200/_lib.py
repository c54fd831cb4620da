"""ctypes view of libfdllm.so (the C ABI in include/fdllm.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels. The library is required; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfdllm.so")

FDLLM_OK = 0
FDLLM_ERR_INVALID_ARG = 1
FDLLM_ERR_UNSUPPORTED = 2
FDLLM_ERR_CUDA = 3
FDLLM_ERR_DEVICE_BOUNDS = 4
FDLLM_ERR_TIMEOUT = 5
FDLLM_BF16 = 0
FDLLM_F32 = 1
FDLLM_INJECT_NONE = 0
FDLLM_INJECT_SPLIT_FLAG_TIMEOUT = 1

# Every function the header declares, with its ctypes signature.
_i32 = ctypes.c_int32
_vp = ctypes.c_void_p
_i32p = ctypes.POINTER(ctypes.c_int32)


class CacheConfig(ctypes.Structure):
    _fields_ = [
        ("n_layers", _i32), ("n_heads", _i32), ("head_dim", _i32), ("page_size", _i32),
        ("num_pages", _i32), ("max_position", _i32), ("max_batch", _i32),
        ("max_slots_per_seq", _i32), ("rope_theta", ctypes.c_float), ("dtype", _i32),
    ]


class Step(ctypes.Structure):
    _fields_ = [
        ("batch", _i32), ("total_rows", _i32), ("max_blocks_per_seq", _i32),
        ("cu_rows", _i32p), ("seq_lens", _i32p), ("slots", _vp), ("validate", _i32),
        ("out_bf16", _i32),
    ]


SIGNATURES = {
    "fdllm_cache_create": (_i32, [ctypes.POINTER(CacheConfig), _vp, _vp, _vp, ctypes.POINTER(_vp)]),
    "fdllm_cache_destroy": (None, [_vp]),
    "fdllm_layer_step": (_i32, [_vp, _i32, ctypes.POINTER(Step), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fdllm_layer_step_noalloc": (_i32, [ctypes.POINTER(CacheConfig), _vp, _vp, _vp, _vp, _i32,
                                        ctypes.POINTER(Step), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _vp]),
    "fdllm_select_tracked": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp]),
    "fdllm_verify_accept": (_i32, [_vp, _i32, _i32, _i32, _vp, _i32, _vp, ctypes.c_float, _vp,
                                   _vp, _vp, _vp]),
    "fdllm_plan_tile_schedule": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "fdllm_oproj": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp]),
    "fdllm_check": (_i32, [_vp, _vp]),
    "fdllm_inject_fault": (_i32, [_vp, _i32, ctypes.c_int64]),
    "fdllm_status_string": (ctypes.c_char_p, [_i32]),
    "fdllm_last_error": (ctypes.c_char_p, []),
    "fdllm_last_launch_count": (_i32, []),
}

_lib = None


class FdllmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"fdllm status {status}: {message}")
        self.status = status


def load() -> ctypes.CDLL:
    """Loads libfdllm.so from the package directory (built by
    kv_cache_attention_flash_b200.build). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m kv_cache_attention_flash_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check_status(status: int) -> None:
    if status != FDLLM_OK:
        lib = load()
        msg = lib.fdllm_last_error().decode()
        raise FdllmError(status, msg or lib.fdllm_status_string(status).decode())

"""The C-ABI library loads, exports every declared symbol, and rejects bad
host-side arguments before touching a GPU (no compute calls here)."""
import ctypes
import os
import re
import subprocess

import pytest

from kv_cache_attention_flash_b200 import _lib
from kv_cache_attention_flash_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"FDLLM_API\s+[\w\s\*]+?\b(fdllm_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "fdllm_layer_step" in names and "fdllm_cache_create" in names
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(fdllm_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    for n in names:
        assert hasattr(lib, n)
        assert n in _lib.SIGNATURES


def test_status_strings(lib):
    assert lib.fdllm_status_string(0) == b"ok"
    assert b"invalid" in lib.fdllm_status_string(1)
    assert lib.fdllm_status_string(99) == b"unknown status"


def test_null_arguments_are_rejected_without_a_gpu(lib):
    out = ctypes.c_void_p()
    assert lib.fdllm_cache_create(None, None, None, None, ctypes.byref(out)) == _lib.FDLLM_ERR_INVALID_ARG
    cfg = _lib.CacheConfig(1, 4, 64, 16, 8, 128, 1, 128, 10000.0, _lib.FDLLM_F32)
    assert lib.fdllm_cache_create(ctypes.byref(cfg), None, None, None, ctypes.byref(out)) == _lib.FDLLM_ERR_INVALID_ARG
    assert b"null pool" in lib.fdllm_last_error()
    # misaligned pools are refused before any allocation
    assert lib.fdllm_cache_create(ctypes.byref(cfg), 8, 8, None, ctypes.byref(out)) == _lib.FDLLM_ERR_INVALID_ARG
    bad = _lib.CacheConfig(1, 4, 64, 16, 8, 128, 1, 128, 10000.0, _lib.FDLLM_BF16)
    assert lib.fdllm_cache_create(ctypes.byref(bad), 256, 256, None, ctypes.byref(out)) == _lib.FDLLM_ERR_UNSUPPORTED
    st = _lib.Step()
    assert lib.fdllm_layer_step(None, 0, ctypes.byref(st), None, None, None, None, None, None, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    assert lib.fdllm_check(None, None) == _lib.FDLLM_ERR_INVALID_ARG
    # select_tracked: bad k / stride are host errors
    assert lib.fdllm_select_tracked(16, 16, 1, 10, 0, None, None, 16, None) == _lib.FDLLM_ERR_UNSUPPORTED
    assert lib.fdllm_select_tracked(16, 16, 1, 10, 2000, None, None, 16, None) == _lib.FDLLM_ERR_UNSUPPORTED
    assert lib.fdllm_select_tracked(16, 16, 1, 70000, 4, None, None, 16, None) == _lib.FDLLM_ERR_UNSUPPORTED
    assert lib.fdllm_select_tracked(16, 16, 1, 10, 4, 16, None, 16, None) == _lib.FDLLM_ERR_INVALID_ARG
    assert lib.fdllm_select_tracked(None, 16, 1, 10, 4, None, None, 16, None) == _lib.FDLLM_ERR_INVALID_ARG


def test_product_path_does_not_import_the_oracle():
    import sys
    code = ("import sys, kv_cache_attention_flash_b200 as p, kv_cache_attention_flash_b200.workloads; "
            "assert not any(m == 'oracle' or m.startswith('oracle.') for m in sys.modules), "
            "[m for m in sys.modules if 'oracle' in m]")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_oproj_host_checks_without_a_gpu(lib):
    """fdllm_oproj refuses bad sizes, null and misaligned pointers before any
    CUDA call (the pointers below are never dereferenced)."""
    A, Wp, Y = 1 << 20, 2 << 20, 3 << 20          # aligned stand-in addresses
    assert lib.fdllm_oproj(A, Wp, None, Y, 4, 100, None, None) == _lib.FDLLM_ERR_UNSUPPORTED
    assert b"multiple of 256" in lib.fdllm_last_error()
    assert lib.fdllm_oproj(A, Wp, None, Y, -1, 256, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    assert lib.fdllm_oproj(A, Wp, None, Y, 4, 0, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    assert lib.fdllm_oproj(None, Wp, None, Y, 4, 256, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    assert lib.fdllm_oproj(A + 8, Wp, None, Y, 4, 256, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    assert b"16-byte aligned" in lib.fdllm_last_error()
    assert lib.fdllm_oproj(A, Wp, A + 8, Y, 4, 256, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    # y may be the residual, but must not overlap the other inputs
    assert lib.fdllm_oproj(A, Wp, Y + 256, Y, 4, 256, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    assert b"overlaps" in lib.fdllm_last_error()
    assert lib.fdllm_oproj(A, Wp, None, A + 256, 4, 256, None, None) == _lib.FDLLM_ERR_INVALID_ARG
    # no rows: nothing to do, nothing enqueued
    assert lib.fdllm_oproj(None, None, None, None, 0, 256, None, None) == _lib.FDLLM_OK
    assert lib.fdllm_last_launch_count() == 0

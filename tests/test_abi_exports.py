"""The C-ABI library loads on a machine without a GPU and exports every
symbol include/kvq.h declares (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from calibration_free_rotated_token_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ctypes.CDLL(_abi.LIB_PATH)


def test_header_and_binding_agree():
    assert _declared() == sorted(_abi.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_last_error_callable_without_gpu(lib):
    lib.kvq_last_error.restype = ctypes.c_char_p
    assert lib.kvq_last_error() == b""


def test_invalid_arguments_are_rejected_on_host(lib):
    lib.kvq_init.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                             ctypes.c_uint32]
    lib.kvq_last_error.restype = ctypes.c_char_p
    h = ctypes.c_void_p()
    assert lib.kvq_init(ctypes.byref(h), 96, 2, 1, 1) == _abi.KVQ_EINVAL
    assert b"d must be" in lib.kvq_last_error()
    assert lib.kvq_init(ctypes.byref(h), 128, 5, 1, 1) == _abi.KVQ_EINVAL
    assert lib.kvq_init(ctypes.byref(h), 128, 2, 1, 8) == _abi.KVQ_EINVAL
    assert lib.kvq_init(None, 128, 2, 1, 1) == _abi.KVQ_EINVAL
    assert lib.kvq_destroy(None) == 0


def test_quantize_batch_rejects_bad_arguments_on_host(lib):
    lib.kvq_quantize_batch.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    lib.kvq_last_error.restype = ctypes.c_char_p
    assert lib.kvq_quantize_batch(None, 0, None, None) == _abi.KVQ_EINVAL
    assert b"null handle" in lib.kvq_last_error()

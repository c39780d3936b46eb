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



@pytest.mark.parametrize("beta", [False, True])
def test_library_codebook_matches_oracle_on_host(lib, beta):
    """The library's codebook (computed on the host, no device) against the
    oracle's: two independent computations, equal to fp32 rounding."""
    import numpy as np

    import oracle
    for d in (64, 128, 256):
        for b in (1, 2, 3, 4):
            c, t = _abi.kvq_codebook(d, b, beta)
            co, to, _, _ = oracle.lloyd_max_sphere(d, b) if beta else oracle.lloyd_max(b)
            np.testing.assert_allclose(c, co, rtol=2.0 ** -23, atol=1e-12)
            np.testing.assert_allclose(t, to, rtol=2.0 ** -23, atol=1e-12)
    import ctypes as C
    buf = (C.c_float * 16)()
    assert lib.kvq_codebook(96, 2, 0, buf, buf) == _abi.KVQ_EINVAL
    assert lib.kvq_codebook(128, 2, 8, buf, buf) == _abi.KVQ_EINVAL
    assert lib.kvq_codebook(128, 2, 0, None, buf) == _abi.KVQ_EINVAL
    # the rotation flag is a valid flag and leaves the codebook unchanged
    ref = (C.c_float * 16)()
    assert lib.kvq_codebook(128, 3, 0, ref, buf) == _abi.KVQ_OK
    got = (C.c_float * 16)()
    assert lib.kvq_codebook(128, 3, _abi.KVQ_CUDA_CORE_ROTATION | _abi.KVQ_QJL, got, buf) == _abi.KVQ_OK
    assert list(got)[:8] == list(ref)[:8]

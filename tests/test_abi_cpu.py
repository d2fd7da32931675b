"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/saga.h declares, and rejects bad arguments before it
touches CUDA."""
import ctypes
import os
import re

import pytest

from sparse_asymmetric_gqa_b200 import _lib
from sparse_asymmetric_gqa_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "saga.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SAGA_API\s+[\w\s\*]+?\b(saga_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("saga_decode_init", "saga_decode_attn", "saga_decode_free", "saga_score",
                 "saga_select", "saga_combine", "saga_decode_attn_host", "saga_decode_status"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_error_strings(lib):
    for code in range(0, 6):
        s = lib.saga_decode_error_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.saga_decode_error_string(0) == b"ok"


@pytest.mark.parametrize("args,code", [
    ((0, 1024, 16, 1, 8, 64, 128), _lib.SAGA_ERR_INVALID_ARG),      # batch 0
    ((1, 0, 16, 1, 8, 64, 128), _lib.SAGA_ERR_INVALID_ARG),         # no positions
    ((1, 1024, 16, 3, 8, 64, 128), _lib.SAGA_ERR_INVALID_ARG),      # h_k does not divide h_q
    ((1, 1024, 16, 1, 6, 64, 128), _lib.SAGA_ERR_INVALID_ARG),      # h_v does not divide h_q
    ((1, 1024, 16, 1, 8, 64, 0), _lib.SAGA_ERR_INVALID_ARG),        # max_N 0
    ((2000, 1024, 16, 1, 8, 64, 128), _lib.SAGA_ERR_INVALID_ARG),   # batch above 1024
    ((1024, 1 << 24, 16, 1, 8, 64, 128), _lib.SAGA_ERR_INVALID_ARG),  # rows overflow int32
    ((1, 1024, 16, 1, 8, 96, 128), _lib.SAGA_ERR_UNSUPPORTED),      # head_dim 96
    ((1, 1024, 128, 1, 8, 64, 128), _lib.SAGA_ERR_UNSUPPORTED),     # group of 128 > 64
])
def test_init_validation_happens_before_cuda(lib, args, code):
    h = ctypes.c_void_p()
    assert lib.saga_decode_init(ctypes.byref(h), *args, None) == code
    assert not h.value


def test_null_handle_rejected(lib):
    assert lib.saga_decode_set_batch(None, 1) == _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_decode_attn(None, None, None, None, None, 1, 1, 1, 64, 1, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_decode_free(None) == _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_decode_selftest_timeout(None) == _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_group_attn(None, None, None, None, None, 1, 1, 1, 64, 1, None, None, None,
                               None) == _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_atopn_calibrate(None, None, None, None, None, 1, 1, 1, 64, 1, None, None,
                                    None, None) == _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_atopn_step(None, None, None, None, None, 1, 1, 1, 64, 1, None, None,
                               None, None) == _lib.SAGA_ERR_INVALID_ARG
    v = ctypes.c_int()
    assert lib.saga_decode_status(None, ctypes.byref(v)) == _lib.SAGA_ERR_INVALID_ARG


def test_unaligned_value_cache_rejected_before_cuda(lib):
    # v_cache must start on a 16-byte boundary; the check comes before any CUDA call
    fake = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    rc = lib.saga_combine_noalloc(fake, fake, odd, fake, 1, 64, 8, 2, 128, 16, fake, None)
    assert rc == _lib.SAGA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load()

"""ctypes declarations of the C ABI in include/saga.h (argument marshalling only)."""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsaga.so")

SAGA_OK = 0
SAGA_ERR_INVALID_ARG = 1
SAGA_ERR_UNSUPPORTED = 2
SAGA_ERR_CUDA = 3
SAGA_ERR_DEVICE = 4
SAGA_ERR_SCRATCH_TOO_SMALL = 5
SAGA_STATUS_BAD_SEQ_LEN = 0x1
SAGA_STATUS_TIMEOUT = 0x2
SAGA_STATUS_BAD_INDEX = 0x4
SAGA_STATUS_INFO_EXACT_FALLBACK = 0x100
SAGA_STATUS_INFO_ROBUST_PATH = 0x200

_P = ctypes.c_void_p
_I = ctypes.c_int

# name -> (restype, argtypes)
SIGNATURES = {
    "saga_decode_init": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I, _P]),
    "saga_decode_init_kv": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "saga_decode_set_batch": (_I, [_P, _I]),
    "saga_decode_set_stream": (_I, [_P, _P]),
    "saga_decode_attn": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "saga_decode_attn_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "saga_decode_attn_host": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "saga_atopn_calibrate": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "saga_atopn_step": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "saga_score": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _I]),
    "saga_select": (_I, [_P, _P, _I, _P, _I, _I, _P, _P]),
    "saga_combine": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "saga_combine_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]),
    "saga_decode_status": (_I, [_P, ctypes.POINTER(_I)]),
    "saga_decode_selftest_timeout": (_I, [_P]),
    "saga_group_attn": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "saga_decode_launch_count": (_I, [_P, ctypes.POINTER(ctypes.c_longlong)]),
    "saga_decode_profile": (_I, [_P, _I, _I]),
    "saga_decode_profile_read": (_I, [_P, ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I)]),
    "saga_decode_error_string": (ctypes.c_char_p, [_I]),
    "saga_decode_free": (_I, [_P]),
}

_lib = None


def load():
    """Load libsaga.so (built in-tree by sparse_asymmetric_gqa_b200/build.py).

    Raises RuntimeError if it is missing: there is no fallback implementation.
    """
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"SAGA CUDA library not built: {LIB_PATH} is missing "
                           "(run `python sparse_asymmetric_gqa_b200/build.py`)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class SagaError(RuntimeError):
    def __init__(self, fn, code, status=None):
        msg = load().saga_decode_error_string(code).decode()
        extra = f", device status 0x{status:x}" if status is not None else ""
        super().__init__(f"{fn} failed: {msg} (code {code}{extra})")
        self.code = code
        self.status = status


def check(fn, code):
    if code != SAGA_OK:
        raise SagaError(fn, code)

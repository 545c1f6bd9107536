"""ctypes view of libw4.so: the C ABI declared in include/w4.h, one Python
callable per entry point, taking raw integer addresses.

Nothing here computes anything: it loads the library (failing loudly if it is
missing) and declares argument types.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# W4_LIBRARY=debug selects libw4_debug.so: the same kernels built with their
# device-side index checks on (tests run the small parity cases against it).
LIB_NAME = "libw4_debug.so" if os.environ.get("W4_LIBRARY") == "debug" else "libw4.so"
LIB_PATH = os.path.join(_HERE, LIB_NAME)

W4_OK = 0
W4_ERR_NULL = 1
W4_ERR_SHAPE = 2
W4_ERR_ALIGN = 3
W4_ERR_UNSUPPORTED_DEVICE = 4
W4_ERR_WORKSPACE = 5
W4_ERR_CUDA = 6
W4_ERR_TIMEOUT = 7
W4_ERR_BOUNDS = 8
W4_OUT_BF16 = 0
W4_OUT_F32 = 1

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int

SIGNATURES = {
    "w4_abi_version": ([], _INT),
    "w4_status_string": ([_INT], ctypes.c_char_p),
    "w4_last_cuda_error": ([], _INT),
    "w4_check_device_error": ([], _INT),
    "w4_pack": ([_P, _I64, _I64, _P, _P, _P, _P], _INT),
    "w4_pack_g32": ([_P, _I64, _I64, _P, _P, _P, _P], _INT),
    "w4_pack_codes": ([_P, _I64, _I64, _P, _P], _INT),
    "w4_unpack": ([_P, _I64, _I64, _P, _P], _INT),
    "w4_gemv": ([_P, _P, _P, _I64, _I64, _P, _INT, _P, _INT, _P], _INT),
    "w4_gemv_g32": ([_P, _P, _P, _I64, _I64, _P, _INT, _P, _INT, _P], _INT),
    "w4a8_gemv": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _INT, _P, _INT, _P], _INT),
    "w4a8_gemv_bf16": ([_P, _P, _P, _I64, _I64, _P, _INT, _P, _INT, _P], _INT),
    "q8_quantize_act": ([_P, _I64, _I64, _P, _P, _P, _P], _INT),
    "w4a8_mmq_workspace_size": ([_I64, _I64, _I64], ctypes.c_size_t),
    "w4a8_mmq": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _INT, _P, ctypes.c_size_t, _P],
                 _INT),
    "w4a8_mmq_static": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _INT, _P], _INT),
    "w4_test_wait_expiry": ([ctypes.c_uint64, _P], _INT),
    "w4a8_gemv_blockdots": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _INT, _P, _INT, _P,
                             ctypes.c_size_t, _P], _INT),
    "w4a8_mmq_blockdots": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _INT, _P,
                            ctypes.c_size_t, _P, ctypes.c_size_t, _P], _INT),
}

W4A8_MMQ_STATIC_SCRATCH_BYTES = 40 * 1024 * 1024


class LibraryMissing(RuntimeError):
    pass


_lib = None


def load() -> ctypes.CDLL:
    """Load libw4.so from the package directory.  Raises LibraryMissing if it
    has not been built (there is no fallback implementation)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise LibraryMissing(
            f"{LIB_PATH} is not built; run `python -m w4_quant_matmul_b200.build` "
            "(with --debug for libw4_debug.so; nvcc, sm_100a).  There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (args, res) in SIGNATURES.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().w4_status_string(int(code)).decode()

"""CPU oracle for the W4-G256 quantized matmul (and its group-32 variant) --
TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper over ``w4_oracle.c`` (plain C, fp64/int64 reductions).
Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``w4_quant_matmul_b200``) never imports it and has no fallback to it.

All arrays are numpy, C-contiguous, on the host.  bf16 and fp16 values travel
as their raw 16-bit patterns (``np.uint16``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4_oracle.c")
_LIB_NAME = "liboracle_w4.so"
_lock = threading.Lock()
_lib = None

GROUP = 256
BLOCK = 32


def compile_oracle(out_path: str | None = None, defines: tuple[str, ...] = (),
                   openmp: bool = True) -> str:
    """Compile the oracle into a shared library and return its path.

    ``defines`` adds ``-D`` macros (the planted-mistake variants used by the
    mutation tests).  fp contraction is off and no fast-math is used, so the
    fp32 quantisers round exactly as written."""
    if out_path is None:
        out_path = os.path.join(_HERE, _LIB_NAME)
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wno-unknown-pragmas"]
    if openmp:
        cmd.append("-fopenmp")
    cmd += ["-D" + d for d in defines]
    cmd += [_SRC, "-o", out_path, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    return out_path


def _needs_build(path: str) -> bool:
    return (not os.path.exists(path)) or os.path.getmtime(path) < os.path.getmtime(_SRC)


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    I = ctypes.c_int64
    sig = {
        "oracle_pack_codes": [P, I, I, P],
        "oracle_unpack": [P, I, I, P],
        "oracle_w4_pack": [P, I, I, P, P, P],
        "oracle_w4_pack_grouped": [P, I, I, I, P, P, P],
        "oracle_q8_quantize": [P, I, I, P, P, P],
        "oracle_gemv_f64_rows": [P, P, P, I, I, P, I, I, I, P],
        "oracle_gemv_rows": [P, P, P, I, I, P, I, I, I, P],
        "oracle_gemv_f64_rows_grouped": [P, P, P, I, I, I, P, I, I, I, P],
        "oracle_gemv_rows_grouped": [P, P, P, I, I, I, P, I, I, I, P],
        "oracle_mmq_blockdots": [P, I, I, P, I, P],
        "oracle_mmq_rows": [P, P, P, I, I, P, P, P, I, I, I, P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_set_num_threads.restype = None
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    return lib


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            p = os.path.join(_HERE, _LIB_NAME)
            if _needs_build(p):
                compile_oracle(p)
            _lib = _bind(ctypes.CDLL(p))
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


class Oracle:
    """The oracle's entry points with numpy in/out.  ``lib`` may be a
    planted-mistake build (mutation tests); the default is the normal one."""

    def __init__(self, lib: ctypes.CDLL | None = None):
        self.lib = lib if lib is not None else load()

    # -- threads ---------------------------------------------------------
    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    # -- packing ---------------------------------------------------------
    def pack_codes(self, q: np.ndarray) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.uint8)
        N, K = q.shape
        out = np.empty((N, K // 2), np.uint8)
        _check(self.lib.oracle_pack_codes(_ptr(q), N, K, _ptr(out)), "pack_codes")
        return out

    def unpack(self, codes: np.ndarray, K: int) -> np.ndarray:
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        N = codes.shape[0]
        out = np.empty((N, K), np.uint8)
        _check(self.lib.oracle_unpack(_ptr(codes), N, K, _ptr(out)), "unpack")
        return out

    def w4_pack(self, w: np.ndarray, group: int = GROUP):
        """fp32 W[N,K] -> (codes u8[N,K/2], d fp16-bits[N,G], m fp16-bits[N,G]),
        G = K / group (256: W4-G256; 32: the group-32 scheme)."""
        w = np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        codes = np.empty((N, K // 2), np.uint8)
        G = K // group
        d = np.empty((N, G), np.uint16)
        m = np.empty((N, G), np.uint16)
        if group == GROUP:
            rc = self.lib.oracle_w4_pack(_ptr(w), N, K, _ptr(codes), _ptr(d), _ptr(m))
        else:
            rc = self.lib.oracle_w4_pack_grouped(_ptr(w), N, K, group, _ptr(codes), _ptr(d),
                                                 _ptr(m))
        _check(rc, "w4_pack")
        return codes, d, m

    # -- activation quantiser --------------------------------------------
    def q8_quantize(self, x_bf16: np.ndarray):
        """bf16-bits x[M,K] -> (qa int8[M,K], dx fp32[M,K/32], S int32[M,K/32])."""
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        M, K = x.shape
        B = K // BLOCK
        qa = np.empty((M, K), np.int8)
        dx = np.empty((M, B), np.float32)
        S = np.empty((M, B), np.int32)
        _check(self.lib.oracle_q8_quantize(_ptr(x), M, K, _ptr(qa), _ptr(dx), _ptr(S)),
               "q8_quantize")
        return qa, dx, S

    # -- products ----------------------------------------------------------
    def gemv(self, codes, d, m, x_bf16, rows: tuple[int, int] | None = None,
             group: int = GROUP) -> np.ndarray:
        """y[M, rows] in fp64 for bf16-bits x[M,K]; d, m are [N, K/group]."""
        codes = np.ascontiguousarray(codes, np.uint8)
        d = np.ascontiguousarray(d, np.uint16)
        m = np.ascontiguousarray(m, np.uint16)
        x = np.ascontiguousarray(x_bf16, np.uint16)
        N = codes.shape[0]
        M, K = x.shape
        n0, n1 = rows if rows is not None else (0, N)
        y = np.empty((M, n1 - n0), np.float64)
        if group == GROUP:
            rc = self.lib.oracle_gemv_rows(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(x), M,
                                           n0, n1, _ptr(y))
        else:
            rc = self.lib.oracle_gemv_rows_grouped(_ptr(codes), _ptr(d), _ptr(m), N, K, group,
                                                   _ptr(x), M, n0, n1, _ptr(y))
        _check(rc, "gemv")
        return y

    def gemv_f64(self, codes, d, m, x: np.ndarray, rows=None, group: int = GROUP) -> np.ndarray:
        """Same product with fp64 activations x[M,K]."""
        codes = np.ascontiguousarray(codes, np.uint8)
        d = np.ascontiguousarray(d, np.uint16)
        m = np.ascontiguousarray(m, np.uint16)
        x = np.ascontiguousarray(x, np.float64)
        N = codes.shape[0]
        M, K = x.shape
        n0, n1 = rows if rows is not None else (0, N)
        y = np.empty((M, n1 - n0), np.float64)
        if group == GROUP:
            rc = self.lib.oracle_gemv_f64_rows(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(x),
                                               M, n0, n1, _ptr(y))
        else:
            rc = self.lib.oracle_gemv_f64_rows_grouped(_ptr(codes), _ptr(d), _ptr(m), N, K,
                                                       group, _ptr(x), M, n0, n1, _ptr(y))
        _check(rc, "gemv_f64")
        return y

    def mmq_blockdots(self, codes, qa) -> np.ndarray:
        """Exact int64 P[M,N,K/32]."""
        codes = np.ascontiguousarray(codes, np.uint8)
        qa = np.ascontiguousarray(qa, np.int8)
        N = codes.shape[0]
        M, K = qa.shape
        P = np.empty((M, N, K // BLOCK), np.int64)
        _check(self.lib.oracle_mmq_blockdots(_ptr(codes), N, K, _ptr(qa), M, _ptr(P)),
               "mmq_blockdots")
        return P

    def mmq(self, codes, d, m, qa, dx, S, rows=None) -> np.ndarray:
        """y[M, rows] in fp64 of the W4A8 product."""
        codes = np.ascontiguousarray(codes, np.uint8)
        d = np.ascontiguousarray(d, np.uint16)
        m = np.ascontiguousarray(m, np.uint16)
        qa = np.ascontiguousarray(qa, np.int8)
        dx = np.ascontiguousarray(dx, np.float32)
        S = np.ascontiguousarray(S, np.int32)
        N = codes.shape[0]
        M, K = qa.shape
        n0, n1 = rows if rows is not None else (0, N)
        y = np.empty((M, n1 - n0), np.float64)
        _check(self.lib.oracle_mmq_rows(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa),
                                        _ptr(dx), _ptr(S), M, n0, n1, _ptr(y)), "mmq")
        return y


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from the unmodified source."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default

"""Build libw4.so in-tree: nvcc for sm_100a, one object per source, linked
with the static CUDA runtime so the library is self-contained.

    python -m w4_quant_matmul_b200.build          # build if sources changed
    python -m w4_quant_matmul_b200.build --force  # rebuild everything
    python -m w4_quant_matmul_b200.build --debug  # libw4_debug.so (-DW4_DEBUG)

The ptxas resource report (registers, spills, shared memory per kernel) is
written to ``_build/ptxas.log``.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
BUILD_DEBUG = os.path.join(BUILD, "debug")
LIB = os.path.join(PKG, "libw4.so")
LIB_DEBUG = os.path.join(PKG, "libw4_debug.so")
SOURCES = ["abi.cu", "pack.cu", "quant.cu", "gemv.cu", "gemv_blockdots.cu", "mmq.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# No --use_fast_math / -ftz=true / -prec-div=false: the W4A8 product's epilogue
# multiplies exact integer products held as fp32 denormals, which a
# flush-to-zero build would zero, and the quantisers depend on IEEE division
# and rounding (tests/test_build_audit.py checks these flags).
NVCC_FLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
                     "-Xptxas", "-v", "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]
# The debug library: the same sources with the device-side index checks on.
DEBUG_FLAGS = ["-DW4_DEBUG"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _deps() -> list[str]:
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return hdrs + [os.path.join(INCLUDE, "w4.h")]


def _stale(target: str, inputs: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in inputs)


def _compile(src: str, force: bool, debug: bool = False) -> tuple[str, str]:
    out_dir = BUILD_DEBUG if debug else BUILD
    obj = os.path.join(out_dir, src.replace(".cu", ".o"))
    path = os.path.join(CSRC, src)
    if not force and not _stale(obj, [path] + _deps()):
        log = obj + ".ptxas"
        return obj, open(log).read() if os.path.exists(log) else ""
    cmd = [_nvcc()] + NVCC_FLAGS + (DEBUG_FLAGS if debug else []) + ["-c", path, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    with open(obj + ".ptxas", "w") as f:
        f.write(r.stderr)
    return obj, r.stderr


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link ``libw4.so`` (with
    ``debug``: the -DW4_DEBUG build with device-side index checks,
    ``libw4_debug.so``)."""
    out_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    os.makedirs(out_dir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, force, debug), SOURCES))
    objs = [o for o, _ in results]
    with open(os.path.join(out_dir, "ptxas.log"), "w") as f:
        for src, (_, log) in zip(SOURCES, results):
            f.write(f"==== {src}\n{log}\n")
    if force or _stale(lib, objs):
        cmd = [_nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    if verbose and not debug:
        print(spill_report())
    return lib


def build_all(force: bool = False) -> tuple[str, str]:
    """The release and the debug library, compiled side by side."""
    with cf.ThreadPoolExecutor(max_workers=2) as ex:
        rel = ex.submit(build, force, False, False)
        dbg = ex.submit(build, force, False, True)
        return rel.result(), dbg.result()


def spill_report() -> str:
    """Kernels whose ptxas report shows spill stores (from the last build)."""
    path = os.path.join(BUILD, "ptxas.log")
    if not os.path.exists(path):
        return "no ptxas log"
    out, func = [], None
    for line in open(path):
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            func = m.group(1)
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and int(m.group(1)) > 0:
            out.append(f"{func}: {line.strip()}")
    return "\n".join(out) if out else "no spills"


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))

"""Register-spill audit of the built library (CPU only: reads the ptxas
resource report that the build writes to _build/ptxas.log).

No kernel may spill, except the measured instantiations listed below (and
the test-only instantiations that store block products), each up to the
bytes it spills today: a new spill, or a larger one, fails.
"""
import os
import re
import shutil
import subprocess

import pytest

# demangled kernel name -> largest spill-store bytes accepted
KNOWN_SPILLS = {
    # bf16 decode GEMV, M = 4, two rows per half-warp (streams of >= 18944
    # rows: the 19456 x 2560 up-projection and the lm_head)
    "w4_gemv_rows_kernel<4, 2, 4, 0, 3, false>": 12,
    # the same for group-32 weights
    "w4_gemv_rows_kernel<4, 2, 4, 0, 0, false>": 4,
    # test instantiations of the keep-quant GEMV that also store the block
    # products (never timed)
    "w4_gemv_rows_kernel<4, 2, 4, 1, 3, true>": 4,
    "w4_gemv_rows_kernel<3, 4, 2, 1, 3, true>": 24,
    # decode GEMV row kernels at M = 5..8, all forms and group sizes: two CTAs
    # per SM (128 registers) with these spills measured faster than one CTA
    # with 248 registers and none
    "w4_gemv_rows_kernel<5, ": 28,
    "w4_gemv_rows_kernel<6, ": 16,
    "w4_gemv_rows_kernel<7, ": 44,
    "w4_gemv_rows_kernel<8, ": 36,
    # the W4A8 prefill kernel (warp-specialised with setmaxnreg)
    "w4a8_mmq_kernel<false>(": 4,
}


@pytest.fixture(scope="module")
def ptxas_log():
    from w4_quant_matmul_b200 import build
    build.build()
    path = os.path.join(build.BUILD, "ptxas.log")
    return open(path).read()


def _demangle(names):
    tool = shutil.which("c++filt")
    if not tool or not names:
        return dict(zip(names, names))
    out = subprocess.run([tool], input="\n".join(names), capture_output=True, text=True)
    return dict(zip(names, out.stdout.splitlines()))


def _spills(text):
    found, func = {}, None
    for line in text.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            func = m.group(1)
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and func and int(m.group(1)) > 0:
            found[func] = max(found.get(func, 0), int(m.group(1)))
    return found


def test_every_source_was_compiled(ptxas_log):
    from w4_quant_matmul_b200 import build
    for src in build.SOURCES:
        assert f"==== {src}" in ptxas_log, src
    assert "Compiling entry function" in ptxas_log


def test_no_spills_beyond_the_known_ones(ptxas_log):
    spills = _spills(ptxas_log)
    names = _demangle(list(spills))
    unexpected = []
    for mangled, nbytes in spills.items():
        name = names[mangled]
        allowed = [b for key, b in KNOWN_SPILLS.items() if key in name]
        if not allowed or nbytes > max(allowed):
            unexpected.append(f"{name}: {nbytes} bytes spill stores")
    assert not unexpected, "\n".join(unexpected)


def test_parser_sees_a_spill():
    # the parser itself, on a hand-written report line pair
    text = ("ptxas info    : Compiling entry function '_Z3foov' for 'sm_100a'\n"
            "ptxas info    : Function properties for _Z3foov\n"
            "    8 bytes stack frame, 4 bytes spill stores, 4 bytes spill loads\n")
    assert _spills(text) == {"_Z3foov": 4}


def test_build_flags_keep_denormals_and_ieee_division():
    # The W4A8 product's epilogue reads exact integer products as fp32
    # denormals (V * 2^-149) and multiplies them at full rate; flushing
    # denormals to zero would silently zero every product.  The quantisers
    # rely on IEEE division and rounding.  So no fast-math-style flag may
    # reach nvcc.
    from w4_quant_matmul_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    for bad in ("--use_fast_math", "-use_fast_math", "-ftz=true", "--ftz=true",
                "-prec-div=false", "--prec-div=false", "-prec-sqrt=false",
                ):
        assert bad not in flags, bad


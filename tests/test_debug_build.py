"""The debug library (libw4_debug.so: the same sources built with -DW4_DEBUG,
device-side index checks on every guarded global and shared-memory access).

On the CPU: it builds and exports every entry point the header declares.
On the GPU: the small parity cases of every kernel run against it in a child
process (W4_LIBRARY=debug) -- results must still match the oracle, and after
each test the device error word must be clear, i.e. no index check failed.
This stands in for a memory checker, which this pool does not offer; it runs
on the small shapes only."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4.h")

SMALL_CASES = [
    "tests/test_pack.py::test_pack_bit_exact_small",
    "tests/test_pack.py::test_pack_signed_zero_groups",
    "tests/test_quant.py::test_quant_bit_exact_small",
    "tests/test_quant.py::test_quant_special_blocks",
    "tests/test_gemv.py::test_small_shapes_all_outputs",
    "tests/test_gemv.py::test_large_k_every_m",
    "tests/test_w4a8_gemv.py::test_integer_block_products_bit_exact",
    "tests/test_g32.py",
    "tests/test_mmq.py::test_small_shapes_all_outputs",
    "tests/test_mmq.py::test_integer_block_products_bit_exact",
]


def test_debug_library_builds_and_exports_the_abi():
    from w4_quant_matmul_b200 import build
    import test_abi
    path = build.build(debug=True)
    assert path.endswith("libw4_debug.so") and os.path.exists(path)
    lib = ctypes.CDLL(path)
    for name in test_abi.declared_functions():
        assert hasattr(lib, name), name


@pytest.mark.gpu
def test_small_parity_cases_with_index_checks():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from w4_quant_matmul_b200 import build
    build.build(debug=True)
    env = dict(os.environ, W4_LIBRARY="debug")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p",
                        "no:cacheprovider"] + SMALL_CASES,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, (r.stdout[-4000:], r.stderr[-2000:])
    assert " passed" in r.stdout

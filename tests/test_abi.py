"""The C ABI: the built library loads and exports every entry point that
include/w4.h declares; argument validation answers before anything touches a
device (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4.h")


@pytest.fixture(scope="module")
def lib():
    from w4_quant_matmul_b200 import build, _lib
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_0-9]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for expected in ["w4_pack", "w4_pack_g32", "w4_pack_codes", "w4_unpack", "w4_gemv",
                     "w4_gemv_g32", "w4a8_gemv",
                     "w4a8_gemv_bf16", "q8_quantize_act",
                     "w4a8_mmq", "w4a8_mmq_workspace_size", "w4_status_string",
                     "w4_abi_version", "w4_last_cuda_error", "w4_check_device_error"]:
        assert expected in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_binding_covers_every_declared_symbol():
    from w4_quant_matmul_b200 import _lib
    assert set(declared_functions()) == set(_lib.SIGNATURES)


def test_version_and_status_strings(lib):
    assert lib.w4_abi_version() == 1
    for code in range(8):
        s = lib.w4_status_string(code).decode()
        assert s.startswith("W4_")
    assert "unknown" in lib.w4_status_string(99).decode()


FAKE = 0x10000  # never dereferenced: validation fails first
MIS = 0x10001   # misaligned


def test_gemv_validation(lib):
    from w4_quant_matmul_b200 import _lib as L
    f = lib.w4_gemv
    # shapes first
    assert f(FAKE, FAKE, FAKE, 256, 300, FAKE, 1, FAKE, 0, None) == L.W4_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, 0, FAKE, 0, None) == L.W4_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, 9, FAKE, 0, None) == L.W4_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, 0, 512, FAKE, 1, FAKE, 0, None) == L.W4_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, 1, FAKE, 7, None) == L.W4_ERR_SHAPE
    # then pointers
    assert f(None, FAKE, FAKE, 256, 512, FAKE, 1, FAKE, 0, None) == L.W4_ERR_NULL
    assert f(FAKE, FAKE, FAKE, 256, 512, None, 1, FAKE, 0, None) == L.W4_ERR_NULL
    assert f(MIS, FAKE, FAKE, 256, 512, FAKE, 1, FAKE, 0, None) == L.W4_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, 1, MIS, 0, None) == L.W4_ERR_ALIGN


def test_w4a8_gemv_validation(lib):
    from w4_quant_matmul_b200 import _lib as L
    f = lib.w4a8_gemv
    assert f(FAKE, FAKE, FAKE, 256, 300, FAKE, FAKE, FAKE, 1, FAKE, 0, None) == L.W4_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, FAKE, FAKE, 9, FAKE, 0, None) == L.W4_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, FAKE, FAKE, 1, FAKE, 7, None) == L.W4_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, None, FAKE, 1, FAKE, 0, None) == L.W4_ERR_NULL
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, FAKE, None, 1, FAKE, 0, None) == L.W4_ERR_NULL
    assert f(FAKE, FAKE, FAKE, 256, 512, MIS, FAKE, FAKE, 1, FAKE, 0, None) == L.W4_ERR_ALIGN
    assert f(FAKE, FAKE, FAKE, 256, 512, FAKE, MIS, FAKE, 1, FAKE, 0, None) == L.W4_ERR_ALIGN


def test_g32_validation(lib):
    from w4_quant_matmul_b200 import _lib as L
    f = lib.w4_gemv_g32
    assert f(FAKE, FAKE, FAKE, 256, 48, FAKE, 1, FAKE, 0, None) == L.W4_ERR_SHAPE   # K % 32
    assert f(FAKE, FAKE, FAKE, 256, 0, FAKE, 1, FAKE, 0, None) == L.W4_ERR_SHAPE    # K < 32
    assert f(FAKE, FAKE, FAKE, 256, 96, FAKE, 9, FAKE, 0, None) == L.W4_ERR_SHAPE   # M
    assert f(FAKE, FAKE, FAKE, 256, 96, FAKE, 1, FAKE, 5, None) == L.W4_ERR_SHAPE   # out dtype
    assert f(None, FAKE, FAKE, 256, 96, FAKE, 1, FAKE, 0, None) == L.W4_ERR_NULL
    assert f(FAKE, FAKE, MIS, 256, 96, FAKE, 1, FAKE, 0, None) == L.W4_ERR_ALIGN
    assert lib.w4_pack_g32(FAKE, 4, 48, FAKE, FAKE, FAKE, None) == L.W4_ERR_SHAPE
    assert lib.w4_pack_g32(None, 4, 96, FAKE, FAKE, FAKE, None) == L.W4_ERR_NULL
    assert lib.w4_pack_g32(FAKE, 4, 96, MIS, FAKE, FAKE, None) == L.W4_ERR_ALIGN
    assert lib.w4_pack_g32(FAKE, 0, 96, FAKE, FAKE, FAKE, None) == L.W4_OK   # nothing to do
    # 256-group rules still hold for the W4-G256 entry points
    assert lib.w4_gemv(FAKE, FAKE, FAKE, 256, 96, FAKE, 1, FAKE, 0, None) == L.W4_ERR_SHAPE
    assert lib.w4_pack(FAKE, 4, 96, FAKE, FAKE, FAKE, None) == L.W4_ERR_SHAPE


def test_pack_and_quantizer_validation(lib):
    from w4_quant_matmul_b200 import _lib as L
    assert lib.w4_pack(FAKE, 4, 300, FAKE, FAKE, FAKE, None) == L.W4_ERR_SHAPE
    assert lib.w4_pack(None, 4, 256, FAKE, FAKE, FAKE, None) == L.W4_ERR_NULL
    assert lib.w4_pack(FAKE, 4, 256, FAKE, MIS, FAKE, None) == L.W4_ERR_ALIGN
    assert lib.w4_pack(FAKE, 0, 256, FAKE, FAKE, FAKE, None) == L.W4_OK  # nothing to do
    assert lib.w4_pack_codes(FAKE, 3, 5, FAKE, None) == L.W4_ERR_SHAPE
    assert lib.w4_unpack(None, 3, 4, FAKE, None) == L.W4_ERR_NULL
    assert lib.q8_quantize_act(FAKE, 2, 48, FAKE, FAKE, FAKE, None) == L.W4_ERR_SHAPE
    assert lib.q8_quantize_act(FAKE, 2, 64, FAKE, None, FAKE, None) == L.W4_ERR_NULL
    assert lib.q8_quantize_act(FAKE, 2, 64, FAKE, FAKE, MIS, None) == L.W4_ERR_ALIGN
    assert lib.q8_quantize_act(FAKE, 0, 64, FAKE, FAKE, FAKE, None) == L.W4_OK


def test_wait_expiry_validation(lib):
    # limits outside (0, 0.1 s] are refused before any device work
    from w4_quant_matmul_b200 import _lib as L
    assert lib.w4_test_wait_expiry(0, None) == L.W4_ERR_SHAPE
    assert lib.w4_test_wait_expiry(100_000_001, None) == L.W4_ERR_SHAPE


def test_mmq_validation(lib):
    from w4_quant_matmul_b200 import _lib as L
    f = lib.w4a8_mmq
    args = [FAKE, FAKE, FAKE, 256, 512, FAKE, FAKE, FAKE, 128, FAKE, 0, None, 0, None]

    def call(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)

    assert call(a4=384) == L.W4_ERR_SHAPE          # K % 256
    assert call(a4=256 * 513) == L.W4_ERR_SHAPE    # K above the supported maximum
    assert call(a8=0) == L.W4_ERR_SHAPE            # M
    assert call(a10=3) == L.W4_ERR_SHAPE           # out dtype
    assert call(a5=None) == L.W4_ERR_NULL
    assert call(a6=MIS) == L.W4_ERR_ALIGN
    # (148 SMs when no device is present) output tiles in whole waves need no
    # workspace; a partial last wave is split along K and needs one
    assert lib.w4a8_mmq_workspace_size(1024, 18944, 2560) == 0
    assert lib.w4a8_mmq_workspace_size(2048, 19456, 2560) > 0


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    from w4_quant_matmul_b200 import _lib as L
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(L.LibraryMissing):
        L.load()


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "w4_quant_matmul_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in src.lower(), fn


def test_without_a_device_valid_calls_fail_loudly(lib):
    # no CPU path: with valid arguments and no usable CUDA device, every entry
    # point stops at the device check and returns an error (nothing computed)
    import torch
    from w4_quant_matmul_b200 import _lib as L
    if torch.cuda.is_available() or lib.w4_check_device_error() == L.W4_OK:
        pytest.skip("a CUDA device is present; this checks the no-device branch only")
    M, N, K = 128, 256, 512
    ws = lib.w4a8_mmq_workspace_size(M, N, K)
    calls = {
        "w4_pack": lambda: lib.w4_pack(FAKE, N, K, FAKE, FAKE, FAKE, None),
        "w4_pack_g32": lambda: lib.w4_pack_g32(FAKE, N, K, FAKE, FAKE, FAKE, None),
        "w4_pack_codes": lambda: lib.w4_pack_codes(FAKE, N, K, FAKE, None),
        "w4_unpack": lambda: lib.w4_unpack(FAKE, N, K, FAKE, None),
        "w4_gemv": lambda: lib.w4_gemv(FAKE, FAKE, FAKE, N, K, FAKE, 1, FAKE, 0, None),
        "w4_gemv_g32": lambda: lib.w4_gemv_g32(FAKE, FAKE, FAKE, N, K, FAKE, 1, FAKE, 0, None),
        "w4a8_gemv": lambda: lib.w4a8_gemv(FAKE, FAKE, FAKE, N, K, FAKE, FAKE, FAKE, 1, FAKE, 0,
                                           None),
        "w4a8_gemv_bf16": lambda: lib.w4a8_gemv_bf16(FAKE, FAKE, FAKE, N, K, FAKE, 1, FAKE, 0,
                                                     None),
        "q8_quantize_act": lambda: lib.q8_quantize_act(FAKE, M, K, FAKE, FAKE, FAKE, None),
        "w4a8_mmq": lambda: lib.w4a8_mmq(FAKE, FAKE, FAKE, N, K, FAKE, FAKE, FAKE, M, FAKE, 0,
                                         FAKE if ws else None, ws, None),
        "w4a8_mmq_static": lambda: lib.w4a8_mmq_static(FAKE, FAKE, FAKE, N, K, FAKE, FAKE, FAKE,
                                                       M, FAKE, 0, None),
    }
    for name, call in calls.items():
        assert call() in (L.W4_ERR_CUDA, L.W4_ERR_UNSUPPORTED_DEVICE), name

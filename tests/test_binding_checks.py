"""The Python binding's argument checks, on the CPU.

The C ABI takes plain pointers and sizes, so it cannot see a plane whose
extent disagrees with (M, N, K); the binding checks every tensor's dtype,
shape and contiguity before its pointer is passed, then that all of them sit
on the current CUDA device.  With CPU tensors a call whose shapes are all
right therefore stops at the device check ("must be a CUDA tensor"), and a
call with one wrong plane stops at that plane's shape check, which names it.
No kernel is launched and the library is not needed.
"""
import pytest

torch = pytest.importorskip("torch")
w4 = pytest.importorskip("w4_quant_matmul_b200")

M, N, K = 3, 40, 512


def _weights(n=N, k=K):
    return (torch.zeros((n, k // 2), dtype=torch.uint8),
            torch.zeros((n, k // 256), dtype=torch.float16),
            torch.zeros((n, k // 256), dtype=torch.float16))


def _acts(m=M, k=K):
    return (torch.zeros((m, k), dtype=torch.int8),
            torch.zeros((m, k // 32), dtype=torch.float32),
            torch.zeros((m, k // 32), dtype=torch.int32))


def _x(m=M, k=K):
    return torch.zeros((m, k), dtype=torch.bfloat16)


def _reaches_device_check(fn, *args, **kw):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn(*args, **kw)


def _rejects_shape(name, fn, *args, **kw):
    with pytest.raises(ValueError, match=rf"^{name} must have shape"):
        fn(*args, **kw)


# argument tuples with every plane right, one of them replaceable by name
def _gemv_args(**over):
    codes, d, m = _weights()
    a = dict(codes=codes, d=d, m=m, x=_x())
    a.update(over)
    return (a["codes"], a["d"], a["m"], a["x"])


def _w4a8_args(**over):
    codes, d, m = _weights()
    qa, dx, bsum = _acts()
    a = dict(codes=codes, d=d, m=m, qa=qa, dx=dx, bsum=bsum)
    a.update(over)
    return (a["codes"], a["d"], a["m"], a["qa"], a["dx"], a["bsum"])


BAD_WEIGHTS = {
    "codes": torch.zeros((N, K // 2 - 16), dtype=torch.uint8),   # too few columns
    "d": torch.zeros((N - 1, K // 256), dtype=torch.float16),    # too few rows
    "m": torch.zeros((N, K // 256 + 1), dtype=torch.float16),    # one group too many
}
BAD_ACTS = {
    "dx": torch.zeros((M, K // 32 - 1), dtype=torch.float32),
    "bsum": torch.zeros((M + 1, K // 32), dtype=torch.int32),
}
X_FNS = [w4.w4_gemv, w4.w4a8_gemv_bf16]
A8_FNS = [w4.w4a8_gemv, w4.w4a8_mmq, w4.w4a8_mmq_static]


@pytest.mark.parametrize("fn", X_FNS)
def test_bf16_activation_calls(fn):
    _reaches_device_check(fn, *_gemv_args())
    for name, bad in BAD_WEIGHTS.items():
        _rejects_shape(name, fn, *_gemv_args(**{name: bad}))
    # y: wrong extent, wrong type for the requested output, wrong rank
    _rejects_shape("y", fn, *_gemv_args(), y=torch.zeros((M, N + 1), dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="^y must be torch.float32"):
        fn(*_gemv_args(), out_dtype=torch.float32, y=torch.zeros((M, N), dtype=torch.bfloat16))
    _rejects_shape("y", fn, *_gemv_args(), y=torch.zeros((M * N,), dtype=torch.bfloat16))
    # a caller y with no out_dtype sets the output type
    _reaches_device_check(fn, *_gemv_args(), y=torch.zeros((M, N), dtype=torch.float32))
    # a strided x is refused, not read with the wrong stride
    xt = torch.zeros((K, M), dtype=torch.bfloat16).t()
    with pytest.raises(ValueError, match="^x must be contiguous"):
        fn(*_gemv_args(x=xt))


@pytest.mark.parametrize("fn", A8_FNS)
def test_int8_activation_calls(fn):
    _reaches_device_check(fn, *_w4a8_args())
    for name, bad in {**BAD_WEIGHTS, **BAD_ACTS}.items():
        _rejects_shape(name, fn, *_w4a8_args(**{name: bad}))
    with pytest.raises(TypeError, match="^dx must be torch.float32"):
        fn(*_w4a8_args(dx=torch.zeros((M, K // 32), dtype=torch.float16)))
    _rejects_shape("y", fn, *_w4a8_args(), y=torch.zeros((M + 1, N), dtype=torch.float32),
                   out_dtype=torch.float32)


def test_group32_planes():
    x = _x()
    codes = torch.zeros((N, K // 2), dtype=torch.uint8)
    d32 = torch.zeros((N, K // 32), dtype=torch.float16)
    _reaches_device_check(w4.w4_gemv_g32, codes, d32, d32, x)
    d256 = torch.zeros((N, K // 256), dtype=torch.float16)
    _rejects_shape("d", w4.w4_gemv_g32, codes, d256, d32, x)
    _rejects_shape("m", w4.w4_gemv_g32, codes, d32, d256, x)
    # and the W4-G256 GEMV refuses group-32 planes
    _rejects_shape("d", w4.w4_gemv, codes, d32, d32, x)
    w = torch.zeros((N, K), dtype=torch.float32)
    _reaches_device_check(w4.w4_pack_g32, w)
    _rejects_shape("d", w4.w4_pack_g32, w, d=d256)


def test_mmq_workspace_is_checked():
    with pytest.raises(TypeError, match="^workspace must be torch.uint8"):
        w4.w4a8_mmq(*_w4a8_args(), workspace=torch.zeros(16, dtype=torch.int32))
    _rejects_shape("workspace", w4.w4a8_mmq, *_w4a8_args(),
                   workspace=torch.zeros((4, 16), dtype=torch.uint8))
    _reaches_device_check(w4.w4a8_mmq, *_w4a8_args(), workspace=torch.zeros(16, dtype=torch.uint8))


def test_quantiser_outputs():
    x = _x()
    _reaches_device_check(w4.q8_quantize_act, x)
    _rejects_shape("qa", w4.q8_quantize_act, x, qa=torch.zeros((M, K - 32), dtype=torch.int8))
    _rejects_shape("dx", w4.q8_quantize_act, x,
                   dx=torch.zeros((M, K // 32 + 1), dtype=torch.float32))
    _rejects_shape("bsum", w4.q8_quantize_act, x,
                   bsum=torch.zeros((M - 1, K // 32), dtype=torch.int32))


def test_pack_and_unpack_outputs():
    w = torch.zeros((N, K), dtype=torch.float32)
    _reaches_device_check(w4.w4_pack, w)
    _rejects_shape("codes", w4.w4_pack, w, codes=torch.zeros((N, K), dtype=torch.uint8))
    _rejects_shape("d", w4.w4_pack, w, d=torch.zeros((N, 1), dtype=torch.float16))
    q = torch.zeros((N, K), dtype=torch.uint8)
    _reaches_device_check(w4.w4_pack_codes, q)
    _rejects_shape("codes", w4.w4_pack_codes, q, codes=torch.zeros((N, K // 4), dtype=torch.uint8))
    codes = torch.zeros((N, K // 2), dtype=torch.uint8)
    _reaches_device_check(w4.w4_unpack, codes, K)
    _rejects_shape("codes", w4.w4_unpack, codes, K + 256)
    _rejects_shape("q", w4.w4_unpack, codes, K, q=torch.zeros((N, K // 2), dtype=torch.uint8))


def test_format_errors_are_left_to_the_library():
    # K not a multiple of the group: the group-derived extents are not checked
    # here (any extent passes) so that the library reports W4_ERR_SHAPE for K
    # itself; the call still stops at the device check on the CPU
    k = 300
    codes = torch.zeros((N, k // 2), dtype=torch.uint8)
    d = torch.zeros((N, 1), dtype=torch.float16)
    _reaches_device_check(w4.w4_gemv, codes, d, d, _x(k=k))

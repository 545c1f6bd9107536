"""Failure detection in the forms that are safe on a shared GPU: a bounded
wait that is made to run out, and host-side rejection of a workspace that is
too small.  Nothing here faults, traps or hangs a GPU: the wait that runs out
is one thread on an mbarrier phase nothing completes, limited to a few
milliseconds of GPU time, after which the kernel returns normally."""
import ctypes

import numpy as np
import pytest

import parity
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    return parity.cuda_or_skip()


@pytest.fixture(scope="module")
def lib(torch):
    from w4_quant_matmul_b200 import _lib
    return _lib.load()


def test_wait_expiry_raises_and_clears_the_error_word(torch, lib):
    from w4_quant_matmul_b200 import _lib
    assert lib.w4_check_device_error() == _lib.W4_OK  # nothing pending before
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.w4_test_wait_expiry(5_000_000, stream)  # 5 ms limit
    assert rc == _lib.W4_OK, _lib.status_string(rc)
    assert lib.w4_check_device_error() == _lib.W4_ERR_TIMEOUT
    # read once, then cleared; the context is still usable
    assert lib.w4_check_device_error() == _lib.W4_OK
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_wait_expiry_takes_about_its_limit(torch, lib):
    from w4_quant_matmul_b200 import _lib
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    rc = lib.w4_test_wait_expiry(20_000_000, ctypes.c_void_p(stream.cuda_stream))  # 20 ms
    e1.record(stream)
    assert rc == _lib.W4_OK
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert 19.0 <= ms < 1000.0, ms
    assert lib.w4_check_device_error() == _lib.W4_ERR_TIMEOUT
    assert lib.w4_check_device_error() == _lib.W4_OK


def test_mmq_rejects_a_workspace_one_byte_short(torch, lib):
    from w4_quant_matmul_b200 import _lib
    M, N, K = 256, 2560, 9728  # a split-K shape: it needs a workspace
    need = lib.w4a8_mmq_workspace_size(M, N, K)
    assert need > 0
    codes, d, m = synth.quantized_weights_direct(N, K, seed=5)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    codes_d, d_d, m_d = dev(codes), dev(d.view(np.int16)), dev(m.view(np.int16))
    qa = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    dx = torch.zeros((M, K // 32), dtype=torch.float32, device="cuda")
    S = torch.zeros((M, K // 32), dtype=torch.int32, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = (p(codes_d), p(d_d), p(m_d), N, K, p(qa), p(dx), p(S), M, p(y), _lib.W4_OUT_F32)
    assert lib.w4a8_mmq(*args, p(ws), need - 1, stream) == _lib.W4_ERR_WORKSPACE
    assert lib.w4a8_mmq(*args, None, need, stream) == _lib.W4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 7.0).all()), "a rejected call must enqueue nothing"
    # the full size is accepted
    assert lib.w4a8_mmq(*args, p(ws), need, stream) == _lib.W4_OK
    torch.cuda.synchronize()
    assert bool((y == 0.0).all())  # all-zero activations give y = 0
    assert lib.w4_check_device_error() == _lib.W4_OK

"""w4a8_mmq_static, the entry point for callers that cannot allocate device
memory (plugins whose host framework owns every device allocation,
deployments with a memory plan fixed before serving): it must give the same
product as w4a8_mmq with a caller workspace -- bit for bit, since both run the
same kernel with the same split count and a fixed-order split-K sum -- call
after call, while using only the library's static scratch.  This file is
collected last on purpose."""
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


def _inputs(torch, orc, M, N, K, seed):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=seed)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=seed + 1))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return (dev(codes), dev(d.view(np.int16)).view(torch.float16),
            dev(m.view(np.int16)).view(torch.float16), dev(qa), dev(dx), dev(S))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_static_scratch_matches_workspace_entry_point(torch, lib, orc):
    from w4_quant_matmul_b200 import _lib
    M, N, K = 256, 2560, 9728  # a split-K shape: this call needs scratch
    need = lib.w4a8_mmq_workspace_size(M, N, K)
    assert 0 < need <= _lib.W4A8_MMQ_STATIC_SCRATCH_BYTES
    codes, d, m, qa, dx, S = _inputs(torch, orc, M, N, K, seed=90)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
    rc = lib.w4a8_mmq(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa), _ptr(dx), _ptr(S), M,
                      _ptr(ref), _lib.W4_OUT_F32, _ptr(ws), need, stream)
    assert rc == _lib.W4_OK
    torch.cuda.synchronize()
    ref_np = ref.cpu().numpy()

    for call in range(2):  # the second call finds the first call's scratch contents
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.w4a8_mmq_static(_ptr(codes), _ptr(d), _ptr(m), N, K, _ptr(qa), _ptr(dx),
                                 _ptr(S), M, _ptr(y), _lib.W4_OUT_F32, stream)
        assert rc == _lib.W4_OK, (call, _lib.status_string(rc))
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        # bitwise: a stale or mixed-up partial from the previous call's scratch
        # contents would hide under a tolerance
        assert np.array_equal(got.view(np.uint32), ref_np.view(np.uint32)), f"call {call}"
        parity.assert_f32_gate(got, ref_np, f"static scratch, call {call}")
    assert lib.w4_check_device_error() == _lib.W4_OK


def test_static_scratch_rejects_oversized_shapes(torch, lib):
    from w4_quant_matmul_b200 import _lib
    # the first split-K shape whose scratch need exceeds the static array
    # (the need depends on the tile shape, so it is asked of the library)
    over = [(M, N, K) for M, N, K in [(1024, 2560, 9728), (1024, 4096, 14336),
                                      (1536, 2560, 14336), (2048, 4096, 14336)]
            if lib.w4a8_mmq_workspace_size(M, N, K) > _lib.W4A8_MMQ_STATIC_SCRATCH_BYTES]
    assert over, "no candidate shape exceeds the static scratch"
    M, N, K = over[0]
    buf = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = _ptr(buf)  # never read: the size check comes first
    rc = lib.w4a8_mmq_static(p, p, p, N, K, p, p, p, M, p, _lib.W4_OUT_F32, None)
    assert rc == _lib.W4_ERR_WORKSPACE

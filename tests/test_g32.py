"""Group-32 weights (w4_pack_g32, w4_gemv_g32) on the GPU against the oracle.

The scheme is the asymmetric int4 group-32 W4A16 format of the ROCM_OCTAVE
page ("Validation"; the sparse-attention evaluation's "Setup"), in the same
w = d*q + m form as W4-G256 with one fp16 d and m per 32 weights.

Gates: the packer is bit-exact (codes, d and m); the GEMV meets the fp32 gate
(normwise max relative error <= 2e-3, NMSE <= 1e-6) against the fp64 oracle,
and its bf16 output is the RN-bf16 of its fp32 output.  Where the W4-G256
GEMV also takes the row kernel (weight streams of 16 MB and more), W4-G256
planes repeated over the eight 32-groups of each 256-group must give the
W4-G256 output bit for bit: the same float operations in the same order.
"""
import numpy as np
import pytest

import parity
import synth

pytestmark = pytest.mark.gpu

G32 = 32


@pytest.fixture(scope="module")
def torch():
    return parity.cuda_or_skip()


@pytest.fixture(scope="module")
def w4(torch):
    import w4_quant_matmul_b200 as w4
    return w4


def _dev_u16(torch, a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dtype)


def _host_u16(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _pack_gpu(torch, w4, w):
    codes, d, m = w4.w4_pack_g32(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    return codes.cpu().numpy(), _host_u16(d), _host_u16(m)


def _planes(torch, codes, d, m):
    return (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
            _dev_u16(torch, m, torch.float16))


def _gemv(torch, w4, dev, x, out):
    y = w4.w4_gemv_g32(*dev, _dev_u16(torch, x, torch.bfloat16), out_dtype=out)
    torch.cuda.synchronize()
    return y.cpu().numpy() if out == torch.float32 else _host_u16(y)


# ---------------------------------------------------------------------------
# packer
# ---------------------------------------------------------------------------

# ragged shapes: N * K/32 groups not a multiple of the 8 groups a warp pass
# covers, K = 32 (one group), K not a multiple of 256
@pytest.mark.parametrize("N,K", [(1, 32), (37, 96), (3, 544), (256, 2560), (129, 4128)])
def test_pack_bit_exact(torch, w4, orc, N, K):
    w = synth.dense_weights(N, K, seed=N * 5 + K)
    got = _pack_gpu(torch, w4, w)
    want = orc.w4_pack(w, group=G32)
    for g, e, name in zip(got, want, ("codes", "d", "m")):
        assert np.array_equal(g, e), name


def test_pack_special_groups(torch, w4, orc):
    # constant 32-groups (d = 0), a zero minimum, exact ties, an outlier
    w = synth.dense_weights(5, 256, seed=9)
    w[0, :32] = 0.25
    w[0, 32:64] = -1.5
    w[1, 64:96] = 0.0
    w[2, :32] = 0.0
    w[2, 1] = 15.0 / 16.0
    for i, t in enumerate([0.5, 1.5, 2.5, 3.5, 12.5]):
        w[2, 2 + i] = np.float32(t / 16.0)
    w[3, 200] = 4.0
    got = _pack_gpu(torch, w4, w)
    want = orc.w4_pack(w, group=G32)
    for g, e, name in zip(got, want, ("codes", "d", "m")):
        assert np.array_equal(g, e), name


def test_pack_signed_zero_groups(torch, w4, orc):
    # 32-groups whose minimum or maximum is a zero, -0 at every position
    w = synth.signed_zero_groups(G32)
    for ww in (w, w[:, ::-1].copy()):
        got = _pack_gpu(torch, w4, ww)
        want = orc.w4_pack(ww, group=G32)
        for g, e, name in zip(got, want, ("codes", "d", "m")):
            assert np.array_equal(g, e), name


def test_pack_bit_exact_full_size(torch, w4, orc):
    N, K = synth.GEMV_SHAPES[2]  # 19456 x 2560
    w = synth.dense_weights(N, K, seed=synth.weight_seed(synth.CONFIG_BATCH1, 2) + 32)
    got = _pack_gpu(torch, w4, w)
    want = orc.w4_pack(w, group=G32)
    for g, e, name in zip(got, want, ("codes", "d", "m")):
        assert np.array_equal(g, e), name


# ---------------------------------------------------------------------------
# GEMV
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (3, 300, 2560), (8, 130, 96), (2, 40, 9728),
                                   (5, 1000, 4128), (8, 17, 32), (4, 6144, 2560)])
def test_gemv_all_outputs(torch, w4, orc, M, N, K):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=M + N + K, group=G32)
    x = synth.activations(M, K, seed=M * N + K)
    dev = _planes(torch, codes, d, m)
    y32 = _gemv(torch, w4, dev, x, torch.float32)
    y16 = _gemv(torch, w4, dev, x, torch.bfloat16)
    ref = orc.gemv(codes, d, m, x, group=G32)
    parity.assert_f32_gate(y32, ref, f"g32 M{M} N{N} K{K}")
    parity.assert_bf16_consistent(y16, y32, ref, f"g32 M{M} N{N} K{K}")


@pytest.mark.parametrize("N,K", [synth.LM_HEAD, (2560, 9728)])
def test_gemv_full_size_sampled_rows(torch, w4, orc, N, K):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=N + K + G32, group=G32)
    dev = _planes(torch, codes, d, m)
    rows = parity.sample_rows(N, count=64)
    for M in (1, 4, 8):
        x = synth.activations(M, K, seed=M + K)
        y32 = _gemv(torch, w4, dev, x, torch.float32)
        ref = np.concatenate([orc.gemv(codes, d, m, x, rows=(int(r), int(r) + 1), group=G32)
                              for r in rows], axis=1)
        parity.assert_f32_gate(y32[:, rows], ref, f"g32 {N}x{K} M{M}")


@pytest.mark.parametrize("N,K", [synth.LM_HEAD, synth.GEMV_SHAPES[2]])
def test_repeated_g256_planes_give_the_g256_output(torch, w4, N, K):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=N + 3)
    dc = torch.from_numpy(codes).cuda()
    d256, m256 = _dev_u16(torch, d, torch.float16), _dev_u16(torch, m, torch.float16)
    d32 = _dev_u16(torch, np.repeat(d, 8, axis=1), torch.float16)
    m32 = _dev_u16(torch, np.repeat(m, 8, axis=1), torch.float16)
    for M in (1, 8):
        x = _dev_u16(torch, synth.activations(M, K, seed=M + 77), torch.bfloat16)
        y256 = w4.w4_gemv(dc, d256, m256, x, out_dtype=torch.float32)
        y32 = w4.w4_gemv_g32(dc, d32, m32, x, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(y256.view(torch.int32), y32.view(torch.int32)), (N, K, M)


def test_pack_then_gemv_and_determinism(torch, w4, orc):
    M, N, K = 4, 3000, 2560
    w = synth.dense_weights(N, K, seed=41)
    x = synth.activations(M, K, seed=42)
    codes, d, m = w4.w4_pack_g32(torch.from_numpy(w).cuda())
    xd = _dev_u16(torch, x, torch.bfloat16)
    y1 = w4.w4_gemv_g32(codes, d, m, xd, out_dtype=torch.float32)
    y2 = w4.w4_gemv_g32(codes, d, m, xd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    oc, od, om = orc.w4_pack(w, group=G32)
    parity.assert_f32_gate(y1.cpu().numpy(), orc.gemv(oc, od, om, x, group=G32), "pack+gemv")
    w4.w4_check_device_error()


def test_rejects_bad_arguments(torch, w4):
    codes = torch.zeros((16, 24), dtype=torch.uint8, device="cuda")
    d = torch.zeros((16, 1), dtype=torch.float16, device="cuda")
    x = torch.zeros((1, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4Error):
        w4.w4_gemv_g32(codes, d, d, x)   # K = 48: not a multiple of 32
    codes = torch.zeros((16, 16), dtype=torch.uint8, device="cuda")
    x = torch.zeros((9, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4Error):
        w4.w4_gemv_g32(codes, d, d, x)   # M = 9
    with pytest.raises(w4.W4Error):
        w4.w4_pack_g32(torch.zeros((2, 48), dtype=torch.float32, device="cuda"),
                       d=torch.zeros((2, 1), dtype=torch.float16, device="cuda"),
                       m=torch.zeros((2, 1), dtype=torch.float16, device="cuda"))
    w4.w4_check_device_error()

"""w4a8_gemv (decode GEMV on int8 activation blocks) on the GPU against the
fp64 W4A8 oracle.

The oracle is the same definition w4a8_mmq is gated against: exact int64
block dot products P = sum q * qa, then y = sum_g sum_b dx * (d * P + m * S)
in fp64.  Gate (fp32 output): normwise max relative error <= 2e-3 and NMSE <=
1e-6; bf16 output: bitwise RN-bf16 of the same kernel's fp32 output.  Small
shapes (the shared-memory ring kernel) compare every output; the full-size
decode shapes, where the largest streams take the row kernel, compare a
seeded sample of rows at M = 1, 2, 4, 8.
"""
import numpy as np
import pytest

import parity
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    return parity.cuda_or_skip()


@pytest.fixture(scope="module")
def w4(torch):
    import w4_quant_matmul_b200 as w4
    return w4


def _dev_u16(torch, a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dtype)


def _run(torch, w4, dev, out):
    y = w4.w4a8_gemv(*dev, out_dtype=out)
    torch.cuda.synchronize()
    if out == torch.float32:
        return y.cpu().numpy()
    return y.view(torch.int16).cpu().numpy().view(np.uint16)


def _both(torch, w4, orc, codes, d, m, qa, dx, S, rows=None, what=""):
    dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
           _dev_u16(torch, m, torch.float16), torch.from_numpy(qa).cuda(),
           torch.from_numpy(dx).cuda(), torch.from_numpy(S).cuda())
    y32 = _run(torch, w4, dev, torch.float32)
    y16 = _run(torch, w4, dev, torch.bfloat16)
    if rows is None:
        ref = orc.mmq(codes, d, m, qa, dx, S)
    else:
        ref = np.concatenate([orc.mmq(codes, d, m, qa, dx, S, rows=(int(r), int(r) + 1))
                              for r in rows], axis=1)
        y32, y16 = y32[:, rows], y16[:, rows]
    parity.assert_f32_gate(y32, ref, what)
    parity.assert_bf16_consistent(y16, y32, ref, what)
    return y32


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (3, 300, 2560), (8, 130, 768),
                                   (2, 40, 9728), (5, 1000, 4096), (8, 17, 256)])
def test_small_shapes_all_outputs(torch, w4, orc, M, N, K):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=M + N + K)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=M * N + K))
    _both(torch, w4, orc, codes, d, m, qa, dx, S, what=f"M{M} N{N} K{K}")


def test_extreme_integer_products(torch, w4, orc):
    # all codes 15 and activations +-127 in every block: |P| = 32 * 15 * 127,
    # the largest block dot product the format allows, with per-block scales
    M, N, K = 8, 200, 1024
    codes = np.full((N, K // 2), 0xFF, np.uint8)
    d = synth.f32_to_f16_bits(np.full((N, K // 256), 0.01, np.float32))
    m = synth.f32_to_f16_bits(np.full((N, K // 256), -0.05, np.float32))
    sign = np.where(np.random.default_rng(3).random((M, K)) < 0.5, -1, 1)
    sign[0] = 1
    sign[1] = -1
    qa = (127 * sign).astype(np.int8)
    dx = np.random.default_rng(4).uniform(0.001, 0.05, (M, K // 32)).astype(np.float32)
    S = qa.astype(np.int32).reshape(M, K // 32, 32).sum(axis=2).astype(np.int32)
    P = orc.mmq_blockdots(codes[:1], qa)
    assert P.max() == 32 * 15 * 127 and P.min() == -32 * 15 * 127
    _both(torch, w4, orc, codes, d, m, qa, dx, S, what="extreme")


def test_zero_blocks_and_zero_scales(torch, w4, orc):
    M, N, K = 4, 260, 512
    codes, d, m = synth.quantized_weights_direct(N, K, seed=5)
    x = synth.outlier_activations(M, K, seed=6)
    x[1, :] = 0
    x[:, 64:96] = 0
    d[9] = 0
    qa, dx, S = orc.q8_quantize(x)
    _both(torch, w4, orc, codes, d, m, qa, dx, S, what="zeros")


@pytest.mark.parametrize("shape_index", range(len(synth.GEMV_SHAPES)))
def test_full_size(torch, w4, orc, shape_index):
    N, K = synth.GEMV_SHAPES[shape_index]
    _, codes, d, m = parity.packed_dense_weights(N, K, synth.weight_seed(synth.CONFIG_BATCH1,
                                                                         shape_index))
    # every row at M = 1 on all five shapes and at M = 8 on the four layer
    # shapes (every row block of the launch the benchmark times); a seeded
    # sample of rows (both ends + 256 interior) otherwise
    sampled = parity.sample_rows(N)
    for M in (1, 2, 4, 8):
        rows = None if (M == 1 or (M == 8 and shape_index < 4)) else sampled
        cfg = synth.CONFIG_BATCH1 if M == 1 else synth.CONFIG_SMALL_BATCH
        qa, dx, S = orc.q8_quantize(synth.activations(M, K, synth.act_seed(cfg, shape_index)))
        _both(torch, w4, orc, codes, d, m, qa, dx, S, rows=rows, what=f"{N}x{K} M{M}")


def test_matches_tensor_core_product(torch, w4, orc):
    # the same W4A8 product through w4a8_mmq: both within the gate of the oracle
    # and within twice the gate of each other
    M, N, K = 8, 384, 2560
    codes, d, m = synth.quantized_weights_direct(N, K, seed=11)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=12))
    dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
           _dev_u16(torch, m, torch.float16), torch.from_numpy(qa).cuda(),
           torch.from_numpy(dx).cuda(), torch.from_numpy(S).cuda())
    yg = w4.w4a8_gemv(*dev, out_dtype=torch.float32)
    ym = w4.w4a8_mmq(*dev, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = orc.mmq(codes, d, m, qa, dx, S)
    parity.assert_f32_gate(yg.cpu().numpy(), ref, "w4a8_gemv")
    parity.assert_f32_gate(ym.cpu().numpy(), ref, "w4a8_mmq")
    max_rel, nmse = parity.errors(yg.cpu().numpy(), ym.cpu().numpy().astype(np.float64))
    assert max_rel <= 2 * parity.MAX_REL and nmse <= 4 * parity.NMSE


def test_pipeline_with_gpu_quantiser_and_determinism(torch, w4, orc):
    M, N, K = 4, 6144, 2560
    codes, d, m = synth.quantized_weights_direct(N, K, seed=13)
    x = synth.activations(M, K, seed=14)
    qa_g, dx_g, S_g = w4.q8_quantize_act(_dev_u16(torch, x, torch.bfloat16))
    dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
           _dev_u16(torch, m, torch.float16), qa_g, dx_g, S_g)
    y1 = w4.w4a8_gemv(*dev, out_dtype=torch.float32)
    y2 = w4.w4a8_gemv(*dev, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    qa, dx, S = orc.q8_quantize(x)
    parity.assert_f32_gate(y1.cpu().numpy(), orc.mmq(codes, d, m, qa, dx, S), "gpu-quantised")
    w4.w4_check_device_error()


def test_rejects_bad_arguments(torch, w4):
    codes = torch.zeros((16, 128), dtype=torch.uint8, device="cuda")
    d = torch.zeros((16, 1), dtype=torch.float16, device="cuda")
    qa = torch.zeros((9, 256), dtype=torch.int8, device="cuda")
    dx = torch.zeros((9, 8), dtype=torch.float32, device="cuda")
    S = torch.zeros((9, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(w4.W4Error):
        w4.w4a8_gemv(codes, d, d, qa, dx, S)   # M = 9
    w4.w4_check_device_error()


@pytest.mark.parametrize("M,N,K", [(1, 6144, 2560), (4, 300, 9728), (8, 151936, 2560)])
def test_fused_quantiser_is_bit_identical(torch, w4, orc, M, N, K):
    # w4a8_gemv_bf16 (quantiser folded in) == q8_quantize_act + w4a8_gemv, bit
    # for bit, on both GEMV kernels (the last shape takes the row kernel)
    codes, d, m = synth.quantized_weights_direct(N, K, seed=N + K)
    x = synth.outlier_activations(M, K, seed=M + 40)
    dc, dd, dm = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
                  _dev_u16(torch, m, torch.float16))
    xd = _dev_u16(torch, x, torch.bfloat16)
    fused = w4.w4a8_gemv_bf16(dc, dd, dm, xd, out_dtype=torch.float32)
    qa, dx, S = w4.q8_quantize_act(xd)
    two_step = w4.w4a8_gemv(dc, dd, dm, qa, dx, S, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(fused.view(torch.int32), two_step.view(torch.int32))
    rows = parity.sample_rows(N, count=64)
    qa_o, dx_o, S_o = orc.q8_quantize(x)
    ref = np.concatenate([orc.mmq(codes, d, m, qa_o, dx_o, S_o, rows=(int(r), int(r) + 1))
                          for r in rows], axis=1)
    parity.assert_f32_gate(fused.cpu().numpy()[:, rows], ref, f"fused M{M} {N}x{K}")


@pytest.mark.parametrize("M,N,K", [(1, 6144, 2560), (3, 300, 768), (8, 260, 2560),
                                   (4, 2560, 9728), (8, 200, 12288), (2, 20000, 2560)])
def test_integer_block_products_bit_exact(torch, w4, orc, M, N, K):
    # The exact int32 block products of the integer core, stored by the test
    # instantiation of the same kernels and dispatch (ring kernel for the small
    # streams, row kernel for the 25.6 MB one; token passes at M = 8, K = 12288),
    # equal the oracle's int64 products element for element; y of the same call
    # is bitwise that of w4a8_gemv.
    codes, d, m = synth.quantized_weights_direct(N, K, seed=3 * M + N + K)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=M + N + 5 * K))
    dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
           _dev_u16(torch, m, torch.float16), torch.from_numpy(qa).cuda(),
           torch.from_numpy(dx).cuda(), torch.from_numpy(S).cuda())
    y, P = w4.w4a8_gemv_blockdots(*dev, out_dtype=torch.float32)
    y2 = w4.w4a8_gemv(*dev, out_dtype=torch.float32)
    torch.cuda.synchronize()
    want = orc.mmq_blockdots(codes, qa)
    got = P.cpu().numpy().astype(np.int64)
    bad = int((got != want).sum())
    assert bad == 0, f"{bad} of {want.size} block products differ"
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    parity.assert_f32_gate(y.cpu().numpy(), orc.mmq(codes, d, m, qa, dx, S), f"M{M} N{N} K{K}")


"""w4a8_mmq (tcgen05 int8 tensor cores) on the GPU against the fp64 oracle.

Gate (fp32 output): normwise max relative error <= 2e-3 and NMSE <= 1e-6
against the W4A8 oracle (exact int block dot products, fp64 scaling).  bf16
output: bitwise RN-bf16 of the same kernel's fp32 output.  Small cases span
several tiles with ragged M and N and compare every output; the full-size
prefill configurations compare all tokens on a seeded sample of weight rows.
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


def _run(torch, w4, codes, d, m, qa, dx, S, out, dev=None):
    if dev is None:
        dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
               _dev_u16(torch, m, torch.float16), torch.from_numpy(qa).cuda(),
               torch.from_numpy(dx).cuda(), torch.from_numpy(S).cuda())
    y = w4.w4a8_mmq(*dev, out_dtype=out)
    torch.cuda.synchronize()
    if out == torch.float32:
        return y.cpu().numpy()
    return y.view(torch.int16).cpu().numpy().view(np.uint16)


def _both(torch, w4, orc, codes, d, m, qa, dx, S, rows=None, what=""):
    dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
           _dev_u16(torch, m, torch.float16), torch.from_numpy(qa).cuda(),
           torch.from_numpy(dx).cuda(), torch.from_numpy(S).cuda())
    y32 = _run(torch, w4, codes, d, m, qa, dx, S, torch.float32, dev)
    y16 = _run(torch, w4, codes, d, m, qa, dx, S, torch.bfloat16, dev)
    if rows is None:
        ref = orc.mmq(codes, d, m, qa, dx, S)
    else:
        ref = np.concatenate([orc.mmq(codes, d, m, qa, dx, S, rows=(int(r), int(r) + 1))
                              for r in rows], axis=1)
        y32, y16 = y32[:, rows], y16[:, rows]
    parity.assert_f32_gate(y32, ref, what)
    parity.assert_bf16_consistent(y16, y32, ref, what)
    return y32


@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (128, 128, 512), (130, 200, 768),
                                   (300, 260, 2560), (64, 384, 4096), (257, 129, 256)])
def test_small_shapes_all_outputs(torch, w4, orc, M, N, K):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=M + N + K)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=M * N + K))
    _both(torch, w4, orc, codes, d, m, qa, dx, S, what=f"M{M} N{N} K{K}")


@pytest.mark.parametrize("scales", ["equal", "varying"])
def test_extreme_integer_products(torch, w4, orc, scales):
    # all codes 15 and all activations +-127: |P| = 32*15*127 per block, the
    # largest block dot product the format allows; token rows 0-63 reach +P
    # in every block, rows 64-95 -P in every block (the two ends of the
    # integer range a 256-group can accumulate), the rest mixed signs.
    # "varying" draws a different scale for every block.
    M, N, K = 128, 128, 1024
    codes = np.full((N, K // 2), 0xFF, np.uint8)
    d = synth.f32_to_f16_bits(np.full((N, K // 256), 0.01, np.float32))
    m = synth.f32_to_f16_bits(np.full((N, K // 256), -0.05, np.float32))
    sign = np.where(np.random.default_rng(1).random((M, K)) < 0.5, -1, 1)
    sign[:64] = 1
    sign[64:96] = -1
    qa = (127 * sign).astype(np.int8)
    if scales == "equal":
        dx = np.full((M, K // 32), 0.03, np.float32)
    else:
        dx = np.random.default_rng(2).uniform(0.001, 0.05, (M, K // 32)).astype(np.float32)
    S = qa.astype(np.int32).reshape(M, K // 32, 32).sum(axis=2).astype(np.int32)
    P = orc.mmq_blockdots(codes[:1], qa)
    assert P.max() == 32 * 15 * 127 and P.min() == -32 * 15 * 127
    _both(torch, w4, orc, codes, d, m, qa, dx, S, what="extreme")


def test_long_k(torch, w4, orc):
    # K = 16384 (64 groups): past the per-tile d/m staging limit of earlier
    # versions; every output against the oracle, split-K or not
    M, N, K = 130, 200, 16384
    codes, d, m = synth.quantized_weights_direct(N, K, seed=21)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=22))
    _both(torch, w4, orc, codes, d, m, qa, dx, S, what="K16384")


def test_zero_blocks_and_zero_scales(torch, w4, orc):
    M, N, K = 140, 130, 512
    codes, d, m = synth.quantized_weights_direct(N, K, seed=2)
    x = synth.outlier_activations(M, K, seed=3)
    x[5, :] = 0
    x[:, 32:64] = 0
    d[7] = 0
    qa, dx, S = orc.q8_quantize(x)
    _both(torch, w4, orc, codes, d, m, qa, dx, S, what="zeros")


@pytest.mark.parametrize("shape_index", range(len(synth.MMQ_SHAPES)))
def test_full_size_sampled_rows(torch, w4, orc, shape_index):
    N, K = synth.MMQ_SHAPES[shape_index]
    gemv_index = synth.GEMV_SHAPES.index((N, K))
    _, codes, d, m = parity.packed_dense_weights(N, K, synth.weight_seed(synth.CONFIG_BATCH1,
                                                                         gemv_index))
    rows = parity.sample_rows(N, count=64)
    for M in synth.MMQ_M:
        x = synth.outlier_activations(M, K, synth.act_seed(synth.CONFIG_MMQ, shape_index))
        qa, dx, S = orc.q8_quantize(x)
        _both(torch, w4, orc, codes, d, m, qa, dx, S, rows=rows, what=f"{N}x{K} M{M}")


def test_rows_are_independent_of_batch(torch, w4, orc):
    # a token's output does not depend on the other tokens in the batch
    M, N, K = 200, 256, 1024
    codes, d, m = synth.quantized_weights_direct(N, K, seed=4)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=5))
    full = _run(torch, w4, codes, d, m, qa, dx, S, torch.float32)
    for t in (0, 127, 128, 199):
        one = _run(torch, w4, codes, d, m, qa[t:t + 1].copy(), dx[t:t + 1].copy(),
                   S[t:t + 1].copy(), torch.float32)
        assert np.array_equal(one[0].view(np.uint32), full[t].view(np.uint32)), t


def test_deterministic(torch, w4, orc):
    M, N, K = 256, 512, 2560
    codes, d, m = synth.quantized_weights_direct(N, K, seed=6)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=7))
    a = _run(torch, w4, codes, d, m, qa, dx, S, torch.float32)
    b = _run(torch, w4, codes, d, m, qa, dx, S, torch.float32)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    w4.w4_check_device_error()


def test_pipeline_with_gpu_quantiser(torch, w4, orc):
    # q8_quantize_act feeding w4a8_mmq on the device, compared with the oracle
    M, N, K = 256, 384, 2560
    codes, d, m = synth.quantized_weights_direct(N, K, seed=10)
    x = synth.outlier_activations(M, K, seed=11)
    xq = _dev_u16(torch, x, torch.bfloat16)
    qa, dx, S = w4.q8_quantize_act(xq)
    y = w4.w4a8_mmq(torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
                    _dev_u16(torch, m, torch.float16), qa, dx, S, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = orc.mmq(codes, d, m, *orc.q8_quantize(x))
    parity.assert_f32_gate(y.cpu().numpy(), ref, "gpu quantiser -> mmq")


@pytest.mark.parametrize("M,N,K", [(130, 200, 768), (257, 129, 512), (64, 384, 4096),
                                   (300, 260, 2560), (256, 384, 9728)])
def test_integer_block_products_bit_exact(torch, w4, orc, M, N, K):
    # The exact int32 block products P[t][n][b], read back from the tensor
    # memory of the same kernel (its test instantiation), equal the oracle's
    # int64 products element for element: ragged M and N, several groups, and
    # (K = 9728 at M = 256) the split-K path.  The y of the same call meets the
    # float gate.
    codes, d, m = synth.quantized_weights_direct(N, K, seed=7 * M + N + K)
    qa, dx, S = orc.q8_quantize(synth.outlier_activations(M, K, seed=M + 3 * N + K))
    dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
           _dev_u16(torch, m, torch.float16), torch.from_numpy(qa).cuda(),
           torch.from_numpy(dx).cuda(), torch.from_numpy(S).cuda())
    y, P = w4.w4a8_mmq_blockdots(*dev, out_dtype=torch.float32)
    torch.cuda.synchronize()
    want = orc.mmq_blockdots(codes, qa)
    got = P.cpu().numpy().astype(np.int64)
    bad = int((got != want).sum())
    assert bad == 0, f"{bad} of {want.size} block products differ"
    parity.assert_f32_gate(y.cpu().numpy(), orc.mmq(codes, d, m, qa, dx, S), f"M{M} N{N} K{K}")
    # the product entry point gives the same y bit for bit
    y2 = w4.w4a8_mmq(*dev, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))


def test_integer_block_products_extreme(torch, w4, orc):
    # every block at the ends of the integer range, +-32*15*127
    M, N, K = 128, 128, 512
    codes = np.full((N, K // 2), 0xFF, np.uint8)
    d = synth.f32_to_f16_bits(np.full((N, K // 256), 0.01, np.float32))
    m = synth.f32_to_f16_bits(np.full((N, K // 256), -0.05, np.float32))
    qa = np.full((M, K), 127, np.int8)
    qa[64:96] = -127
    qa[96:, ::2] = -127
    dx = np.full((M, K // 32), 0.01, np.float32)
    S = qa.astype(np.int32).reshape(M, K // 32, 32).sum(axis=2).astype(np.int32)
    dev = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
           _dev_u16(torch, m, torch.float16), torch.from_numpy(qa).cuda(),
           torch.from_numpy(dx).cuda(), torch.from_numpy(S).cuda())
    _, P = w4.w4a8_mmq_blockdots(*dev, out_dtype=torch.float32)
    torch.cuda.synchronize()
    want = orc.mmq_blockdots(codes, qa)
    assert want.max() == 60960 and want.min() == -60960
    assert np.array_equal(P.cpu().numpy().astype(np.int64), want)


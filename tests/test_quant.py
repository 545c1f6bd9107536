"""q8_quantize_act on the GPU: codes, scales and block sums bit-exact against
the oracle."""
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


def _quant_gpu(torch, w4, x_bits):
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    qa, dx, S = w4.q8_quantize_act(x)
    torch.cuda.synchronize()
    return qa.cpu().numpy(), dx.cpu().numpy(), S.cpu().numpy()


def _check(torch, w4, orc, x_bits):
    got = _quant_gpu(torch, w4, x_bits)
    want = orc.q8_quantize(x_bits)
    assert np.array_equal(got[0], want[0]), "qa"
    assert np.array_equal(got[1].view(np.uint32), want[1].view(np.uint32)), "dx"
    assert np.array_equal(got[2], want[2]), "S"


@pytest.mark.parametrize("M,K", [(1, 32), (3, 96), (7, 2560), (130, 768)])
def test_quant_bit_exact_small(torch, w4, orc, M, K):
    _check(torch, w4, orc, synth.outlier_activations(M, K, seed=M + K))


def test_quant_special_blocks(torch, w4, orc):
    x = np.zeros((3, 128), np.float32)
    x[0, :7] = [127.0, 2.5, -2.5, 3.5, 0.5, 1.5, -127.0]   # unit scale, ties
    x[1, 32:64] = -0.0                                      # signed zero block
    x[1, 64] = 1e-30                                        # tiny amax
    x[2, 96:128] = np.linspace(-3, 3, 32)
    _check(torch, w4, orc, synth.f32_to_bf16_bits(x))


def test_quant_subnormal_scales(torch, w4, orc):
    # blocks whose dx = amax / 127 is subnormal (amax below 127 * 2^-126), so
    # that 1 / dx overflows: amax near 1e-38, amax at the smallest normal, and
    # blocks made only of bf16 subnormals (bf16 shares fp32's exponent range)
    rng = np.random.default_rng(41)
    x = np.zeros((4, 256), np.float32)
    x[0, :32] = rng.uniform(-1e-38, 1e-38, 32)
    x[0, 0] = 1e-38
    x[0, 32:64] = rng.uniform(-1.0, 1.0, 32) * np.float32(2.0 ** -126)
    x[1, :32] = np.float32(2.0 ** -126) * 127.0 * rng.uniform(-1, 1, 32)   # dx just normal
    x[1, 32:64] = np.float32(2.0 ** -126) * 126.0 * rng.uniform(-1, 1, 32)  # dx just subnormal
    sub = (rng.integers(1, 128, (2, 256)) * np.where(rng.random((2, 256)) < 0.5, -1, 1))
    x[2:4] = sub.astype(np.float32) * np.float32(2.0 ** -133)             # bf16 subnormals
    x[3, 64:96] = -0.0
    bits = synth.f32_to_bf16_bits(x)
    assert np.any(synth.bf16_bits_to_f32(bits[2]) != 0)
    _check(torch, w4, orc, bits)


@pytest.mark.parametrize("M,K", [(2048, 2560), (2048, 9728)])
def test_quant_bit_exact_full_size(torch, w4, orc, M, K):
    _check(torch, w4, orc, synth.outlier_activations(M, K, seed=synth.act_seed(
        synth.CONFIG_MMQ, 0 if K == 2560 else 1)))


def test_quant_near_half_integer_quotients(torch, w4, orc):
    # Every block holds its amax (which fixes dx = amax / 127) and 31 bf16
    # values on or next to half-integer multiples (k + 1/2) dx: the quotients
    # whose rounding to an integer depends on the last bit of x / dx.  The
    # codes must equal rint(fl(x / dx)) exactly.
    rng = np.random.default_rng(31)
    nblk = 4096
    x = np.zeros((nblk, 32), np.float32)
    amax = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        (2.0 ** rng.uniform(-20, 20, nblk)).astype(np.float32)))
    dx = (amax / np.float32(127.0)).astype(np.float32)
    k = rng.integers(0, 127, (nblk, 31)).astype(np.float64)
    target = ((k + 0.5) * dx[:, None].astype(np.float64)).astype(np.float32)
    bits = synth.f32_to_bf16_bits(target).astype(np.int32)
    bits += rng.integers(-2, 3, bits.shape)            # the nearest bf16 values and neighbours
    vals = synth.bf16_bits_to_f32(bits.astype(np.uint16))
    vals = np.minimum(np.abs(vals), amax[:, None]) * np.where(rng.random(vals.shape) < 0.5, -1, 1)
    x[:, 0] = amax
    x[:, 1:] = vals
    _check(torch, w4, orc, synth.f32_to_bf16_bits(x.reshape(64, -1)))

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


@pytest.mark.parametrize("M,K", [(2048, 2560), (2048, 9728)])
def test_quant_bit_exact_full_size(torch, w4, orc, M, K):
    _check(torch, w4, orc, synth.outlier_activations(M, K, seed=synth.act_seed(
        synth.CONFIG_MMQ, 0 if K == 2560 else 1)))

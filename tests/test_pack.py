"""w4_pack / w4_pack_codes / w4_unpack on the GPU: bit-exact against the
oracle, including the full-size decode shapes."""
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


def _pack_gpu(torch, w4, w):
    codes, d, m = w4.w4_pack(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    return (codes.cpu().numpy(), d.view(torch.int16).cpu().numpy().view(np.uint16),
            m.view(torch.int16).cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("N,K", [(1, 256), (3, 512), (37, 768), (256, 2560)])
def test_pack_bit_exact_small(torch, w4, orc, N, K):
    w = synth.dense_weights(N, K, seed=N * 7 + K)
    got = _pack_gpu(torch, w4, w)
    want = orc.w4_pack(w)
    for g, e, name in zip(got, want, ("codes", "d", "m")):
        assert np.array_equal(g, e), name


def test_pack_special_groups(torch, w4, orc):
    # constant groups (d = 0), exact ties, a zero minimum, negative constants
    w = synth.dense_weights(6, 512, seed=3)
    w[0, :256] = 0.25
    w[1, 256:] = 0.0
    w[2, :256] = 0.0
    w[2, 1] = 15.0 / 16.0
    for i, t in enumerate([0.5, 1.5, 2.5, 3.5, 12.5]):
        w[2, 2 + i] = np.float32(t / 16.0)
    w[3, :] = -3.0
    w[4, 10] = 5.0   # outlier widens the range
    got = _pack_gpu(torch, w4, w)
    want = orc.w4_pack(w)
    for g, e, name in zip(got, want, ("codes", "d", "m")):
        assert np.array_equal(g, e), name


def test_pack_signed_zero_groups(torch, w4, orc):
    # groups whose minimum or maximum is a zero, -0 at every position: the
    # stored d and m bits must not depend on where the -0 sits
    w = synth.signed_zero_groups(256)
    for ww in (w, w[:, ::-1].copy()):
        got = _pack_gpu(torch, w4, ww)
        want = orc.w4_pack(ww)
        for g, e, name in zip(got, want, ("codes", "d", "m")):
            assert np.array_equal(g, e), name


@pytest.mark.parametrize("shape_index", range(len(synth.GEMV_SHAPES)))
def test_pack_bit_exact_full_size(torch, w4, shape_index):
    N, K = synth.GEMV_SHAPES[shape_index]
    w, codes, d, m = parity.packed_dense_weights(N, K, synth.weight_seed(synth.CONFIG_BATCH1,
                                                                         shape_index))
    got = _pack_gpu(torch, w4, w)
    assert np.array_equal(got[0], codes)
    assert np.array_equal(got[1], d)
    assert np.array_equal(got[2], m)


@pytest.mark.parametrize("N,K", [(1, 2), (5, 6), (64, 512), (33, 1000)])
def test_pack_codes_unpack_bit_exact(torch, w4, orc, N, K):
    rng = np.random.default_rng(N + K)
    q = synth.random_codes(N, K, rng)
    qt = torch.from_numpy(q).cuda()
    codes = w4.w4_pack_codes(qt)
    back = w4.w4_unpack(codes, K)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), orc.pack_codes(q))
    assert np.array_equal(back.cpu().numpy(), q)
    b = synth.random_code_bytes(N, K, rng)
    assert np.array_equal(w4.w4_unpack(torch.from_numpy(b).cuda(), K).cpu().numpy(),
                          orc.unpack(b, K))

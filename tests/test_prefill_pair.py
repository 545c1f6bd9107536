"""The prefill pair: q8_quantize_act then w4a8_mmq on the same stream, the
product consuming the quantiser's outputs.  The product is launched
programmatically dependent on the quantiser (it requests its first code tiles
before waiting), so this checks that it never reads the activation codes,
scales or sums early: the quantiser's output buffers are poisoned before every
run, eagerly and as one CUDA graph, and the product is compared with the
oracle on the oracle's own quantisation of the same x.
"""
import numpy as np
import pytest

import parity
import synth

pytestmark = pytest.mark.gpu

M, N, K = 1024, 4096, 2560  # 256 output tiles: one K slice, no split-K workspace


@pytest.fixture(scope="module")
def torch():
    return parity.cuda_or_skip()


@pytest.fixture(scope="module")
def w4(torch):
    import w4_quant_matmul_b200 as w4
    return w4


def _dev_u16(torch, a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dtype)


def test_quantiser_then_product_reads_the_fresh_codes(torch, w4, orc):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=9300)
    x_bits = synth.outlier_activations(M, K, seed=9301)
    qa_ref, dx_ref, s_ref = orc.q8_quantize(x_bits)
    rows = parity.sample_rows(N, count=64, seed=9302)
    ref = np.concatenate([orc.mmq(codes, d, m, qa_ref, dx_ref, s_ref, rows=(int(r), int(r) + 1))
                          for r in rows], axis=1)

    dev_w = (torch.from_numpy(codes).cuda(), _dev_u16(torch, d, torch.float16),
             _dev_u16(torch, m, torch.float16))
    x = _dev_u16(torch, x_bits, torch.bfloat16)
    qa = torch.empty((M, K), dtype=torch.int8, device="cuda")
    dx = torch.empty((M, K // 32), dtype=torch.float32, device="cuda")
    s = torch.empty((M, K // 32), dtype=torch.int32, device="cuda")
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(w4.w4a8_mmq_workspace_size(M, N, K), 16), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.Stream()

    def pair():
        cur = torch.cuda.current_stream()
        w4.q8_quantize_act(x, qa=qa, dx=dx, bsum=s, stream=cur)
        w4.w4a8_mmq(*dev_w, qa, dx, s, out_dtype=torch.float32, y=y, workspace=ws, stream=cur)

    def poison():
        qa.fill_(127)
        dx.fill_(1.0e3)
        s.fill_(12345)
        y.fill_(float("nan"))
        torch.cuda.synchronize()

    def check(what):
        torch.cuda.synchronize()
        assert np.array_equal(qa.cpu().numpy(), qa_ref), what
        parity.assert_f32_gate(y.cpu().numpy()[:, rows], ref, what)

    for _ in range(2):
        poison()
        with torch.cuda.stream(stream):
            pair()
        check("eager")

    with torch.cuda.stream(stream):
        pair()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            pair()
    for _ in range(2):
        poison()
        graph.replay()
        check("graph")
    del graph
    w4.w4_check_device_error()

"""Decode GEMVs launched back to back, each one's activations the previous
one's output: the programmatic dependent launch lets a GEMV start (and stream
its weights) before the previous kernel has finished, so this checks that no
GEMV reads its activations early.  The output buffers are filled with a poison
value before every run; each link is compared with the oracle applied to the
activations the link actually received.  Both kernels are on the path: the
shared-memory ring kernel (streams below 16 MB) and the row kernel under
programmatic dependent launch (16 to 64 MB).
"""
import numpy as np
import pytest

import parity
import synth

pytestmark = pytest.mark.gpu

# x0 [1, 2560] -> 6144 -> 2560 -> 19456 -> 2560 -> 4096: every K is the
# previous N
SHAPES = [(6144, 2560), (2560, 6144), (19456, 2560), (2560, 19456), (4096, 2560)]
POISON = 1000.0


@pytest.fixture(scope="module")
def torch():
    return parity.cuda_or_skip()


@pytest.fixture(scope="module")
def w4(torch):
    import w4_quant_matmul_b200 as w4
    return w4


def _planes(torch, i, N, K):
    codes, d, m = synth.quantized_weights_direct(N, K, seed=9100 + i)
    dev = (torch.from_numpy(codes).cuda(),
           torch.from_numpy(d.view(np.int16)).cuda().view(torch.float16),
           torch.from_numpy(m.view(np.int16)).cuda().view(torch.float16))
    return (codes, d, m), dev


def _bits(torch, t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _check_links(torch, orc, host, x0_bits, ys, what):
    x_bits = x0_bits
    for i, ((codes, d, m), y) in enumerate(zip(host, ys)):
        y_bits = _bits(torch, y)
        ref = orc.gemv(codes, d, m, x_bits)
        got = synth.bf16_bits_to_f32(y_bits).astype(np.float64)
        # bf16 output: half an ulp is 2^-9 of each element
        err = np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30)
        assert err <= 1e-2, f"{what}: link {i} ({SHAPES[i]}) reads stale activations: {err:.3g}"
        x_bits = y_bits


def test_back_to_back_gemvs_read_the_previous_output(torch, w4, orc):
    host, dev = zip(*[_planes(torch, i, N, K) for i, (N, K) in enumerate(SHAPES)])
    x0_bits = synth.activations(1, SHAPES[0][1], seed=9199)
    x0 = torch.from_numpy(x0_bits.view(np.int16)).cuda().view(torch.bfloat16)
    ys = [torch.empty((1, N), dtype=torch.bfloat16, device="cuda") for N, _ in SHAPES]
    stream = torch.cuda.Stream()

    def chain():
        x = x0
        for (codes, d, m), y in zip(dev, ys):
            w4.w4_gemv(codes, d, m, x, out_dtype=torch.bfloat16, y=y,
                       stream=torch.cuda.current_stream())
            x = y

    # eager, twice, with poisoned outputs
    for _ in range(2):
        for y in ys:
            y.fill_(POISON)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            chain()
        torch.cuda.synchronize()
        _check_links(torch, orc, host, x0_bits, ys, "eager")

    # one CUDA graph of the whole chain, replayed after poisoning
    with torch.cuda.stream(stream):
        chain()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            chain()
    for _ in range(2):
        for y in ys:
            y.fill_(POISON)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        _check_links(torch, orc, host, x0_bits, ys, "graph")
    del graph
    w4.w4_check_device_error()

"""The CPU oracle against its pins (no GPU needed)."""
import json
import os
import time

import numpy as np
import pytest

import oracle_pins
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def _codes_from_rule(orc, q):
    return orc.pack_codes(q.astype(np.uint8))


def _f16(a):
    return synth.f32_to_f16_bits(np.asarray(a, np.float32))


def _bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_worked_examples(orc):
    ex = json.load(open(GOLDEN))
    g = {e["name"]: e for e in ex["gemv"]}

    e = g["ramp_codes_first_eight_ones"]
    q = (np.arange(256) % 16).reshape(1, 256)
    x = np.zeros((1, 256)); x[0, :8] = 1
    y = orc.gemv(_codes_from_rule(orc, q), _f16(e["d"]), _f16(e["m"]), _bf16(x))
    assert y.tolist() == e["y"]

    e = g["two_groups_constant_codes"]
    q = np.zeros((2, 512)); q[0] = 3; q[1, :256] = 15
    x = np.ones((1, 512)); x[0, 256:] = -2
    y = orc.gemv(_codes_from_rule(orc, q), _f16(e["d"]), _f16(e["m"]), _bf16(x))
    assert y.tolist() == e["y"]

    e = ex["q8"][0]
    x = np.full((1, 32), e["x_rest"]); x[0, :len(e["x_first"])] = e["x_first"]
    qa, dx, S = orc.q8_quantize(_bf16(x))
    assert dx[0, 0] == e["dx"]
    assert qa[0, :len(e["qa_first"])].tolist() == e["qa_first"]
    assert np.all(qa[0, len(e["qa_first"]):] == 0)
    assert S[0, 0] == e["S"]

    e = ex["mmq"][0]
    q = np.zeros((1, 256)); q[0, :32] = 2; q[0, 32:64] = 1
    qa = np.zeros((1, 256), np.int8); qa[0, :32] = 3; qa[0, 32:64] = -1
    dx = np.array([e["dx"]], np.float32)
    S = np.array([e["S"]], np.int32)
    assert np.array_equal(S[0], qa.astype(np.int32).reshape(8, 32).sum(axis=1))
    y = orc.mmq(_codes_from_rule(orc, q), _f16(e["d"]), _f16(e["m"]), qa, dx, S)
    assert y.tolist() == e["y"]


def test_worked_examples_group32(orc):
    ex = {e["name"]: e for e in json.load(open(GOLDEN))["g32"]}

    e = ex["pack_two_ramps"]
    k = np.arange(64)
    w = np.where(k < 32, (k % 16) / 16.0, -0.5 + (k % 16) / 8.0).astype(np.float32)[None, :]
    codes, d, m = orc.w4_pack(w, group=e["group"])
    assert synth.f16_bits_to_f32(d).tolist() == e["d"]
    assert synth.f16_bits_to_f32(m).tolist() == e["m"]
    assert orc.unpack(codes, 64)[0].tolist() == (k % 16).tolist()

    e = ex["gemv_two_groups"]
    q = np.where(k < 32, k % 16, 15 - k % 16)[None, :]
    x = np.ones((2, 64))
    x[1, 32:] = -1
    y = orc.gemv(_codes_from_rule(orc, q), _f16(e["d"]), _f16(e["m"]), _bf16(x),
                 group=e["group"])
    assert y.tolist() == e["y"]


def test_tiny_case_runs_fast(orc):
    codes, d, m, x = synth.tiny(0)
    t0 = time.perf_counter()
    y = orc.gemv(codes, d, m, x)
    dt = time.perf_counter() - t0
    assert y.shape == (1, 256)
    assert np.all(np.isfinite(y))
    assert dt < 1.0


def test_oracle_rejects_bad_shapes(orc):
    with pytest.raises(ValueError):
        orc.w4_pack(np.zeros((2, 300), np.float32))
    with pytest.raises(ValueError):
        orc.q8_quantize(np.zeros((2, 48), np.uint16))
    # group 32: K must be a multiple of 32; 256-wide and odd groups too
    with pytest.raises(ValueError):
        orc.w4_pack(np.zeros((2, 48), np.float32), group=32)
    with pytest.raises(ValueError):
        orc.w4_pack(np.zeros((2, 66), np.float32), group=33)
    codes, d, m = synth.quantized_weights_direct(3, 96, seed=1, group=32)
    with pytest.raises(ValueError):
        orc.gemv(codes, d, m, synth.activations(1, 100, seed=2), group=32)


def test_threads_do_not_change_results(orc):
    codes, d, m = synth.quantized_weights_direct(64, 1024, seed=31)
    x = synth.activations(2, 1024, seed=32)
    n = orc.num_threads()
    try:
        orc.set_num_threads(1)
        y1 = orc.gemv(codes, d, m, x)
        orc.set_num_threads(max(2, n))
        y2 = orc.gemv(codes, d, m, x)
    finally:
        orc.set_num_threads(n)
    assert np.array_equal(y1, y2)

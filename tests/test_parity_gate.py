"""The parity gates themselves, on the CPU: they accept an exact match and
reject each kind of miss the GPU tests rely on them to catch."""
import numpy as np
import pytest

import parity
import synth


def _ref(shape=(3, 50), seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def test_f32_gate_accepts_fp32_rounding_of_the_oracle():
    ref = _ref()
    parity.assert_f32_gate(ref.astype(np.float32), ref)


def test_f32_gate_rejects_one_large_error():
    ref = _ref()
    y = ref.copy()
    y[1, 7] += 3e-3 * np.abs(ref).max()  # above the max-rel bound of 2e-3
    with pytest.raises(AssertionError):
        parity.assert_f32_gate(y, ref)


def test_f32_gate_rejects_many_small_errors():
    # every element off by 1.5e-3 of its own magnitude: max-rel passes,
    # NMSE = 2.25e-6 does not
    ref = _ref()
    y = ref * (1 + 1.5e-3)
    max_rel, nmse = parity.errors(y, ref)
    assert max_rel <= parity.MAX_REL and nmse > parity.NMSE
    with pytest.raises(AssertionError):
        parity.assert_f32_gate(y, ref)


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_f32_gate_rejects_non_finite_outputs(bad):
    ref = _ref()
    y = ref.copy()
    y[0, 0] = bad
    with pytest.raises(AssertionError):
        parity.assert_f32_gate(y, ref)


def test_f32_gate_rejects_a_shape_mismatch():
    ref = _ref((4, 10))
    with pytest.raises(AssertionError):
        parity.assert_f32_gate(ref[:1], ref)      # one row broadcast over four
    with pytest.raises(AssertionError):
        parity.assert_f32_gate(ref.T, ref.T.T)


def test_f32_gate_on_an_all_zero_reference():
    ref = np.zeros((2, 8))
    parity.assert_f32_gate(np.zeros((2, 8), np.float32), ref)
    with pytest.raises(AssertionError):
        parity.assert_f32_gate(np.full((2, 8), 1e-2), ref)


def test_bf16_consistency():
    ref = _ref()
    y32 = ref.astype(np.float32)
    y16 = parity.bf16_bits_rn(y32)
    parity.assert_bf16_consistent(y16, y32, ref)
    off = y16.copy()
    off[2, 3] ^= 1  # one bf16 ulp away from RN of the fp32 output
    with pytest.raises(AssertionError):
        parity.assert_bf16_consistent(off, y32, ref)
    # RN of an fp32 output that is itself far from the oracle
    far32 = (ref * 1.05).astype(np.float32)
    with pytest.raises(AssertionError):
        parity.assert_bf16_consistent(parity.bf16_bits_rn(far32), far32, ref)


def test_bf16_rounding_is_round_to_nearest_even():
    # 1 + 2^-8 lies halfway between the bf16 neighbours 1 and 1 + 2^-7: even -> 1
    bits = parity.bf16_bits_rn(np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], np.float32))
    assert synth.bf16_bits_to_f32(bits).tolist() == [1.0, 1.0 + 2.0 ** -6]


def test_sample_rows():
    rows = parity.sample_rows(151936, count=64)
    assert np.all(np.diff(rows) > 0) and rows[0] == 0 and rows[-1] == 151935
    assert set(range(32)) <= set(rows.tolist()) and len(rows) == 64 + 64
    small = parity.sample_rows(40)
    assert small.tolist() == list(range(40))

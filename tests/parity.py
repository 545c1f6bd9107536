"""Shared helpers for the GPU parity tests: the float-output gate, bf16 bit
helpers and cached full-size inputs (drawn by ``synth``, quantised by the
oracle: no expected value ever comes from the CUDA path)."""
from __future__ import annotations

import functools

import numpy as np
import pytest

import synth

# Float-output acceptance (fp32 output mode): normwise max relative error and
# normalised mean squared error against the fp64 oracle.
MAX_REL = 2e-3
NMSE = 1e-6


def cuda_or_skip():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch


def errors(y: np.ndarray, ref: np.ndarray):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    # equal shapes: broadcasting must never stand in for an element-wise match
    assert y.shape == ref.shape, f"shape {y.shape} against the oracle's {ref.shape}"
    scale = np.abs(ref).max()
    max_rel = np.abs(y - ref).max() / scale if scale > 0 else np.abs(y).max()
    den = (ref ** 2).sum()
    nmse = ((y - ref) ** 2).sum() / den if den > 0 else ((y - ref) ** 2).sum()
    return float(max_rel), float(nmse)


def assert_f32_gate(y, ref, what=""):
    max_rel, nmse = errors(y, ref)
    assert max_rel <= MAX_REL and nmse <= NMSE, f"{what}: max_rel={max_rel:.3e} nmse={nmse:.3e}"
    return max_rel, nmse


def bf16_bits_rn(a: np.ndarray) -> np.ndarray:
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def assert_bf16_consistent(y_bf16_bits: np.ndarray, y_f32: np.ndarray, ref: np.ndarray, what=""):
    """bf16 output == RN-bf16 of the same kernel's fp32 output, and close to
    the oracle (one bf16 rounding plus the fp32 gate)."""
    want = bf16_bits_rn(y_f32)
    mism = int((y_bf16_bits != want).sum())
    assert mism == 0, f"{what}: {mism} bf16 outputs differ from RN(fp32 output)"
    yb = synth.bf16_bits_to_f32(y_bf16_bits).astype(np.float64)
    scale = np.abs(ref).max()
    assert np.all(np.abs(yb - ref) <= 2.0 ** -8 * np.abs(ref) + MAX_REL * scale), what


def sample_rows(N: int, count: int = 256, seed: int = 1234) -> np.ndarray:
    """Sorted row sample: both ends plus seeded random interior rows."""
    rng = np.random.default_rng(seed)
    edge = min(N, 32)
    rows = set(range(edge)) | set(range(max(0, N - edge), N))
    if N > 2 * edge:
        rows |= set(rng.choice(np.arange(edge, N - edge), size=min(count, N - 2 * edge),
                               replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int64)


@functools.lru_cache(maxsize=3)
def packed_dense_weights(N: int, K: int, seed: int):
    """fp32 N(0, 0.02) weights and their oracle quantisation."""
    import oracle
    w = synth.dense_weights(N, K, seed)
    codes, d, m = oracle.get().w4_pack(w)
    return w, codes, d, m

"""Seeded synthetic inputs for the W4-G256 matmul workloads.

This module only draws random numbers and rounds them to the storage types the
format fixes (bf16 activations, fp16 scales and mins, random code bytes).  It
holds none of the method's arithmetic: no quantiser, no packing rule, no
product.  Both the CPU oracle and the CUDA path are fed from here, and nothing
here imports either of them.

Workloads (a 4B-class decoder with hidden size 2560, as in the pages' batch-1
decode campaign and pp 256-2048 prefill sweep):

* ``TINY``      W[256,512] codes iid U{0..15}, d ~ U(0.001, 0.02) -> fp16,
                m ~ U(-0.1, 0) -> fp16, x ~ N(0,1) -> bf16, M = 1, seed 0.
* ``GEMV_SHAPES`` the five (N, K) decode shapes; weights fp32 N(0, 0.02) that the
                caller quantises with its own w4_pack; x ~ N(0,1) -> bf16.
* ``SMALL_BATCH`` M in {2, 4, 8} over the same shapes.
* ``MMQ``       M in {256, 512, 1024, 2048} x (N,K) in {(19456,2560),
                (2560,9728)}; activations N(0,1) with an iid Bernoulli(0.01)
                mask scaled x20, -> bf16.
* ``CHAIN``     36 layers x the four layer shapes + the lm_head, M = 1.

Seeds: weights of (config c, shape s) use 1000*c + s, activations use
1000*c + s + 500; the tiny case uses seed 0 for everything.
"""
from __future__ import annotations

import numpy as np

GROUP = 256
BLOCK = 32

GEMV_SHAPES = [(6144, 2560), (2560, 4096), (19456, 2560), (2560, 9728), (151936, 2560)]
LAYER_SHAPES = GEMV_SHAPES[:4]
LM_HEAD = GEMV_SHAPES[4]
SMALL_BATCH = [2, 4, 8]
MMQ_SHAPES = [(19456, 2560), (2560, 9728)]
MMQ_M = [256, 512, 1024, 2048]
CHAIN_LAYERS = 36

CONFIG_TINY = 1
CONFIG_BATCH1 = 2
CONFIG_SMALL_BATCH = 3
CONFIG_MMQ = 4
CONFIG_CHAIN = 5


def weight_seed(config: int, shape_index: int) -> int:
    return 1000 * config + shape_index


def act_seed(config: int, shape_index: int) -> int:
    return 1000 * config + shape_index + 500


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the bits.
    Inputs are finite (the generators below never produce NaN or inf)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def f16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float32)


def random_code_bytes(N: int, K: int, rng: np.random.Generator) -> np.ndarray:
    """Packed code bytes [N, K/2]: uniform bytes, so every 4-bit code is iid
    U{0..15} whatever the nibble order."""
    return rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)


def random_codes(N: int, K: int, rng: np.random.Generator) -> np.ndarray:
    """Unpacked codes [N, K], iid U{0..15}, one per byte."""
    return rng.integers(0, 16, size=(N, K), dtype=np.uint8)


def uniform_f16_bits(shape, lo: float, hi: float, rng: np.random.Generator) -> np.ndarray:
    v = rng.uniform(lo, hi, size=shape).astype(np.float32)
    return f32_to_f16_bits(v)


def normal_bf16_bits(shape, rng: np.random.Generator, std: float = 1.0) -> np.ndarray:
    v = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    return f32_to_bf16_bits(v)


def dense_weights(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    """fp32 W[N,K] ~ N(0, std^2), to be quantised by min/max per group."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal(size=(N, K), dtype=np.float32) * np.float32(std)


def activations(M: int, K: int, seed: int) -> np.ndarray:
    """bf16 bits x[M,K] ~ N(0,1)."""
    return normal_bf16_bits((M, K), np.random.default_rng(seed))


def outlier_activations(M: int, K: int, seed: int, p: float = 0.01,
                        scale: float = 20.0) -> np.ndarray:
    """bf16 bits x[M,K] ~ N(0,1), each element independently scaled by
    ``scale`` with probability ``p`` (sparse large outliers)."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal(size=(M, K), dtype=np.float32)
    mask = rng.random(size=(M, K)) < p
    v = np.where(mask, v * np.float32(scale), v).astype(np.float32)
    return f32_to_bf16_bits(v)


def tiny(seed: int = 0):
    """The tiny GEMV case: (codes[256,256] packed bytes, d[256,2], m[256,2]
    fp16 bits, x[1,512] bf16 bits)."""
    N, K = 256, 512
    rng = np.random.default_rng(seed)
    codes = random_code_bytes(N, K, rng)
    d = uniform_f16_bits((N, K // GROUP), 0.001, 0.02, rng)
    m = uniform_f16_bits((N, K // GROUP), -0.1, 0.0, rng)
    x = normal_bf16_bits((1, K), rng)
    return codes, d, m, x


def quantized_weights_direct(N: int, K: int, seed: int, group: int = GROUP):
    """Directly drawn W4 weights (no quantiser involved): uniform code bytes,
    d ~ U(0.001, 0.02), m ~ U(-0.1, 0), as fp16 bits, one d and m per `group`
    weights (256: W4-G256; 32: the group-32 variant)."""
    rng = np.random.default_rng(seed)
    codes = random_code_bytes(N, K, rng)
    d = uniform_f16_bits((N, K // group), 0.001, 0.02, rng)
    m = uniform_f16_bits((N, K // group), -0.1, 0.0, rng)
    return codes, d, m

def signed_zero_groups(group: int) -> np.ndarray:
    """fp32 rows of one weight group each whose minimum or maximum is zero,
    with -0.0 at different positions (first, middle, last, all, every other
    slot) and ramps that end or start on -0.0: the inputs on which a min/max
    search can return either zero."""
    rows = []
    z = np.zeros(group, np.float32)
    a = z.copy(); a[0] = -0.0; rows.append(a)
    a = z.copy(); a[group // 2] = -0.0; rows.append(a)
    a = z.copy(); a[-1] = -0.0; rows.append(a)
    rows.append(np.full(group, -0.0, np.float32))
    a = z.copy(); a[1::2] = -0.0; rows.append(a)
    a = np.linspace(0.0, 0.5, group).astype(np.float32); a[0] = -0.0; rows.append(a)
    a = np.linspace(0.0, 0.5, group).astype(np.float32)[::-1].copy(); a[-1] = -0.0
    rows.append(a)
    a = np.linspace(-0.5, 0.0, group).astype(np.float32); a[-1] = -0.0; rows.append(a)
    a = np.linspace(-0.5, 0.0, group).astype(np.float32)[::-1].copy(); a[0] = -0.0
    rows.append(a)
    return np.stack(rows)

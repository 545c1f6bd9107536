"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises ``AssertionError`` when the
oracle disagrees with what the format definition and the mathematics fix:
hand-built bytes, closed forms, invariants, special cases that reduce to a
library routine (numpy integer/fp64 matmul), and brute force on tiny inputs.
They are shared by ``test_oracle.py`` (the real oracle must pass all) and
``test_mutation.py`` (every planted-mistake build must fail at least one).

Worked values cited here come from the format definition (W4-G256: groups of
256, 4-bit codes, fp16 d and m, w = d*q + m; int8 activation blocks of 32 with
an fp32 scale and an int32 block sum, the Q8_1-style layout of the hipfire
MMQ prefill article, "What changed" list) and the readings recorded in the
design notes (nibble order, rounding).
"""
from __future__ import annotations

import numpy as np

import synth

GROUP = 256
BLOCK = 32


def _f16(v) -> np.ndarray:
    return synth.f32_to_f16_bits(np.asarray(v, np.float32))


def _bf16(v) -> np.ndarray:
    return synth.f32_to_bf16_bits(np.asarray(v, np.float32))


def _dequant_dense(o, codes, d, m, K, group=GROUP):
    """Dense fp64 W[N,K] from the oracle's own unpack (pinned separately) and
    numpy broadcasting of the per-group d, m."""
    q = o.unpack(codes, K).astype(np.float64)
    dd = synth.f16_bits_to_f32(d).astype(np.float64)
    mm = synth.f16_bits_to_f32(m).astype(np.float64)
    N = q.shape[0]
    G = K // group
    W = q.reshape(N, G, group) * dd[:, :, None] + mm[:, :, None]
    return W.reshape(N, K)


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

def pin_pack_hand_bytes(o):
    # byte j holds k = 2j in bits 0-3 and k = 2j+1 in bits 4-7
    q = np.array([[1, 2, 15, 0, 0, 15, 10, 5]], np.uint8)
    got = o.pack_codes(q)
    assert got.tolist() == [[0x21, 0x0F, 0xF0, 0x5A]], [hex(b) for b in got[0]]
    back = o.unpack(np.array([[0xA5, 0x3C]], np.uint8), 4)
    assert back.tolist() == [[5, 10, 12, 3]], back


def pin_pack_roundtrip(o):
    rng = np.random.default_rng(11)
    q = synth.random_codes(7, 512, rng)
    assert np.array_equal(o.unpack(o.pack_codes(q), 512), q)
    b = synth.random_code_bytes(5, 768, rng)
    assert np.array_equal(o.pack_codes(o.unpack(b, 768)), b)


# --------------------------------------------------------------------------
# weight quantiser
# --------------------------------------------------------------------------

def pin_wpack_constant_group(o):
    w = np.full((2, 512), 0.75, np.float32)
    w[1, 256:] = -1.5
    codes, d, m = o.w4_pack(w)
    assert np.all(codes == 0)
    assert np.all(d == 0)  # fp16 +0
    assert synth.f16_bits_to_f32(m).tolist() == [[0.75, 0.75], [0.75, -1.5]]


def pin_wpack_grid_idempotent(o):
    # weights already on the grid w = d*q + m with min code 0 and max code 15,
    # d = k * 2^-10 and m = j * 2^-6 (exact in fp16 and in fp32 arithmetic),
    # re-quantise to the same (q, d, m).
    rng = np.random.default_rng(5)
    N, K = 6, 512
    G = K // GROUP
    dk = rng.integers(1, 64, size=(N, G))
    mj = rng.integers(-32, 32, size=(N, G))
    dval = (dk * 2.0 ** -10).astype(np.float32)
    mval = (mj * 2.0 ** -6).astype(np.float32)
    q = synth.random_codes(N, K, rng)
    q[:, 0::GROUP] = 0
    q[:, 1::GROUP] = 15
    w = (q.reshape(N, G, GROUP).astype(np.float32) * dval[:, :, None]
         + mval[:, :, None]).reshape(N, K).astype(np.float32)
    codes, d, m = o.w4_pack(w)
    assert np.array_equal(synth.f16_bits_to_f32(d), dval)
    assert np.array_equal(synth.f16_bits_to_f32(m), mval)
    assert np.array_equal(o.unpack(codes, K), q)


def pin_wpack_ties_to_even(o):
    # group min 0, max 15/16 -> d = 1/16 exactly, m = 0; (w - m)/d lands on
    # x.5 exactly for these weights: 0.5->0, 1.5->2, 2.5->2, 3.5->4, 12.5->12
    w = np.zeros((1, 256), np.float32)
    w[0, 1] = 15.0 / 16.0
    ties = [0.5, 1.5, 2.5, 3.5, 12.5, 13.5]
    for i, t in enumerate(ties):
        w[0, 2 + i] = np.float32(t / 16.0)
    codes, d, m = o.w4_pack(w)
    assert synth.f16_bits_to_f32(d)[0, 0] == 1.0 / 16.0
    assert synth.f16_bits_to_f32(m)[0, 0] == 0.0
    q = o.unpack(codes, 256)[0]
    assert q[0] == 0 and q[1] == 15
    assert q[2:2 + len(ties)].tolist() == [0, 2, 2, 4, 12, 14], q[2:2 + len(ties)]


def pin_wpack_error_bound(o):
    # |w - (d*q + m)| <= d/2 plus the rounding of d and m to fp16
    N, K = 16, 1024
    w = synth.dense_weights(N, K, seed=77)
    codes, d, m = o.w4_pack(w)
    q = o.unpack(codes, K).astype(np.float64)
    dd = synth.f16_bits_to_f32(d).astype(np.float64)
    mm = synth.f16_bits_to_f32(m).astype(np.float64)
    G = K // GROUP
    wg = w.reshape(N, G, GROUP).astype(np.float64)
    deq = q.reshape(N, G, GROUP) * dd[:, :, None] + mm[:, :, None]
    mn = wg.min(axis=2)
    mx = wg.max(axis=2)
    slack = np.abs(mm - mn) + 15.0 * np.abs(dd - (mx - mn) / 15.0) + 1e-7
    err = np.abs(wg - deq)
    assert np.all(err <= dd[:, :, None] / 2 + slack[:, :, None]), float(err.max())
    # the extreme weights of each group map to codes 0 and 15
    assert np.all(q.reshape(N, G, GROUP).min(axis=2) == 0)
    assert np.all(q.reshape(N, G, GROUP).max(axis=2) == 15)


def _check_signed_zero(o, group):
    w = synth.signed_zero_groups(group)
    codes, d, m = o.w4_pack(w, group=group)
    # a zero minimum is stored as +0, whatever the position of the -0
    mf = synth.f16_bits_to_f32(m)
    assert np.all(m[mf == 0] == 0), m[:, 0].tolist()
    # the same values in another order give the same d and m: flip each row
    codes2, d2, m2 = o.w4_pack(w[:, ::-1].copy(), group=group)
    assert np.array_equal(d, d2) and np.array_equal(m, m2)
    # groups of zeros alone: d = +0, m = +0, codes 0
    assert np.all(d[:5] == 0) and np.all(m[:5] == 0) and np.all(codes[:5] == 0)
    # zero maximum with a negative minimum: d from the range, m = the minimum
    assert synth.f16_bits_to_f32(m)[7, 0] == np.float32(-0.5)
    assert synth.f16_bits_to_f32(d)[7, 0] == synth.f16_bits_to_f32(
        synth.f32_to_f16_bits(np.float32(0.5) / np.float32(15.0)))


def pin_wpack_signed_zero(o):
    _check_signed_zero(o, GROUP)


def pin_g32_wpack_signed_zero(o):
    _check_signed_zero(o, 32)


# --------------------------------------------------------------------------
# activation quantiser
# --------------------------------------------------------------------------

def pin_q8_unit_scale_ties(o):
    # amax = 127 -> dx = 1 exactly; codes are rint(x), ties to even
    vals = [127.0, 2.5, -2.5, 3.5, -3.5, 0.5, 1.5, -0.5, 100.0, -127.0]
    x = np.zeros((1, 32), np.float32)
    x[0, :len(vals)] = vals
    qa, dx, S = o.q8_quantize(_bf16(x))
    assert dx[0, 0] == 1.0
    assert qa[0, :len(vals)].tolist() == [127, 2, -2, 4, -4, 0, 2, 0, 100, -127]
    assert S[0, 0] == int(qa[0].astype(np.int64).sum())


def pin_q8_grid_codes(o):
    # x = j * (amax/127) with amax/127 = 2^-3 exactly reproduces j
    rng = np.random.default_rng(9)
    j = rng.integers(-127, 128, size=(3, 64))
    j[:, 0] = 127
    j[:, 32] = -127
    x = (j * 2.0 ** -3).astype(np.float32)
    qa, dx, S = o.q8_quantize(_bf16(x))
    assert np.all(dx == np.float32(2.0 ** -3))
    assert np.array_equal(qa.astype(np.int64), j)
    assert np.array_equal(S.astype(np.int64), j.reshape(3, 2, 32).sum(axis=2))


def pin_q8_zero_block(o):
    x = np.zeros((2, 64), np.float32)
    x[1, 40] = -3.0
    qa, dx, S = o.q8_quantize(_bf16(x))
    assert dx[0].tolist() == [0.0, 0.0] and dx[1, 0] == 0.0
    assert np.all(qa[0] == 0) and np.all(qa[1, :32] == 0)
    assert S[0].tolist() == [0, 0] and S[1, 0] == 0
    assert qa[1, 40] == -127 and S[1, 1] == -127


def pin_q8_reconstruction(o):
    # random activations with outliers: |x - dx*qa| <= dx/2 (+ fp32 slack),
    # the amax element gets +-127, S is the integer sum
    x = synth.outlier_activations(4, 1024, seed=3)
    qa, dx, S = o.q8_quantize(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64).reshape(4, 32, 32)
    qb = qa.astype(np.int64).reshape(4, 32, 32)
    dd = dx.astype(np.float64)[:, :, None]
    assert np.all(np.abs(xf - dd * qb) <= dd * (0.5 + 1e-5))
    amax_pos = np.argmax(np.abs(xf), axis=2)
    picked = np.take_along_axis(qb, amax_pos[:, :, None], axis=2)[:, :, 0]
    assert np.all(np.abs(picked) == 127)
    assert np.array_equal(S.astype(np.int64), qb.sum(axis=2))
    assert np.allclose(dx.astype(np.float64), np.abs(xf).max(axis=2) / 127.0, rtol=1e-7)


# --------------------------------------------------------------------------
# GEMV (dequantised weights x bf16 activations, fp64)
# --------------------------------------------------------------------------

def pin_gemv_library_matmul(o):
    # brute force on tiny shapes: numpy fp64 matmul of the dense dequantised
    # matrix, built by broadcasting (not by the oracle's k loop)
    codes, d, m = synth.quantized_weights_direct(40, 768, seed=21)
    x = synth.activations(3, 768, seed=22)
    y = o.gemv(codes, d, m, x)
    W = _dequant_dense(o, codes, d, m, 768)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ W.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), float(np.abs(y - ref).max())


def pin_gemv_constant_codes(o):
    # all codes c: y = sum_g (d_g*c + m_g) * sum_{k in g} x_k
    rng = np.random.default_rng(4)
    N, K = 5, 1024
    G = K // GROUP
    for c in (0, 7, 15):
        codes = np.full((N, K // 2), c | (c << 4), np.uint8)
        d = synth.uniform_f16_bits((N, G), 0.001, 0.02, rng)
        m = synth.uniform_f16_bits((N, G), -0.1, 0.0, rng)
        x = synth.normal_bf16_bits((2, K), rng)
        y = o.gemv(codes, d, m, x)
        xs = synth.bf16_bits_to_f32(x).astype(np.float64).reshape(2, G, GROUP).sum(axis=2)
        dd = synth.f16_bits_to_f32(d).astype(np.float64)
        mm = synth.f16_bits_to_f32(m).astype(np.float64)
        ref = xs @ (dd * c + mm).T
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), (c, float(np.abs(y - ref).max()))


def pin_gemv_zero_scale(o):
    # d = 0: y = sum_g m_g * sum_{k in g} x_k whatever the codes
    rng = np.random.default_rng(6)
    N, K = 4, 768
    G = K // GROUP
    codes = synth.random_code_bytes(N, K, rng)
    d = np.zeros((N, G), np.uint16)
    m = synth.uniform_f16_bits((N, G), -0.1, 0.1, rng)
    x = synth.normal_bf16_bits((1, K), rng)
    y = o.gemv(codes, d, m, x)
    xs = synth.bf16_bits_to_f32(x).astype(np.float64).reshape(1, G, GROUP).sum(axis=2)
    ref = xs @ synth.f16_bits_to_f32(m).astype(np.float64).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def pin_gemv_integer_exact(o):
    # d = 1, m = 0 and integer activations: exactly the int64 product q @ x
    rng = np.random.default_rng(8)
    N, K = 9, 512
    q = synth.random_codes(N, K, rng)
    codes = o.pack_codes(q)
    one = np.full((N, K // GROUP), 0x3C00, np.uint16)  # fp16 1.0
    zero = np.zeros((N, K // GROUP), np.uint16)
    xi = rng.integers(-8, 9, size=(2, K))
    y = o.gemv(codes, one, zero, _bf16(xi.astype(np.float32)))
    ref = xi.astype(np.int64) @ q.astype(np.int64).T
    assert np.array_equal(y, ref.astype(np.float64))


def pin_gemv_linearity(o):
    rng = np.random.default_rng(10)
    codes, d, m = synth.quantized_weights_direct(6, 512, seed=12)
    x1 = rng.standard_normal((1, 512))
    x2 = rng.standard_normal((1, 512))
    a, b = 0.75, -2.0
    y = o.gemv_f64(codes, d, m, a * x1 + b * x2)
    ref = a * o.gemv_f64(codes, d, m, x1) + b * o.gemv_f64(codes, d, m, x2)
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-11)


def pin_gemv_row_window(o):
    codes, d, m = synth.quantized_weights_direct(20, 512, seed=13)
    x = synth.activations(2, 512, seed=14)
    full = o.gemv(codes, d, m, x)
    part = o.gemv(codes, d, m, x, rows=(5, 17))
    assert np.array_equal(part, full[:, 5:17])


# --------------------------------------------------------------------------
# W4A8 product
# --------------------------------------------------------------------------

def pin_mmq_blockdots_int_matmul(o):
    rng = np.random.default_rng(15)
    N, K, M = 7, 512, 3
    q = synth.random_codes(N, K, rng)
    codes = o.pack_codes(q)
    qa = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    P = o.mmq_blockdots(codes, qa)
    ref = np.einsum("tbi,nbi->tnb", qa.astype(np.int64).reshape(M, K // BLOCK, BLOCK),
                    q.astype(np.int64).reshape(N, K // BLOCK, BLOCK))
    assert np.array_equal(P, ref)


def pin_mmq_integer_gemm(o):
    # dx = 1, d = 1, m = 0: y is the integer GEMM qa @ q^T, exactly
    rng = np.random.default_rng(16)
    N, K, M = 6, 768, 4
    q = synth.random_codes(N, K, rng)
    codes = o.pack_codes(q)
    qa = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    dx = np.ones((M, K // BLOCK), np.float32)
    S = qa.astype(np.int32).reshape(M, K // BLOCK, BLOCK).sum(axis=2).astype(np.int32)
    one = np.full((N, K // GROUP), 0x3C00, np.uint16)
    zero = np.zeros((N, K // GROUP), np.uint16)
    y = o.mmq(codes, one, zero, qa, dx, S)
    ref = qa.astype(np.int64) @ q.astype(np.int64).T
    assert np.array_equal(y, ref.astype(np.float64))


def pin_mmq_matches_gemv_on_dequantised_acts(o):
    # cross-oracle invariant: the W4A8 product on (qa, dx, S) equals the
    # dequantised-weight product on x' = dx * qa (fp64), min term included
    codes, d, m = synth.quantized_weights_direct(12, 1024, seed=17)
    x = synth.outlier_activations(5, 1024, seed=18)
    qa, dx, S = o.q8_quantize(x)
    y = o.mmq(codes, d, m, qa, dx, S)
    xprime = (qa.astype(np.float64).reshape(5, 32, 32)
              * dx.astype(np.float64)[:, :, None]).reshape(5, 1024)
    ref = o.gemv_f64(codes, d, m, xprime)
    scale = np.abs(ref).max()
    assert np.abs(y - ref).max() <= 1e-12 * scale, float(np.abs(y - ref).max() / scale)


def pin_mmq_row_window(o):
    codes, d, m = synth.quantized_weights_direct(10, 512, seed=19)
    qa, dx, S = o.q8_quantize(synth.activations(3, 512, seed=20))
    full = o.mmq(codes, d, m, qa, dx, S)
    part = o.mmq(codes, d, m, qa, dx, S, rows=(2, 9))
    assert np.array_equal(part, full[:, 2:9])


# --------------------------------------------------------------------------
# group-32 variant (one d and m per 32 weights; "ROCM_OCTAVE", "Validation":
# W4A16 int4 group 32, asymmetric)
# --------------------------------------------------------------------------

G32 = 32


def pin_g32_wpack_constant_groups(o):
    # every 32-group constant, a different constant per group: codes 0, d = +0,
    # m = the constant, group by group (a 256-wide or shifted group fails)
    N, K = 2, 256
    vals = (np.arange(N * (K // G32)).reshape(N, K // G32) * 0.125 - 1.0).astype(np.float32)
    w = np.repeat(vals, G32, axis=1)
    codes, d, m = o.w4_pack(w, group=G32)
    assert d.shape == (N, K // G32) and np.all(d == 0) and np.all(codes == 0)
    assert np.array_equal(synth.f16_bits_to_f32(m), vals)


def pin_g32_wpack_grid_idempotent(o):
    # weights on the grid w = d*q + m of each 32-group (codes 0 and 15 present,
    # d = k * 2^-10, m = j * 2^-6, exact in fp16 and fp32) re-quantise to
    # themselves
    rng = np.random.default_rng(25)
    N, K = 5, 512
    G = K // G32
    dval = (rng.integers(1, 64, size=(N, G)) * 2.0 ** -10).astype(np.float32)
    mval = (rng.integers(-32, 32, size=(N, G)) * 2.0 ** -6).astype(np.float32)
    q = synth.random_codes(N, K, rng)
    q[:, 0::G32] = 0
    q[:, 7::G32] = 15
    w = (q.reshape(N, G, G32).astype(np.float32) * dval[:, :, None]
         + mval[:, :, None]).reshape(N, K).astype(np.float32)
    codes, d, m = o.w4_pack(w, group=G32)
    assert np.array_equal(synth.f16_bits_to_f32(d), dval)
    assert np.array_equal(synth.f16_bits_to_f32(m), mval)
    assert np.array_equal(o.unpack(codes, K), q)


def pin_g32_wpack_error_bound(o):
    # |w - (d*q + m)| <= d/2 plus the fp16 rounding of d and m, per 32-group;
    # each group's extreme weights take codes 0 and 15
    N, K = 12, 512
    w = synth.dense_weights(N, K, seed=78)
    codes, d, m = o.w4_pack(w, group=G32)
    G = K // G32
    q = o.unpack(codes, K).astype(np.float64).reshape(N, G, G32)
    dd = synth.f16_bits_to_f32(d).astype(np.float64)
    mm = synth.f16_bits_to_f32(m).astype(np.float64)
    wg = w.reshape(N, G, G32).astype(np.float64)
    deq = q * dd[:, :, None] + mm[:, :, None]
    mn, mx = wg.min(axis=2), wg.max(axis=2)
    slack = np.abs(mm - mn) + 15.0 * np.abs(dd - (mx - mn) / 15.0) + 1e-7
    assert np.all(np.abs(wg - deq) <= dd[:, :, None] / 2 + slack[:, :, None])
    assert np.all(q.min(axis=2) == 0) and np.all(q.max(axis=2) == 15)


def pin_g32_gemv_library_matmul(o):
    # brute force: numpy fp64 matmul of the dense matrix built by broadcasting
    # one (d, m) pair over each 32 weights
    N, K = 33, 320
    codes, d, m = synth.quantized_weights_direct(N, K, seed=31, group=G32)
    x = synth.activations(4, K, seed=32)
    y = o.gemv(codes, d, m, x, group=G32)
    W = _dequant_dense(o, codes, d, m, K, group=G32)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ W.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), float(np.abs(y - ref).max())


def pin_g32_gemv_constant_codes(o):
    # all codes c: y = sum_g (d_g*c + m_g) * sum_{k in 32-group g} x_k
    rng = np.random.default_rng(33)
    N, K = 4, 256
    G = K // G32
    for c in (0, 9, 15):
        codes = np.full((N, K // 2), c | (c << 4), np.uint8)
        d = synth.uniform_f16_bits((N, G), 0.001, 0.02, rng)
        m = synth.uniform_f16_bits((N, G), -0.1, 0.0, rng)
        x = synth.normal_bf16_bits((3, K), rng)
        y = o.gemv(codes, d, m, x, group=G32)
        xs = synth.bf16_bits_to_f32(x).astype(np.float64).reshape(3, G, G32).sum(axis=2)
        dd = synth.f16_bits_to_f32(d).astype(np.float64)
        mm = synth.f16_bits_to_f32(m).astype(np.float64)
        ref = xs @ (dd * c + mm).T
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), (c, float(np.abs(y - ref).max()))


def pin_g32_gemv_reduces_to_g256(o):
    # W4-G256 planes repeated over the eight 32-groups of each 256-group are
    # the same matrix: the group-32 product equals the (separately pinned)
    # W4-G256 product bit for bit, same weights in the same k order
    N, K = 9, 768
    codes, d, m = synth.quantized_weights_direct(N, K, seed=34)
    x = synth.activations(2, K, seed=35)
    y256 = o.gemv(codes, d, m, x)
    y32 = o.gemv(codes, np.repeat(d, 8, axis=1), np.repeat(m, 8, axis=1), x, group=G32)
    assert np.array_equal(y32, y256)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]

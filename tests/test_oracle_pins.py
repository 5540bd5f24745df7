"""Pins of the fp64 oracle to things other than itself.

Each test ties an oracle function to something the definition or mathematics
fixes: numpy's IEEE binary16 conversions (library routines), exhaustive
enumeration of the Q4 nibble positions, exactly representable quantiser
inputs, hand-derived worked blocks (tests/golden), closed forms (one-hot and
all-ones activations) and exact rational brute force on tiny matrices.  A
plausible slip in the oracle (swapped nibbles, a transposed operand, a dropped
-8 offset, a wrong rounding rule, a mis-strided scale plane) fails at least
one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import synth
from tests.conftest import read_golden


# ------------------------------------------------------------------ fp16 ----
def test_half_to_double_exhaustive_vs_numpy():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_double_to_half_vs_numpy_rne():
    r = np.random.default_rng(7)
    vals = np.concatenate([
        r.standard_normal(20000) * 10.0 ** r.integers(-9, 6, 20000),
        # exact midpoints between neighbouring fp16 values (ties to even)
        (np.arange(0, 4096, dtype=np.float64) + 0.5) * 2.0 ** -24,          # subnormal ties
        (1024 + np.arange(0, 1024, dtype=np.float64) + 0.5) * 2.0 ** -10,  # [1, 2) ties
        [65504.0, 65519.99, 65520.0, 70000.0, 2.0 ** -25, 2.0 ** -25 * 1.0000001,
         2.0 ** -14, 2.0 ** -14 * (1 - 2.0 ** -12), 0.0, -0.0, 1e-30, -65520.0],
    ])
    vals = np.concatenate([vals, -vals])
    ours = oracle.double_to_half(vals)
    with np.errstate(over="ignore"):          # overflow to inf is one of the cases checked
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------ quantisers ----
def _expect_exact(fmt, N, nb, e, seed):
    """w = d*v with d = 2^-e and one element per block at +-levels."""
    r = np.random.default_rng(seed)
    lv = {2: 1, 3: 3, 4: 7, 5: 15, 6: 31, 8: 127}[fmt]
    v = r.integers(-lv, lv + 1, size=(N, nb, 32))
    pin = r.integers(0, 32, size=(N, nb))
    sgn = r.choice([-1, 1], size=(N, nb))
    for n in range(N):
        for j in range(nb):
            v[n, j, pin[n, j]] = sgn[n, j] * lv
    d = 2.0 ** -e
    w = (v * d).astype(np.float32).reshape(N, nb * 32)
    assert np.array_equal(w.astype(np.float64), (v * d).reshape(N, nb * 32))
    return v, w, d


@pytest.mark.parametrize("e", [4, 7, 10, 15, 18, 24])
def test_quantize_q4_exact_representable(e):
    N, nb = 5, 9                       # K = 288: ldS = 16 (padded from 9)
    v, w, d = _expect_exact(4, N, nb, e, 100 + e)
    codes, scales = oracle.quantize_q4(w)
    assert scales.shape == (N, 16)
    # fp16 bits of 2^-e: normal (e <= 14) or subnormal, from the format definition
    dbits = ((15 - e) << 10) if e <= 14 else (1 << (24 - e))
    assert np.all(scales[:, :nb] == dbits) and np.all(scales[:, nb:] == 0)
    q = v + 8
    lo, hi = q[..., :16], q[..., 16:]
    assert np.array_equal(codes.reshape(N, nb, 16), (lo | (hi << 4)).astype(np.uint8))
    assert np.array_equal(oracle.dequantize_q4(codes, scales), w.astype(np.float64))


def _q6_planes(q):
    """Q6 code rows [N, nb, 32] -> the packed row [N, 3K/4], from the format
    text: the low-nibble plane (Q4's layout) then the 2-bit plane."""
    N, nb, _ = q.shape
    lo = (q[..., :16] & 15) | ((q[..., 16:] & 15) << 4)
    h = q >> 4
    hi = h[..., 0:8] | (h[..., 8:16] << 2) | (h[..., 16:24] << 4) | (h[..., 24:32] << 6)
    return np.concatenate([lo.reshape(N, nb * 16), hi.reshape(N, nb * 8)], axis=1).astype(np.uint8)


def _q5_planes(q):
    """Q5 code rows [N, nb, 32] -> the packed row [N, 5K/8], from the format
    text: the low-nibble plane then the 1-bit plane."""
    N, nb, _ = q.shape
    lo = (q[..., :16] & 15) | ((q[..., 16:] & 15) << 4)
    top = (q >> 4).reshape(N, nb, 8, 4)        # [.., p, i] = element i + 4p
    hi = np.zeros((N, nb, 4), dtype=np.int64)
    for p in range(8):
        hi |= top[:, :, p, :] << p
    return np.concatenate([lo.reshape(N, nb * 16), hi.reshape(N, nb * 4)], axis=1).astype(np.uint8)


def _two_bit_plane(q):
    """[N, nb, 32] -> [N, nb, 8]: byte i holds bits 0-1 of elements i, i+8,
    i+16, i+24 in bits 0-1, 2-3, 4-5, 6-7."""
    q = q & 3
    return q[..., 0:8] | (q[..., 8:16] << 2) | (q[..., 16:24] << 4) | (q[..., 24:32] << 6)


def _q2_planes(q):
    """Q2 code rows [N, nb, 32] -> the packed row [N, K/4], from the format text."""
    N, nb, _ = q.shape
    return _two_bit_plane(q).reshape(N, nb * 8).astype(np.uint8)


def _q3_planes(q):
    """Q3 code rows [N, nb, 32] -> the packed row [N, 3K/8], from the format
    text: the 2-bit plane of the low bits, then the 1-bit plane of bit 2."""
    N, nb, _ = q.shape
    top = (q >> 2).reshape(N, nb, 8, 4)        # [.., p, i] = element i + 4p
    hi = np.zeros((N, nb, 4), dtype=np.int64)
    for p in range(8):
        hi |= top[:, :, p, :] << p
    return np.concatenate([_two_bit_plane(q).reshape(N, nb * 8), hi.reshape(N, nb * 4)],
                          axis=1).astype(np.uint8)


@pytest.mark.parametrize("e", [4, 7, 10, 15, 18, 24])
def test_quantize_q2_exact_representable(e):
    N, nb = 4, 10                      # K = 320: ldS = 16 (padded from 10)
    v, w, d = _expect_exact(2, N, nb, e, 700 + e)
    codes, scales = oracle.quantize_q2(w)
    assert codes.shape == (N, 320 // 4) and scales.shape == (N, 16)
    dbits = ((15 - e) << 10) if e <= 14 else (1 << (24 - e))
    assert np.all(scales[:, :nb] == dbits) and np.all(scales[:, nb:] == 0)
    assert np.array_equal(codes, _q2_planes(v + 2))
    assert np.array_equal(oracle.dequantize_q2(codes, scales), w.astype(np.float64))


@pytest.mark.parametrize("e", [4, 7, 10, 15, 18, 24])
def test_quantize_q3_exact_representable(e):
    N, nb = 4, 12                      # K = 384: ldS = 16 (padded from 12)
    v, w, d = _expect_exact(3, N, nb, e, 600 + e)
    codes, scales = oracle.quantize_q3(w)
    assert codes.shape == (N, 3 * 384 // 8) and scales.shape == (N, 16)
    dbits = ((15 - e) << 10) if e <= 14 else (1 << (24 - e))
    assert np.all(scales[:, :nb] == dbits) and np.all(scales[:, nb:] == 0)
    assert np.array_equal(codes, _q3_planes(v + 4))
    assert np.array_equal(oracle.dequantize_q3(codes, scales), w.astype(np.float64))


@pytest.mark.parametrize("e", [4, 7, 10, 15, 18, 24])
def test_quantize_q5_exact_representable(e):
    N, nb = 4, 12                      # K = 384: ldS = 16 (padded from 12)
    v, w, d = _expect_exact(5, N, nb, e, 500 + e)
    codes, scales = oracle.quantize_q5(w)
    assert codes.shape == (N, 5 * 384 // 8) and scales.shape == (N, 16)
    dbits = ((15 - e) << 10) if e <= 14 else (1 << (24 - e))
    assert np.all(scales[:, :nb] == dbits) and np.all(scales[:, nb:] == 0)
    assert np.array_equal(codes, _q5_planes(v + 16))
    assert np.array_equal(oracle.dequantize_q5(codes, scales), w.astype(np.float64))


@pytest.mark.parametrize("e", [4, 7, 10, 15, 18, 24])
def test_quantize_q6_exact_representable(e):
    N, nb = 4, 10                      # K = 320: ldS = 16 (padded from 10)
    v, w, d = _expect_exact(6, N, nb, e, 300 + e)
    codes, scales = oracle.quantize_q6(w)
    assert codes.shape == (N, 3 * 320 // 4) and scales.shape == (N, 16)
    dbits = ((15 - e) << 10) if e <= 14 else (1 << (24 - e))
    assert np.all(scales[:, :nb] == dbits) and np.all(scales[:, nb:] == 0)
    assert np.array_equal(codes, _q6_planes(v + 32))
    assert np.array_equal(oracle.dequantize_q6(codes, scales), w.astype(np.float64))


@pytest.mark.parametrize("e", [4, 7, 10, 16, 24])
def test_quantize_q8_exact_representable(e):
    N, nb = 3, 8
    v, w, d = _expect_exact(8, N, nb, e, 200 + e)
    # the scale a/127 = d is exact only when d*127 is exact in fp32 (always here)
    codes, scales = oracle.quantize_q8(w)
    dbits = ((15 - e) << 10) if e <= 14 else (1 << (24 - e))
    assert np.all(scales[:, :nb] == dbits)
    assert np.array_equal(codes.reshape(N, nb, 32), v.astype(np.int8))
    assert np.array_equal(oracle.dequantize_q8(codes, scales), w.astype(np.float64))


def test_quantize_zero_block_and_tiny_scale():
    w = np.zeros((2, 64), dtype=np.float32)
    w[1, 32:] = 1e-9                      # a/7 rounds to fp16 zero
    c4, s4 = oracle.quantize_q4(w)
    assert np.all(s4 == 0) and np.all(c4 == 0x88)
    c8, s8 = oracle.quantize_q8(w)
    assert np.all(s8 == 0) and np.all(c8 == 0)
    c6, s6 = oracle.quantize_q6(w)        # q = 32: low nibbles 0, top bits 2 (0b10)
    assert np.all(s6 == 0) and np.all(c6[:, :32] == 0) and np.all(c6[:, 32:] == 0xAA)
    c5, s5 = oracle.quantize_q5(w)        # q = 16: low nibbles 0, every top bit 1
    assert np.all(s5 == 0) and np.all(c5[:, :32] == 0) and np.all(c5[:, 32:] == 0xFF)
    c3, s3 = oracle.quantize_q3(w)        # q = 4: low 2 bits 0, every bit 2 set
    assert np.all(s3 == 0) and np.all(c3[:, :16] == 0) and np.all(c3[:, 16:] == 0xFF)
    c2, s2 = oracle.quantize_q2(w)        # q = 2: every 2-bit field 0b10
    assert np.all(s2 == 0) and np.all(c2 == 0xAA)


def test_quantize_round_half_away_and_ties():
    d = 2.0 ** -6
    w = np.zeros((1, 32), dtype=np.float32)
    w[0, 0] = 7 * d                       # absmax -> d exactly
    w[0, 1] = -7 * d                      # the symmetric tie of the absmax
    w[0, 2] = 2.5 * d                     # half: away from zero -> 3 (even rule: 2)
    w[0, 3] = -2.5 * d                    # -> -3
    w[0, 4] = 0.5 * d                     # -> 1
    w[0, 5] = -0.5 * d                    # -> -1
    w[0, 6] = 1.49 * d                    # -> 1
    codes, scales = oracle.quantize_q4(w)
    q = [(codes[0, i % 16] >> (4 * (i // 16))) & 15 for i in range(32)]
    assert q[:7] == [15, 1, 11, 5, 9, 7, 9]
    assert scales[0, 0] == (15 - 6) << 10


def test_quantize_rejects_overflow_and_nonfinite():
    w = np.zeros((1, 32), dtype=np.float32)
    w[0, 0] = 7 * 65600.0                 # a/7 > 65504 -> fp16 overflow
    with pytest.raises(ValueError):
        oracle.quantize_q4(w)
    w[0, 0] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize_q8(w)


def test_quantize_nearest_grid_point():
    """Away from ties, every dequantised weight is the nearest point of its
    block's grid d*{-8..7} (Q4) / d*{-127..127} (Q8) to w."""
    w = synth.weights_f32(synth.key(0, 90, 0, 0, 0), 16, 256)
    c4, s4 = oracle.quantize_q4(w)
    c8, s8 = oracle.quantize_q8(w)
    c6, s6 = oracle.quantize_q6(w)
    c5, s5 = oracle.quantize_q5(w)
    c3, s3 = oracle.quantize_q3(w)
    c2, s2 = oracle.quantize_q2(w)
    for fmt, codes, scales, lv in ((4, c4, s4, (-8, 7)), (8, c8, s8, (-127, 127)),
                                   (6, c6, s6, (-32, 31)), (5, c5, s5, (-16, 15)),
                                   (3, c3, s3, (-4, 3)), (2, c2, s2, (-2, 1))):
        deq = {2: oracle.dequantize_q2, 3: oracle.dequantize_q3, 4: oracle.dequantize_q4,
               5: oracle.dequantize_q5, 6: oracle.dequantize_q6,
               8: oracle.dequantize_q8}[fmt](codes, scales)
        d = oracle.half_to_double(scales[:, :8]).repeat(32, axis=1)
        grid = np.arange(lv[0], lv[1] + 1)[None, None, :] * d[..., None]
        nearest = np.abs(grid - w.astype(np.float64)[..., None]).min(axis=-1)
        assert np.all(np.abs(deq - w) <= nearest + 1e-18)


@pytest.mark.parametrize("fmt,levels,zero", [(4, 7, 8), (8, 127, 0), (6, 31, 32), (5, 15, 16),
                                             (3, 3, 4), (2, 1, 2)])
def test_quantize_scale_and_codes_recomputed_in_numpy(fmt, levels, zero):
    """Random blocks (N(0, 0.02) rows scaled over six decades, some with
    outliers): the oracle's stored fp16 scale bits equal
    fp16(fp32(absmax) / fp32(levels)) computed by numpy's IEEE fp32 divide and
    nearest-even fp16 conversion, and every dequantised weight equals
    d * (q - zero) with q = clamp(round_half_away(fp32(w) / fp32(d)) + zero)
    -- the quotient an IEEE fp32 division by the *stored* scale.  Dividing by
    the unrounded fp32 scale instead changes codes on random blocks and fails
    here.  (Dividing in fp64 gives the same codes: the stored scale has 11
    significant bits, so (k + 1/2) * d is an fp32 number and no fp32 quotient
    of an fp32 w can round onto a tie the exact quotient misses.)"""
    rng = np.random.default_rng([fmt, 4242])
    N, K = 96, 512
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w *= (10.0 ** rng.uniform(-4, 2, size=(N, 1))).astype(np.float32)
    out = rng.random((N, K)) < 0.01
    w[out] *= np.float32(9.0)
    quant = {2: oracle.quantize_q2, 3: oracle.quantize_q3, 4: oracle.quantize_q4,
             5: oracle.quantize_q5, 6: oracle.quantize_q6, 8: oracle.quantize_q8}[fmt]
    deq = {2: oracle.dequantize_q2, 3: oracle.dequantize_q3, 4: oracle.dequantize_q4,
           5: oracle.dequantize_q5, 6: oracle.dequantize_q6, 8: oracle.dequantize_q8}[fmt]
    codes, scales = quant(w)
    blocks = w.reshape(N, K // 32, 32)
    amax = np.abs(blocks).max(axis=2).astype(np.float32)
    d16 = (amax / np.float32(levels)).astype(np.float16)          # fp32 divide, RNE to fp16
    assert np.array_equal(scales[:, :K // 32], d16.view(np.uint16))
    d32 = d16.astype(np.float32)
    q = np.zeros(blocks.shape, dtype=np.float64)
    nz = d32 != 0
    quot = (blocks / np.where(nz, d32, np.float32(1))[..., None]).astype(np.float32)
    r = np.sign(quot) * np.floor(np.abs(quot.astype(np.float64)) + 0.5)   # half away from zero
    lo, hi = (-127, 127) if fmt == 8 else (0, 2 * zero - 1)
    q = np.clip(r + zero, lo, hi)
    q = np.where(nz[..., None], q, zero)
    want = (d32.astype(np.float64)[..., None] * (q - zero)).reshape(N, K)
    got = deq(codes, scales)
    assert np.array_equal(got, want)


# ---------------------------------------------------------- golden files ----
@pytest.mark.parametrize("name,fmt", [("q4_block_worked.txt", 4), ("q8_block_worked.txt", 8),
                                      ("q6_block_worked.txt", 6), ("q5_block_worked.txt", 5),
                                      ("q3_block_worked.txt", 3), ("q2_block_worked.txt", 2)])
def test_golden_worked_block(name, fmt):
    g = read_golden(name)
    v = np.array([int(t) for t in g["w_over_d"]])
    d = 2.0 ** int(g["d_log2"][0])
    w = (v * d).astype(np.float32)[None, :]
    x = np.array([float(t) for t in g["x"]], dtype=np.float16).view(np.uint16)[None, :]
    if fmt == 4:
        codes, scales = oracle.quantize_q4(w)
        assert [int(b) for b in codes[0]] == [int(t, 16) for t in g["packed"]]
        q = [(codes[0, i % 16] >> (4 * (i // 16))) & 15 for i in range(32)]
        y, a = oracle.gemv_q4(codes, scales, x)
    elif fmt in (2, 3, 5, 6):
        quant, deq, gemv = {
            2: (oracle.quantize_q2, oracle.dequantize_q2, oracle.gemv_q2),
            3: (oracle.quantize_q3, oracle.dequantize_q3, oracle.gemv_q3),
            5: (oracle.quantize_q5, oracle.dequantize_q5, oracle.gemv_q5),
            6: (oracle.quantize_q6, oracle.dequantize_q6, oracle.gemv_q6)}[fmt]
        codes, scales = quant(w)
        assert [int(b) for b in codes[0]] == [int(t, 16) for t in g["packed"]]
        zero = {2: 2, 3: 4, 5: 16, 6: 32}[fmt]
        q = [int(round(v)) + zero for v in deq(codes, scales)[0] / d]
        y, a = gemv(codes, scales, x)
    else:
        codes, scales = oracle.quantize_q8(w)
        q = [int(c) for c in codes[0]]
        y, a = oracle.gemv_q8(codes, scales, x)
    assert q == [int(t) for t in g["codes"]]
    assert scales[0, 0] == int(g["scale_bits"][0], 16)
    assert y[0, 0] == float(g["y"][0])
    assert a[0, 0] == float(g["abs_sum"][0])


def _pack_from_format_text(fmt, q):
    """32 codes of one block -> its bytes, by the plane packers above (written
    from the format text, independent of the oracle)."""
    b = np.array(q, dtype=np.int64).reshape(1, 1, 32)
    if fmt == 4:
        return [int(c) for c in (b[0, 0, :16] | (b[0, 0, 16:] << 4))]
    pack = {2: _q2_planes, 3: _q3_planes, 5: _q5_planes, 6: _q6_planes}[fmt]
    return [int(c) for c in pack(b)[0]]


@pytest.mark.parametrize("name,fmt", [("q2_block_worked.txt", 2), ("q3_block_worked.txt", 3),
                                      ("q4_block_worked.txt", 4), ("q5_block_worked.txt", 5),
                                      ("q6_block_worked.txt", 6), ("q8_block_worked.txt", 8)])
def test_golden_worked_block_is_self_consistent(name, fmt):
    """Each hand-derived fixture agrees with itself, without the oracle: the
    codes are w/d plus the format's zero point, the largest |w/d| equals the
    format's level count (so absmax / levels is the stated power of two), the
    scale bits are that power of two in fp16, the packed bytes follow the
    layout stated in the header, and y and sum |w x| are the exact sums."""
    from fractions import Fraction
    g = read_golden(name)
    levels, zero = {2: (1, 2), 3: (3, 4), 4: (7, 8), 5: (15, 16), 6: (31, 32), 8: (127, 0)}[fmt]
    v = [int(t) for t in g["w_over_d"]]
    assert len(v) == 32 and int(g["N"][0]) == 1 and int(g["K"][0]) == 32
    assert max(abs(t) for t in v) == levels and all(-levels - (fmt != 8) <= t <= levels for t in v)
    q = [t + zero for t in v]
    assert q == [int(t) for t in g["codes"]]
    e = int(g["d_log2"][0])
    assert -14 <= e <= 15 and int(g["scale_bits"][0], 16) == (e + 15) << 10   # normal fp16 2^e
    if fmt != 8:
        assert _pack_from_format_text(fmt, q) == [int(t, 16) for t in g["packed"]]
        assert len(g["packed"]) == {2: 8, 3: 12, 4: 16, 5: 20, 6: 24}[fmt]
    x = [Fraction(float(np.float16(t))) for t in g["x"]]
    assert all(float(np.float16(t)) == float(t) for t in g["x"])             # x exact in fp16
    d = Fraction(2) ** e
    assert Fraction(g["y"][0]) == d * sum(vi * xi for vi, xi in zip(v, x))
    assert Fraction(g["abs_sum"][0]) == d * sum(abs(vi * xi) for vi, xi in zip(v, x))


# ---------------------------------------------------------- nibble order ----
def test_q4_nibble_order_exhaustive():
    """Every (position, code) of a 1x32 block: element i < 16 lives in the low
    nibble of byte i, element i >= 16 in the high nibble of byte i-16."""
    one = np.array([0x3C00], dtype=np.uint16)          # fp16 1.0
    scales = np.zeros((1, 8), dtype=np.uint16)
    scales[0, 0] = one[0]
    for p in range(32):
        xo = np.zeros((1, 32), dtype=np.uint16)
        xo[0, p] = one[0]
        for c in range(16):
            q = [8] * 32
            q[p] = c
            packed = np.array([[q[i] | (q[i + 16] << 4) for i in range(16)]], dtype=np.uint8)
            deq = oracle.dequantize_q4(packed, scales)
            expect = np.zeros((1, 32))
            expect[0, p] = c - 8
            assert np.array_equal(deq, expect), (p, c)
            y, _ = oracle.gemv_q4(packed, scales, xo)
            assert y[0, 0] == c - 8


def test_q6_bit_positions_exhaustive():
    """Every (position, code) of a 1x32 Q6 block: element i's low 4 bits are
    in the low (i < 16) or high (i >= 16) nibble of byte i mod 16, its top 2
    bits in bit pair i // 8 of byte K/2 + i mod 8."""
    one = np.array([0x3C00], dtype=np.uint16)          # fp16 1.0
    scales = np.zeros((1, 8), dtype=np.uint16)
    scales[0, 0] = one[0]
    for p in range(32):
        xo = np.zeros((1, 32), dtype=np.uint16)
        xo[0, p] = one[0]
        for c in range(64):
            q = [32] * 32
            q[p] = c
            lo = [(q[i] & 15) | ((q[i + 16] & 15) << 4) for i in range(16)]
            hi = [(q[i] >> 4) | ((q[i + 8] >> 4) << 2) | ((q[i + 16] >> 4) << 4) |
                  ((q[i + 24] >> 4) << 6) for i in range(8)]
            packed = np.array([lo + hi], dtype=np.uint8)
            deq = oracle.dequantize_q6(packed, scales)
            expect = np.zeros((1, 32))
            expect[0, p] = c - 32
            assert np.array_equal(deq, expect), (p, c)
            y, _ = oracle.gemv_q6(packed, scales, xo)
            assert y[0, 0] == c - 32


def test_q5_bit_positions_exhaustive():
    """Every (position, code) of a 1x32 Q5 block: element i's low 4 bits as
    Q4's, its top bit in bit i // 4 of byte K/2 + i mod 4."""
    one = np.array([0x3C00], dtype=np.uint16)          # fp16 1.0
    scales = np.zeros((1, 8), dtype=np.uint16)
    scales[0, 0] = one[0]
    for p in range(32):
        xo = np.zeros((1, 32), dtype=np.uint16)
        xo[0, p] = one[0]
        for c in range(32):
            q = [16] * 32
            q[p] = c
            lo = [(q[i] & 15) | ((q[i + 16] & 15) << 4) for i in range(16)]
            hi = [sum((q[i + 4 * b] >> 4) << b for b in range(8)) for i in range(4)]
            packed = np.array([lo + hi], dtype=np.uint8)
            deq = oracle.dequantize_q5(packed, scales)
            expect = np.zeros((1, 32))
            expect[0, p] = c - 16
            assert np.array_equal(deq, expect), (p, c)
            y, _ = oracle.gemv_q5(packed, scales, xo)
            assert y[0, 0] == c - 16


def test_q3_bit_positions_exhaustive():
    """Every (position, code) of a 1x32 Q3 block: element i's low 2 bits in
    bit pair i // 8 of byte i mod 8, its bit 2 in bit i // 4 of byte K/4 + i mod 4."""
    one = np.array([0x3C00], dtype=np.uint16)          # fp16 1.0
    scales = np.zeros((1, 8), dtype=np.uint16)
    scales[0, 0] = one[0]
    for p in range(32):
        xo = np.zeros((1, 32), dtype=np.uint16)
        xo[0, p] = one[0]
        for c in range(8):
            q = [4] * 32
            q[p] = c
            lo = [(q[i] & 3) | ((q[i + 8] & 3) << 2) | ((q[i + 16] & 3) << 4) |
                  ((q[i + 24] & 3) << 6) for i in range(8)]
            hi = [sum((q[i + 4 * b] >> 2) << b for b in range(8)) for i in range(4)]
            packed = np.array([lo + hi], dtype=np.uint8)
            deq = oracle.dequantize_q3(packed, scales)
            expect = np.zeros((1, 32))
            expect[0, p] = c - 4
            assert np.array_equal(deq, expect), (p, c)
            y, _ = oracle.gemv_q3(packed, scales, xo)
            assert y[0, 0] == c - 4


def test_q2_bit_positions_exhaustive():
    """Every (position, code) of a 1x32 Q2 block: element i in bit pair
    i // 8 of byte i mod 8."""
    one = np.array([0x3C00], dtype=np.uint16)          # fp16 1.0
    scales = np.zeros((1, 8), dtype=np.uint16)
    scales[0, 0] = one[0]
    for p in range(32):
        xo = np.zeros((1, 32), dtype=np.uint16)
        xo[0, p] = one[0]
        for c in range(4):
            q = [2] * 32
            q[p] = c
            packed = np.array([[q[i] | (q[i + 8] << 2) | (q[i + 16] << 4) | (q[i + 24] << 6)
                                for i in range(8)]], dtype=np.uint8)
            deq = oracle.dequantize_q2(packed, scales)
            expect = np.zeros((1, 32))
            expect[0, p] = c - 2
            assert np.array_equal(deq, expect), (p, c)
            y, _ = oracle.gemv_q2(packed, scales, xo)
            assert y[0, 0] == c - 2


def test_scale_plane_stride_and_block_index():
    """Scale (n, j) scales exactly block j of row n, with rows ldS apart."""
    N, K = 3, 96                                       # ldS = 8 > K/32 = 3
    codes = np.full((N, K // 2), 0x99, dtype=np.uint8)  # every code 9 -> v = 1
    scales = np.zeros((N, 8), dtype=np.uint16)
    for n in range(N):
        for j in range(3):
            scales[n, j] = oracle.double_to_half(float(10 * n + j + 1))
        scales[n, 3:] = 0x7C00                          # padding must be ignored (inf)
    deq = oracle.dequantize_q4(codes, scales)
    for n in range(N):
        for k in range(K):
            assert deq[n, k] == 10 * n + k // 32 + 1
    c8 = np.ones((N, K), dtype=np.int8)
    deq8 = oracle.dequantize_q8(c8, scales)
    assert np.array_equal(deq8, deq)
    # Q6 code 33 (v = 1): low nibbles 1, top bits 2 in every pair
    c6 = np.concatenate([np.full((N, K // 2), 0x11, dtype=np.uint8),
                         np.full((N, K // 4), 0xAA, dtype=np.uint8)], axis=1)
    assert np.array_equal(oracle.dequantize_q6(c6, scales), deq)
    # Q5 code 17 (v = 1): low nibbles 1, every top bit 1
    c5 = np.concatenate([np.full((N, K // 2), 0x11, dtype=np.uint8),
                         np.full((N, K // 8), 0xFF, dtype=np.uint8)], axis=1)
    assert np.array_equal(oracle.dequantize_q5(c5, scales), deq)
    # Q3 code 5 (v = 1): low 2 bits 1 in every pair, every bit 2 set
    c3 = np.concatenate([np.full((N, K // 4), 0x55, dtype=np.uint8),
                         np.full((N, K // 8), 0xFF, dtype=np.uint8)], axis=1)
    assert np.array_equal(oracle.dequantize_q3(c3, scales), deq)
    # Q2 code 3 (v = 1) in every pair
    assert np.array_equal(oracle.dequantize_q2(np.full((N, K // 4), 0xFF, dtype=np.uint8),
                                               scales), deq)


# ------------------------------------------------------------------ GEMV ----
def _rand_planes(fmt, N, K, seed):
    w = synth.weights_f32(synth.key(seed, 91, 0, 0, 0), N, K)
    return {2: oracle.quantize_q2, 3: oracle.quantize_q3, 4: oracle.quantize_q4,
            5: oracle.quantize_q5, 6: oracle.quantize_q6, 8: oracle.quantize_q8}[fmt](w)


_DEQ = {2: lambda c, s: oracle.dequantize_q2(c, s), 3: lambda c, s: oracle.dequantize_q3(c, s),
        4: lambda c, s: oracle.dequantize_q4(c, s), 5: lambda c, s: oracle.dequantize_q5(c, s),
        6: lambda c, s: oracle.dequantize_q6(c, s), 8: lambda c, s: oracle.dequantize_q8(c, s)}
_GEMV = {2: lambda *a, **k: oracle.gemv_q2(*a, **k), 3: lambda *a, **k: oracle.gemv_q3(*a, **k),
         4: lambda *a, **k: oracle.gemv_q4(*a, **k), 5: lambda *a, **k: oracle.gemv_q5(*a, **k),
         6: lambda *a, **k: oracle.gemv_q6(*a, **k), 8: lambda *a, **k: oracle.gemv_q8(*a, **k)}


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
def test_gemv_one_hot_returns_columns(fmt):
    N, K = 7, 96
    codes, scales = _rand_planes(fmt, N, K, 1)
    deq = _DEQ[fmt](codes, scales)
    gemv = _GEMV[fmt]
    one = np.float16(1.0).view(np.uint16)
    x = np.zeros((K, K), dtype=np.uint16)
    x[np.arange(K), np.arange(K)] = one                 # B = K one-hot rows, 8 at a time
    for b0 in range(0, K, 8):
        y, _ = gemv(codes, scales, x[b0:b0 + 8])
        assert np.array_equal(y, deq[:, b0:b0 + 8].T)


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
def test_gemv_all_ones_returns_row_sums(fmt):
    import math
    N, K = 11, 160
    codes, scales = _rand_planes(fmt, N, K, 2)
    deq = _DEQ[fmt](codes, scales)
    gemv = _GEMV[fmt]
    x = np.full((2, K), np.float16(1.0).view(np.uint16), dtype=np.uint16)
    y, a = gemv(codes, scales, x)
    for n in range(N):
        assert y[0, n] == y[1, n] == math.fsum(deq[n])
        assert a[0, n] == math.fsum(np.abs(deq[n]))


def _unpack_fraction(fmt, codes, scales, n, k):
    """Independent unpack straight from the format text, as an exact Fraction."""
    bits = int(scales[n, k // 32])
    d = Fraction(np.uint16(bits).view(np.float16).item())
    if fmt == 8:
        return d * int(codes[n, k])
    i = k % 32
    if fmt in (2, 3):
        lo = (int(codes[n, (k // 32) * 8 + i % 8]) >> (2 * (i // 8))) & 3
        if fmt == 2:
            return d * (lo - 2)
        K = codes.shape[1] * 8 // 3
        top = (int(codes[n, K // 4 + (k // 32) * 4 + i % 4]) >> (i // 4)) & 1
        return d * ((lo | (top << 2)) - 4)
    byte = int(codes[n, (k // 32) * 16 + i % 16])
    q = byte & 15 if i < 16 else byte >> 4
    if fmt == 6:
        K = codes.shape[1] * 4 // 3
        top = (int(codes[n, K // 2 + (k // 32) * 8 + i % 8]) >> (2 * (i // 8))) & 3
        return d * ((q | (top << 4)) - 32)
    if fmt == 5:
        K = codes.shape[1] * 8 // 5
        top = (int(codes[n, K // 2 + (k // 32) * 4 + i % 4]) >> (i // 4)) & 1
        return d * ((q | (top << 4)) - 16)
    return d * (q - 8)


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("N,K,B", [(1, 32, 1), (3, 64, 2), (8, 96, 8), (5, 32, 3), (2, 96, 5)])
def test_gemv_brute_force_exact(fmt, N, K, B):
    codes, scales = _rand_planes(fmt, N, K, 10 * N + K + B)
    x = synth.activations_f16_bits(synth.key(3, 91, N, K, 1), B, K)
    gemv = _GEMV[fmt]
    y, a = gemv(codes, scales, x)
    xf = x.view(np.float16)
    for b in range(B):
        for n in range(N):
            terms = [_unpack_fraction(fmt, codes, scales, n, k) * Fraction(xf[b, k].item())
                     for k in range(K)]
            exact = sum(terms)
            exact_abs = sum(abs(t) for t in terms)
            assert abs(Fraction(y[b, n]) - exact) <= exact_abs * Fraction(1, 2 ** 50)
            assert abs(Fraction(a[b, n]) - exact_abs) <= exact_abs * Fraction(1, 2 ** 50)


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("B", [16, 32])
def test_gemv_brute_force_exact_wide_batch(fmt, B):
    """Batches beyond the GEMV's 8 (the size of a speculative-decoding
    verification batch): the oracle has no batch limit and stays exact."""
    N, K = 3, 64
    codes, scales = _rand_planes(fmt, N, K, 900 + B)
    x = synth.activations_f16_bits(synth.key(5, 91, B, K, 1), B, K)
    y, a = _GEMV[fmt](codes, scales, x)
    xf = x.view(np.float16)
    for b in range(B):
        for n in range(N):
            terms = [_unpack_fraction(fmt, codes, scales, n, k) * Fraction(xf[b, k].item())
                     for k in range(K)]
            exact = sum(terms)
            exact_abs = sum(abs(t) for t in terms)
            assert abs(Fraction(y[b, n]) - exact) <= exact_abs * Fraction(1, 2 ** 50)
            assert abs(Fraction(a[b, n]) - exact_abs) <= exact_abs * Fraction(1, 2 ** 50)


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
def test_gemv_batch_rows_independent_and_threads(fmt):
    N, K, B = 37, 256, 6
    codes, scales = _rand_planes(fmt, N, K, 5)
    x = synth.activations_f16_bits(synth.key(4, 91, 0, 0, 1), B, K)
    gemv = _GEMV[fmt]
    y, a = gemv(codes, scales, x)
    y4, a4 = gemv(codes, scales, x, nthreads=4)
    assert np.array_equal(y, y4) and np.array_equal(a, a4)
    for b in range(B):
        yb, _ = gemv(codes, scales, x[b:b + 1])
        assert np.array_equal(yb[0], y[b])


# ------------------------------------------------------------------- MoE ----
def _moe_stack(E, N, K, seed):
    cs, ss = [], []
    for e in range(E):
        c, s = oracle.quantize_q4(synth.weights_f32(synth.key(seed, 92, 0, e, 0), N, K))
        cs.append(c)
        ss.append(s)
    return np.stack(cs), np.stack(ss)


def test_moe_identical_experts_uniform_weights_is_dense():
    E, N, K, B, topk = 6, 24, 64, 3, 4
    c, s = oracle.quantize_q4(synth.weights_f32(synth.key(1, 92, 0, 0, 0), N, K))
    codes, scales = np.stack([c] * E), np.stack([s] * E)
    x = synth.activations_f16_bits(synth.key(1, 92, 0, 0, 1), B, K)
    idx = np.array([[0, 2, 3, 5], [1, 2, 4, 0], [5, 4, 3, 2]], dtype=np.int32)
    r = np.full((B, topk), 0.25, dtype=np.float32)
    y, _, bad = oracle.moe_gemv_q4(codes, scales, x, False, idx, r)
    yd, _ = oracle.gemv_q4(c, s, x)
    assert not bad
    np.testing.assert_allclose(y, yd, rtol=1e-14, atol=1e-15)


def test_moe_slot_permutation_invariance_and_combine():
    E, N, K, B, topk = 9, 16, 96, 4, 3
    codes, scales = _moe_stack(E, N, K, 2)
    x = synth.activations_f16_bits(synth.key(2, 92, 0, 0, 1), B, topk, K)
    idx, r = synth.routing(synth.key(2, 92, 0, 0, 2), synth.key(2, 92, 0, 0, 3), B, E, topk)
    y, a, _ = oracle.moe_gemv_q4(codes, scales, x, True, idx, r)
    perm = np.array([2, 0, 1])
    yp, ap, _ = oracle.moe_gemv_q4(codes, scales, x[:, perm], True, idx[:, perm], r[:, perm])
    np.testing.assert_allclose(yp, y, rtol=1e-13, atol=1e-15)
    per, aper, _ = oracle.moe_gemv_q4(codes, scales, x, True, idx, None)
    assert per.shape == (B, topk, N)
    comb = (r.astype(np.float64)[..., None] * per).sum(axis=1)
    np.testing.assert_allclose(comb, y, rtol=1e-13, atol=1e-15)
    # each per-slot output is the dense GEMV of the routed expert
    for b in range(B):
        for t in range(topk):
            yd, _ = oracle.gemv_q4(codes[idx[b, t]], scales[idx[b, t]], x[b, t][None])
            assert np.array_equal(per[b, t], yd[0])


def test_moe_single_expert_is_dense_batch():
    E, N, K, B = 4, 20, 64, 5
    codes, scales = _moe_stack(E, N, K, 3)
    x = synth.activations_f16_bits(synth.key(3, 92, 0, 0, 1), B, K)
    idx = np.full((B, 1), 2, dtype=np.int32)
    per, _, _ = oracle.moe_gemv_q4(codes, scales, x, False, idx, None)
    yd, _ = oracle.gemv_q4(codes[2], scales[2], x)
    assert np.array_equal(per[:, 0], yd)


def test_moe_out_of_range_index_flags_and_skips():
    E, N, K, B, topk = 3, 8, 32, 2, 2
    codes, scales = _moe_stack(E, N, K, 4)
    x = synth.activations_f16_bits(synth.key(4, 92, 0, 0, 1), B, K)
    idx = np.array([[0, 3], [-1, 1]], dtype=np.int32)
    r = np.array([[0.5, 0.5], [0.25, 0.75]], dtype=np.float32)
    y, _, bad = oracle.moe_gemv_q4(codes, scales, x, False, idx, r)
    assert bad
    y0, _ = oracle.gemv_q4(codes[0], scales[0], x[0:1])
    y1, _ = oracle.gemv_q4(codes[1], scales[1], x[1:2])
    np.testing.assert_allclose(y[0], 0.5 * y0[0], rtol=1e-15)
    np.testing.assert_allclose(y[1], np.float64(np.float32(0.75)) * y1[0], rtol=1e-15)
    per, _, bad = oracle.moe_gemv_q4(codes, scales, x, False, idx, None)
    assert bad and np.all(per[0, 1] == 0) and np.all(per[1, 0] == 0)


# ------------------------------------------------------------- SwiGLU ----
def test_silu_closed_forms():
    """silu(z) = z * sigmoid(z): sigmoid(0) = 1/2 and sigmoid(ln 3) = 3/4 give
    exact values; sigmoid(z) + sigmoid(-z) = 1 gives the odd part
    silu(z) - silu(-z) = z, and sigmoid(z) - sigmoid(-z) = tanh(z/2) the even
    part silu(z) + silu(-z) = z tanh(z/2) (library tanh, an independent
    function); large |z| saturates to z and to 0."""
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    assert oracle.silu(-math.log(3.0)) == pytest.approx(-0.25 * math.log(3.0), rel=1e-15)
    for z in (0.1, 0.5, 1.0, 2.5, 7.0, 20.0):
        assert oracle.silu(z) - oracle.silu(-z) == pytest.approx(z, rel=1e-14)
        assert oracle.silu(z) + oracle.silu(-z) == pytest.approx(z * math.tanh(z / 2.0), rel=1e-12)
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(oracle.silu(-40.0)) < 1e-15


def test_swiglu_f16_rounds_the_product_once():
    """h = fp16(silu(g) * u): with sigmoid(ln 3) = 3/4 and u a power of two the
    exact value is (3/4) ln 3 * 2^k, whose nearest fp16 numpy's float16 gives;
    u = 0 gives a zero; silu(+-40) * u saturates to u*40 and to -0."""
    ln3 = math.log(3.0)
    g = np.array([ln3, ln3, ln3, -ln3, 0.0, 40.0, -40.0])
    u = np.array([1.0, 4.0, -0.125, 2.0, 3.0, 0.5, 1.0])
    h = oracle.swiglu_f16(g, u)
    want = np.array([0.75 * ln3, 3.0 * ln3, -0.75 * ln3 / 8.0, -0.5 * ln3, 0.0, 20.0, -0.0],
                    dtype=np.float64).astype(np.float16).view(np.uint16)
    assert np.array_equal(h[:6], want[:6])
    assert h[6] == 0x8000        # -40 * sigmoid(-40) = -1.7e-16: rounds to -0

"""Pins of the oracle's decode attention over a Q8 KV cache
(oracle_attn_decode_q8) against what the mathematics fixes, with no second
implementation of the same formula: a single position returns its value
vector exactly; a zero query weighs every position equally (the plain mean);
two positions whose scores differ by ln 3 get weights 3/4 and 1/4 exactly;
the result is invariant under permuting positions, ignores positions beyond
the sequence length, survives scores far outside exp's range, and groups
query heads onto KV heads as i / G.  The KV rows are quantised by the
oracle's own (separately pinned) Q8 quantiser."""
import math

import numpy as np
import pytest

import oracle


def kv_cache(kf, vf):
    """Q8 caches of float keys / values [B, Hkv, T, D]: (k_codes, k_scales,
    vt_codes, v_scales) in the oracle's layouts."""
    B, Hkv, T, D = kf.shape
    kc, ks = oracle.quantize_q8(np.ascontiguousarray(kf.reshape(-1, D), dtype=np.float32))
    vc, vs = oracle.quantize_q8(np.ascontiguousarray(vf.reshape(-1, D), dtype=np.float32))
    nb = D // 32
    kc = kc.reshape(B, Hkv, T, D)
    ks = ks[:, :nb].reshape(B, Hkv, T, nb)
    vt = np.ascontiguousarray(vc.reshape(B, Hkv, T, D).transpose(0, 1, 3, 2))
    vs = vs[:, :nb].reshape(B, Hkv, T, nb)
    return kc, ks, vt, vs


def deq_v(vt, vs):
    """Dequantised values [B, Hkv, T, D] in fp64."""
    d = oracle.half_to_double(vs)
    return vt.transpose(0, 1, 3, 2).astype(np.float64) * np.repeat(d, 32, axis=-1)


def rand_case(seed, B=2, Hkv=2, G=3, T=40, D=64):
    rng = np.random.default_rng(seed)
    kf = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    vf = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    q = rng.standard_normal((B, Hkv * G, D)).astype(np.float16).view(np.uint16)
    return kf, vf, q


def test_single_position_returns_its_value_exactly():
    kf, vf, q = rand_case(1, T=1)
    kc, ks, vt, vs = kv_cache(kf, vf)
    lens = np.ones(2, dtype=np.int32)
    o, ao, empty = oracle.attn_decode_q8(kc, ks, vt, vs, q, lens, 0.125)
    assert not empty
    V = deq_v(vt, vs)                                   # [B, Hkv, 1, D]
    G = q.shape[1] // 2
    for i in range(q.shape[1]):
        assert np.array_equal(o[:, i], V[:, i // G, 0])
        assert np.array_equal(ao[:, i], np.abs(V[:, i // G, 0]))


def test_zero_query_weighs_positions_equally():
    kf, vf, q = rand_case(2, T=37)
    q[:] = 0
    kc, ks, vt, vs = kv_cache(kf, vf)
    lens = np.array([37, 5], dtype=np.int32)
    o, _, _ = oracle.attn_decode_q8(kc, ks, vt, vs, q, lens, 0.125)
    V = deq_v(vt, vs)
    G = q.shape[1] // 2
    for b, L in enumerate(lens):
        for i in range(q.shape[1]):
            np.testing.assert_allclose(o[b, i], V[b, i // G, :L].mean(axis=0), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("dim", [0, 40, 127])
def test_score_gap_ln3_gives_weights_three_quarters_and_one_quarter(dim):
    """Key 0 = 2.5 e_dim (in block dim / 32 of the head), key 1 = 0, q = e_dim:
    with scale = ln 3 / (the stored key component) the scores are ln 3 and 0."""
    D, T = 128, 2
    kf = np.zeros((1, 1, T, D), dtype=np.float32)
    kf[0, 0, 0, dim] = 2.5
    kf[0, 0, 1, (dim + 64) % D] = 3.0          # key 1: orthogonal to q, other scales non-zero
    vf = np.random.default_rng(3).standard_normal((1, 1, T, D)).astype(np.float32)
    kc, ks, vt, vs = kv_cache(kf, vf)
    kd = oracle.half_to_double(ks[0, 0, 0, dim // 32]) * kc[0, 0, 0, dim]   # the stored component
    q = np.zeros((1, 1, D), dtype=np.float16)
    q[0, 0, dim] = 1.0
    o, _, _ = oracle.attn_decode_q8(kc, ks, vt, vs, q.view(np.uint16), np.array([2], np.int32),
                                    math.log(3.0) / kd)
    V = deq_v(vt, vs)[0, 0]
    np.testing.assert_allclose(o[0, 0], 0.75 * V[0] + 0.25 * V[1], rtol=1e-14, atol=1e-16)


def test_permuting_positions_leaves_output_unchanged():
    kf, vf, q = rand_case(4, T=29)
    perm = np.random.default_rng(5).permutation(29)
    lens = np.array([29, 29], dtype=np.int32)
    o1, a1, _ = oracle.attn_decode_q8(*kv_cache(kf, vf), q, lens, 0.2)
    o2, a2, _ = oracle.attn_decode_q8(*kv_cache(kf[:, :, perm], vf[:, :, perm]), q, lens, 0.2)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(a1, a2, rtol=1e-12, atol=1e-14)


def test_positions_beyond_length_are_never_read():
    kf, vf, q = rand_case(6, T=50)
    kc, ks, vt, vs = kv_cache(kf, vf)
    lens = np.array([17, 50], dtype=np.int32)
    o1, _, _ = oracle.attn_decode_q8(kc, ks, vt, vs, q, lens, 0.1)
    kc2, ks2, vt2, vs2 = kc.copy(), ks.copy(), vt.copy(), vs.copy()
    kc2[0, :, 17:] = 127
    ks2[0, :, 17:] = 0x7C00                   # +inf scales past the length
    vt2[0, :, :, 17:] = -127
    vs2[0, :, 17:] = 0x7E00                   # NaN scales past the length
    o2, _, _ = oracle.attn_decode_q8(kc2, ks2, vt2, vs2, q, lens, 0.1)
    assert np.array_equal(o1, o2)


def test_scores_far_outside_exp_range_stay_finite():
    """Scores of order 1e5 (exp overflows without the max subtraction): the
    output is finite and, with one position far ahead, equals its value."""
    kf, vf, q = rand_case(7, B=1, Hkv=1, G=1, T=12, D=32)
    kf[0, 0, 5] = 4.0 * np.sign(q.view(np.float16)[0, 0]).astype(np.float32)   # aligned with q
    kc, ks, vt, vs = kv_cache(kf, vf)
    o, _, _ = oracle.attn_decode_q8(kc, ks, vt, vs, q, np.array([12], np.int32), 1e4)
    assert np.all(np.isfinite(o))
    np.testing.assert_array_equal(o[0, 0], deq_v(vt, vs)[0, 0, 5])


def test_query_heads_grouped_onto_kv_heads():
    """G query heads per KV head: head i of a G-grouped call equals a G = 1
    call on KV head i // G alone."""
    kf, vf, q = rand_case(8, B=1, Hkv=3, G=4, T=21, D=96)
    lens = np.array([21], dtype=np.int32)
    o, _, _ = oracle.attn_decode_q8(*kv_cache(kf, vf), q, lens, 0.3)
    for i in range(12):
        h = i // 4
        oi, _, _ = oracle.attn_decode_q8(*kv_cache(kf[:, h:h + 1], vf[:, h:h + 1]), q[:, i:i + 1],
                                         lens, 0.3)
        assert np.array_equal(o[:, i], oi[:, 0])


def test_empty_sequence_gives_zero_and_is_flagged():
    kf, vf, q = rand_case(9)
    o, ao, empty = oracle.attn_decode_q8(*kv_cache(kf, vf), q, np.array([0, 40], np.int32), 0.1)
    assert empty and not np.any(o[0]) and not np.any(ao[0]) and np.any(o[1])

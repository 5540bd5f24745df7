"""The seeded input generators follow the stated recipe: weights N(0, 0.02) in
fp32, activations N(0, 1) rounded to fp16, routed-expert indices drawn without
replacement with softmax routing weights, sequence lengths uniform in 1 .. Tmax,
every stream determined by its key and distinct across keys; and the workload
shapes have the sizes the benchmark and the design state."""
import os

import numpy as np
import pytest

from quantised_weight_gemv_b200 import synth
from tests.conftest import ROOT


def test_streams_are_determined_by_their_key_and_distinct_across_keys():
    k = synth.key(3, 5, 7, 1, synth.KIND_W)
    a, b = synth.weights_f32(k, 64, 256), synth.weights_f32(k, 64, 256)
    assert np.array_equal(a, b)
    for other in (synth.key(4, 5, 7, 1, synth.KIND_W), synth.key(3, 6, 7, 1, synth.KIND_W),
                  synth.key(3, 5, 8, 1, synth.KIND_W), synth.key(3, 5, 7, 2, synth.KIND_W),
                  synth.key(3, 5, 7, 1, synth.KIND_X)):
        assert not np.array_equal(a, synth.weights_f32(other, 64, 256)), other
    s = synth.torch_seed(k)
    assert s == synth.torch_seed(list(k)) and 0 <= s < (1 << 63)
    assert s != synth.torch_seed(synth.key(3, 5, 7, 1, synth.KIND_X))


def test_weights_are_normal_with_standard_deviation_0_02():
    w = synth.weights_f32(synth.key(0, 1, 0, 0, synth.KIND_W), 1024, 1024)
    assert w.dtype == np.float32 and w.shape == (1024, 1024)
    # 2^20 draws: the sample std is within 0.3% and the mean within 5e-5 of N(0, 0.02)
    assert abs(float(w.std()) / 0.02 - 1) < 3e-3 and abs(float(w.mean())) < 5e-5
    # normal tails: about 4.55% beyond two standard deviations
    assert abs(float(np.mean(np.abs(w) > 0.04)) - 0.0455) < 2e-3


def test_weights_on_torch_have_the_same_distribution():
    import torch
    w = synth.weights_f32_torch(synth.key(0, 1, 0, 0, synth.KIND_W), 1024, 1024, "cpu")
    assert w.dtype == torch.float32 and tuple(w.shape) == (1024, 1024)
    assert abs(float(w.std()) / 0.02 - 1) < 3e-3 and abs(float(w.mean())) < 5e-5
    again = synth.weights_f32_torch(synth.key(0, 1, 0, 0, synth.KIND_W), 1024, 1024, "cpu")
    assert torch.equal(w, again)


def test_activations_are_fp16_roundings_of_standard_normal_draws():
    bits = synth.activations_f16_bits(synth.key(0, 1, 0, 0, synth.KIND_X), 8, 65536)
    assert bits.dtype == np.uint16 and bits.shape == (8, 65536)
    x = bits.view(np.float16).astype(np.float64)
    assert np.all(np.isfinite(x))
    assert abs(float(x.std()) - 1) < 3e-3 and abs(float(x.mean())) < 3e-3
    # each value lies within half an fp16 ulp of the fp32 draw of the same
    # stream: rounded to the nearest fp16
    raw = np.random.default_rng(synth.key(0, 1, 0, 0, synth.KIND_X)).standard_normal(
        (8, 65536), dtype=np.float32).astype(np.float64)
    ulp = np.spacing(np.abs(x).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(x - raw) <= ulp / 2)


@pytest.mark.parametrize("B,E,topk", [(1, 128, 8), (8, 128, 8), (3, 5, 4), (64, 16, 2)])
def test_routing_draws_distinct_experts_and_softmax_weights(B, E, topk):
    idx, w = synth.routing(synth.key(0, 4, 0, 0, synth.KIND_IDX),
                           synth.key(0, 4, 0, 0, synth.KIND_LOGIT), B, E, topk)
    assert idx.dtype == np.int32 and idx.shape == (B, topk)
    assert w.dtype == np.float32 and w.shape == (B, topk)
    assert np.all((idx >= 0) & (idx < E))
    assert all(len(set(row.tolist())) == topk for row in idx)
    assert np.all(w > 0) and np.allclose(w.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)


def test_routing_is_uniform_over_experts():
    """Many tokens: each of E experts is picked about B * topk / E times."""
    B, E, topk = 4096, 32, 4
    idx, _ = synth.routing(synth.key(0, 4, 1, 0, synth.KIND_IDX),
                           synth.key(0, 4, 1, 0, synth.KIND_LOGIT), B, E, topk)
    counts = np.bincount(idx.ravel(), minlength=E)
    expect = B * topk / E
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < 80          # 31 degrees of freedom: p < 1e-5 beyond this


def test_sequence_lengths_are_uniform_in_one_to_tmax():
    lens = synth.seq_lens(synth.key(0, 12, 0, 0, synth.KIND_LEN), 20000, 8192)
    assert lens.dtype == np.int32 and lens.min() >= 1 and lens.max() <= 8192
    assert abs(float(lens.mean()) / (8193 / 2) - 1) < 0.02
    wl = synth.attn_h2048(8, 8192)
    assert not wl.full and np.array_equal(wl.lens(), wl.lens())
    assert np.all((wl.lens() >= 1) & (wl.lens() <= 8192))
    full = synth.attn_h5120(1, 32768)
    assert np.array_equal(full.lens(), [32768])


def test_workload_sizes():
    q4 = lambda wl: wl.layers * sum(synth.packed_bytes(4, m.N, m.K) for m in wl.mats)
    # 64-layer hidden-5120 decoder: 16.42 GB of Q4 weights
    assert round(q4(synth.DENSE_H5120) / 1e9, 2) == 16.42
    assert synth.DENSE_H5120.layer_weights() == 5120 * 5120 * 2 + 1024 * 5120 * 2 + 25600 * 5120 * 3
    # 16-layer hidden-2048 decoder
    assert synth.DENSE_H2048.layer_weights() == 2048 * 2048 * 2 + 512 * 2048 * 2 + 8192 * 2048 * 3
    # routed experts: 48 layers of 128 experts, gate|up 1536 x 2048 and down 2048 x 768
    moe = synth.moe_h2048(1)
    assert moe.gateup() == (1536, 2048) and moe.down() == (2048, 768)
    per_expert = synth.packed_bytes(4, 1536, 2048) + synth.packed_bytes(4, 2048, 768)
    assert round(moe.layers * moe.E * per_expert / 1e9, 1) == 16.3
    # packed bytes of each format: per 32-weight block, 32 codes of `bits` bits
    # plus one 2-byte scale (a 32 x 256 matrix holds 256 blocks)
    for fmt, bits in ((2, 2), (3, 3), (4, 4), (5, 5), (6, 6), (8, 8)):
        assert synth.packed_bytes(fmt, 32, 256) == 256 * (32 * bits // 8 + 2)
    # independent copies of a sweep shape cover at least 512 MB (at most 256 copies)
    sw = synth.sweep_workload(4, 25600, 5120)
    assert sw.independent and sw.layers * synth.packed_bytes(4, 25600, 5120) >= 512 << 20


def test_workload_ids_separate_the_seed_streams():
    """Distinct workload families draw from distinct streams (the id is part
    of every key); the formats of one family share its weights."""
    fams = [synth.SINGLE_Q8, synth.DENSE_H2048, synth.dense_h4096(4, 1), synth.moe_h2048(1),
            synth.DENSE_H5120, synth.sweep_workload(4, 512, 512), synth.single_workload(4, 512, 512),
            synth.dense_h2048(8), synth.verify_h4096(4, 32),
            synth.verify_sweep_workload(4, 24576, 4096, 32), synth.attn_h5120(1, 4096),
            synth.attn_h2048(8, 8192)]
    assert len({f.wid for f in fams}) == len(fams)
    assert synth.dense_h2048(8).mats == synth.DENSE_H2048.mats
    assert synth.dense_h2048(3).wid == synth.dense_h2048(6).wid


def test_generators_hold_no_method_arithmetic():
    """The input module imports neither the oracle nor the library."""
    with open(os.path.join(ROOT, "quantised_weight_gemv_b200", "synth.py")) as f:
        src = f.read()
    for banned in ("import oracle", "from oracle", "libbq", "from . import bq",
                   "from quantised_weight_gemv_b200 import bq", "ctypes"):
        assert banned not in src, banned

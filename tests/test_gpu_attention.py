"""GPU parity of decode attention over a Q8 KV cache (bq_attn_decode_q8)
against the fp64 oracle (oracle_attn_decode_q8).

The caches are built on the CPU by the oracle's Q8 quantiser from seeded
N(0, 1) keys and values (no oracle input comes from the CUDA path).  Shapes
follow the decoders of the workloads: head dimension 128, G = 4 query heads
per KV head (the hidden-2048 decoder: 16 query heads, 4 KV heads), G = 5 (the
hidden-5120 decoder: 40 and 8) and G = 8 (a routed-expert model's 32 and 4).

Tolerance, per output element: |o - o_ref| <= 1e-3 * sum_t p_t |V[t][d]| +
1e-5.  The kernel's products of codes are exact and each softmax weight times
its value scale enters the tensor core rounded once to fp16 (2^-11 relative);
scores accumulate in fp32 and the exponential is exp2's approximation
(2^-22 relative), both far below the bound."""
import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import DEV, new_status

pytestmark = pytest.mark.gpu
REL, ABS = 1e-3, 1e-5


def build_cache(seed, B, Hkv, Tmax, D=128):
    """Q8 cache planes (numpy, oracle layouts) of seeded N(0, 1) keys/values."""
    kf = synth.kv_values_f32(synth.key(seed, 91, B, Hkv, synth.KIND_KEY), B * Hkv * Tmax, D)
    vf = synth.kv_values_f32(synth.key(seed, 91, B, Hkv, synth.KIND_VAL), B * Hkv * Tmax, D)
    kc, ks = oracle.quantize_q8(kf)
    vc, vs = oracle.quantize_q8(vf)
    nb = D // 32
    kc = kc.reshape(B, Hkv, Tmax, D)
    ks = np.ascontiguousarray(ks[:, :nb]).reshape(B, Hkv, Tmax, nb)
    vt = np.ascontiguousarray(vc.reshape(B, Hkv, Tmax, D).transpose(0, 1, 3, 2))
    vs = np.ascontiguousarray(vs[:, :nb]).reshape(B, Hkv, Tmax, nb)
    return kc, ks, vt, vs


def to_dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(DEV)


def run_gpu(kc, ks, vt, vs, q_bits, lens, G, scale, ws=None):
    import torch
    B, Hkv, Tmax, D = kc.shape
    kv = bq.kv_cache(to_dev(kc), to_dev(ks), to_dev(vt), to_dev(vs))
    qd, ld = to_dev(q_bits), to_dev(lens.astype(np.int32))
    o = torch.full((B, Hkv * G, D), float("nan"), dtype=torch.float32, device=DEV)
    ws = ws if ws is not None else bq.workspace(bq.lib().bq_attn_workspace_bytes(B, Hkv), DEV)
    st = new_status()
    bq.attn_decode_q8(kv, qd, ld, G, scale, o, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item()):#x}"
    return o.cpu().numpy(), ws


def check(o, o_ref, abso):
    assert np.all(np.isfinite(o))
    err = np.abs(o.astype(np.float64) - o_ref)
    bound = REL * abso + ABS
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{len(bad)} outputs out of tolerance, first {bad[:5].tolist()}, " \
                          f"max ratio {float(np.max(err / bound))}"


CASES = [
    # (B, Hkv, G, Tmax, lens)
    (1, 4, 4, 128, [1]),
    (1, 4, 4, 128, [128]),
    (1, 4, 4, 256, [129]),
    (2, 2, 8, 256, [200, 37]),
    (3, 8, 5, 1024, [1000, 1, 513]),
    (1, 1, 1, 4096, [4096]),
    (2, 4, 4, 8192, [8192, 5000]),
    (4, 8, 5, 2048, [2048, 17, 1500, 640]),
    (1, 2, 3, 32768, [32768]),
]


@pytest.mark.parametrize("B,Hkv,G,Tmax,lens", CASES)
def test_attention_parity(B, Hkv, G, Tmax, lens):
    kc, ks, vt, vs = build_cache(0, B, Hkv, Tmax)
    q = synth.activations_f16_bits(synth.key(0, 91, B, Hkv * G, synth.KIND_X), B, Hkv * G, 128)
    lens = np.array(lens, dtype=np.int32)
    scale = 1.0 / np.sqrt(128.0)
    o, _ = run_gpu(kc, ks, vt, vs, q, lens, G, scale)
    o_ref, abso, _ = oracle.attn_decode_q8(kc, ks, vt, vs, q, lens, scale)
    check(o, o_ref, abso)


def test_attention_sharp_scores():
    """A large softmax scale (peaked weights; scores of order 100s): still
    within tolerance, nothing overflows."""
    B, Hkv, G, Tmax = 2, 2, 4, 512
    kc, ks, vt, vs = build_cache(1, B, Hkv, Tmax)
    q = synth.activations_f16_bits(synth.key(1, 91, B, Hkv * G, synth.KIND_X), B, Hkv * G, 128)
    lens = np.array([512, 300], dtype=np.int32)
    o, _ = run_gpu(kc, ks, vt, vs, q, lens, G, 2.0)
    o_ref, abso, _ = oracle.attn_decode_q8(kc, ks, vt, vs, q, lens, 2.0)
    check(o, o_ref, abso)


def test_attention_ignores_cache_past_length():
    """Codes of 127 and infinite / NaN scales past each length change nothing."""
    B, Hkv, G, Tmax = 2, 2, 4, 512
    kc, ks, vt, vs = build_cache(2, B, Hkv, Tmax)
    q = synth.activations_f16_bits(synth.key(2, 91, B, Hkv * G, synth.KIND_X), B, Hkv * G, 128)
    lens = np.array([77, 300], dtype=np.int32)
    o1, ws = run_gpu(kc, ks, vt, vs, q, lens, G, 0.09)
    for b, L in enumerate(lens):
        kc[b, :, L:] = 127
        ks[b, :, L:] = 0x7C00
        vt[b, :, :, L:] = -127
        vs[b, :, L:] = 0x7E00
    o2, _ = run_gpu(kc, ks, vt, vs, q, lens, G, 0.09, ws=ws)
    assert np.array_equal(o1, o2)
    o_ref, abso, _ = oracle.attn_decode_q8(kc, ks, vt, vs, q, lens, 0.09)
    check(o2, o_ref, abso)


def test_attention_empty_sequence_and_single_position():
    """lens 0 gives zeros; lens 1 returns the first value vector (p = 1)."""
    B, Hkv, G, Tmax = 2, 1, 2, 128
    kc, ks, vt, vs = build_cache(3, B, Hkv, Tmax)
    q = synth.activations_f16_bits(synth.key(3, 91, B, Hkv * G, synth.KIND_X), B, Hkv * G, 128)
    lens = np.array([0, 1], dtype=np.int32)
    o, _ = run_gpu(kc, ks, vt, vs, q, lens, G, 0.1)
    assert not np.any(o[0])
    v0 = vt[1, 0, :, 0].astype(np.float64) * np.repeat(oracle.half_to_double(vs[1, 0, 0]), 32)
    for i in range(G):
        assert np.all(np.abs(o[1, i] - v0) <= 2.0 ** -11 * np.abs(v0) + 1e-30)


def test_attention_deterministic_and_workspace_returns_to_zero():
    import torch
    B, Hkv, G, Tmax = 2, 4, 4, 8192
    kc, ks, vt, vs = build_cache(4, B, Hkv, Tmax)
    q = synth.activations_f16_bits(synth.key(4, 91, B, Hkv * G, synth.KIND_X), B, Hkv * G, 128)
    lens = np.array([8192, 7001], dtype=np.int32)
    o1, ws = run_gpu(kc, ks, vt, vs, q, lens, G, 0.1)
    assert int(ws.view(torch.int32).abs().sum().item()) == 0       # counters and partials
    o2, _ = run_gpu(kc, ks, vt, vs, q, lens, G, 0.1, ws=ws)
    assert np.array_equal(o1, o2)

"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Inputs come from the seeded generators in quantised_weight_gemv_b200.synth;
packed planes for the small cases come from the oracle's own quantiser, so no
oracle input is produced by the CUDA path.  Tolerance per output element:
|y - y_ref| <= 1e-3 * sum_k |deq(w) x| + 1e-5; packing is bit-exact.
"""
import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import DEV, check_tol, dev, gpu_gemv, new_status, oracle_gemv, quantize

pytestmark = pytest.mark.gpu

SHAPES = [(1, 32), (15, 32), (16, 256), (17, 288), (33, 800), (100, 2048), (257, 4128),
          (1000, 96), (4, 25600), (48, 768)]


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 6, 7, 8])
def test_gemv_parity_small(fmt, N, K, B):
    w = synth.weights_f32(synth.key(0, 80, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(0, 80, N, K, synth.KIND_X), B, K)
    y = gpu_gemv(fmt, codes, scales, x)
    y_ref, absy = oracle_gemv(fmt, codes, scales, x)
    check_tol(y, y_ref, absy)


@pytest.mark.parametrize("rows", [16, 32])
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("B", [1, 3, 4, 8])
def test_q4_chunk_heights_parity(rows, N, K, B):
    """Q4 with 16-row and with 32-row work units (BQ_GEMV_ROWS16 / ROWS32):
    both within the oracle's tolerance."""
    w = synth.weights_f32(synth.key(0, 82, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(4, w)
    x = synth.activations_f16_bits(synth.key(0, 82, N, K, synth.KIND_X), B, K)
    flag = bq.BQ_GEMV_ROWS16 if rows == 16 else bq.BQ_GEMV_ROWS32
    y = gpu_gemv(4, codes, scales, x, flags=flag)
    y_ref, absy = oracle_gemv(4, codes, scales, x)
    check_tol(y, y_ref, absy)


@pytest.mark.parametrize("fmt,N,K,rows", [(4, 2048, 8192, 32), (4, 2000, 8192, 32),
                                          (4, 4096, 4096, 32), (4, 1024, 16384, 32),
                                          (4, 2048, 8192, 16), (8, 1024, 8192, 16),
                                          (4, 1024, 5120, 32), (4, 1024, 1536, 32),
                                          (4, 1000, 1792, 32), (8, 512, 2560, 16)])
@pytest.mark.parametrize("B", [1, 3, 4, 8])
def test_bands_summed_across_ctas_in_clusters(fmt, N, K, rows, B):
    """Shapes whose bands are split among several CTAs (each band's chunks
    outnumber a CTA's warps) with cluster boundaries on band boundaries: the
    launch runs as clusters of 2, 4 or 8 CTAs and sums each band's CTA
    partials in the shared memory of its first CTA.  (K = 5120, 1536, 1792
    and 2560 would need clusters of 3, 5 or 7, which the library does not
    use: those cases check the workspace path on the same kind of split.)"""
    w = synth.weights_f32(synth.key(0, 83, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(0, 83, N, K, synth.KIND_X), B, K)
    flag = bq.BQ_GEMV_ROWS16 if rows == 16 else bq.BQ_GEMV_ROWS32
    y = gpu_gemv(fmt, codes, scales, x, flags=flag)
    y_ref, absy = oracle_gemv(fmt, codes, scales, x)
    check_tol(y, y_ref, absy)
    # and the same call again: every receive area and barrier starts clean
    assert np.array_equal(y, gpu_gemv(fmt, codes, scales, x, flags=flag))


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("B", [1, 3, 4, 8])
def test_gemv_static_weights_parity(fmt, N, K, B):
    """With BQ_GEMV_STATIC_WEIGHTS the weight ring fills before the wait on
    the previous kernel; the arithmetic is the plain call's, so y is the
    oracle's within tolerance and bit-identical to the plain call's."""
    w = synth.weights_f32(synth.key(0, 81, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(0, 81, N, K, synth.KIND_X), B, K)
    y = gpu_gemv(fmt, codes, scales, x, flags=bq.BQ_GEMV_STATIC_WEIGHTS)
    y_ref, absy = oracle_gemv(fmt, codes, scales, x)
    check_tol(y, y_ref, absy)
    assert np.array_equal(y, gpu_gemv(fmt, codes, scales, x))


@pytest.mark.parametrize("fmt", [4, 8])
def test_gemv_one_hot_is_correctly_rounded(fmt):
    """x = e_k returns column k of deq(W); the only rounding is fp32's."""
    N, K = 40, 512
    w = synth.weights_f32(synth.key(1, 80, 0, 0, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    for k0 in (0, 17, 255, 256, 500):
        x = np.zeros((8, K), dtype=np.float16)
        for b in range(8):
            x[b, (k0 + 3 * b) % K] = np.float16(1.5 - 0.25 * b)
        xb = x.view(np.uint16)
        y = gpu_gemv(fmt, codes, scales, xb)
        y_ref, _ = oracle_gemv(fmt, codes, scales, xb)
        assert np.array_equal(y, y_ref.astype(np.float32))


def test_q4_nibble_order_exhaustive_on_gpu():
    """Row r = 32*c + p holds code c at element p (all other codes 8, d = 1):
    with x = e_p the GPU must return c - 8 exactly at row 32*c + p."""
    N, K = 512, 32
    codes = np.full((N, 16), 0x88, dtype=np.uint8)
    for c in range(16):
        for p in range(32):
            r = 32 * c + p
            i = p % 16
            codes[r, i] = (codes[r, i] & 0xF0) | c if p < 16 else (codes[r, i] & 0x0F) | (c << 4)
    scales = np.zeros((N, 8), dtype=np.uint16)
    scales[:, 0] = 0x3C00
    for p0 in range(0, 32, 8):
        x = np.zeros((8, K), dtype=np.float16)
        for b in range(8):
            x[b, p0 + b] = 1.0
        y = gpu_gemv(4, codes, scales, x.view(np.uint16))
        for b in range(8):
            p = p0 + b
            expect = np.zeros(N, dtype=np.float32)
            for c in range(16):
                expect[32 * c + p] = c - 8
            assert np.array_equal(y[b], expect), p


@pytest.mark.parametrize("fmt", [4, 8])
def test_batch_columns_independent_and_deterministic(fmt):
    N, K = 777, 3072
    w = synth.weights_f32(synth.key(2, 80, 0, 0, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(2, 80, 0, 0, synth.KIND_X), 8, K)
    y8 = gpu_gemv(fmt, codes, scales, x)
    assert np.array_equal(y8, gpu_gemv(fmt, codes, scales, x))
    for b in range(8):
        assert np.array_equal(gpu_gemv(fmt, codes, scales, x[b:b + 1])[0], y8[b])


@pytest.mark.parametrize("fmt", [4, 8])
def test_device_quantiser_bit_exact(fmt):
    import torch
    from tests.test_abi_cpu import _edge_weights
    w = _edge_weights()
    N, K = w.shape
    codes_ref, scales_ref = quantize(fmt, w)
    c = torch.zeros((N, K // 2 if fmt == 4 else K), dtype=torch.uint8, device=DEV)
    s = torch.full((N, bq.scales_ld(K)), 0x1234, dtype=torch.int16, device=DEV)
    st = new_status()
    bq.quantize_dev(fmt, dev(w), c, s, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(c.cpu().numpy(), codes_ref.view(np.uint8))
    assert np.array_equal(s.cpu().numpy().view(np.uint16), scales_ref)
    wbad = w.copy()
    wbad[7, 40] = np.inf
    bq.quantize_dev(fmt, dev(wbad), c, s, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 1 << bq.BQ_ERR_RANGE


def test_workspace_counters_return_to_zero():
    import torch
    N, K = 300, 5120
    w = synth.weights_f32(synth.key(3, 80, 0, 0, synth.KIND_W), N, K)
    codes, scales = quantize(4, w)
    ws = bq.workspace(bq.lib().bq_gemv_workspace_bytes(N, K), DEV)
    x = synth.activations_f16_bits(synth.key(3, 80, 0, 0, synth.KIND_X), 2, K)
    y1 = gpu_gemv(4, codes, scales, x, ws=ws)
    y2 = gpu_gemv(4, codes, scales, x, ws=ws)
    assert np.array_equal(y1, y2)
    assert int(torch.count_nonzero(ws).item()) == 0      # counters and scratch alike


@pytest.mark.parametrize("fmt", [4, 8])
def test_one_workspace_shared_by_calls_of_different_shapes(fmt):
    """Calls of different shapes one after another on one workspace (as a
    chain of per-projection launches does): a few-row, very long-K call whose
    bands span many CTAs (its cross-CTA partial sums go through the
    workspace), then a many-row call whose arrival counters cover the bytes
    those partials used.  Every call leaves the workspace all-zero, and the
    second call matches the oracle."""
    import torch
    shapes = [(64, 25600, 1), (12288, 1024, 8), (40, 8192, 3), (6000, 4096, 2)]
    ws = bq.workspace(max(bq.lib().bq_gemv_workspace_bytes(N, K) for N, K, _ in shapes), DEV)
    for i, (N, K, B) in enumerate(shapes):
        w = synth.weights_f32(synth.key(4, 80, i, 0, synth.KIND_W), N, K)
        codes, scales = quantize(fmt, w)
        x = synth.activations_f16_bits(synth.key(4, 80, i, 0, synth.KIND_X), B, K)
        y = gpu_gemv(fmt, codes, scales, x, ws=ws)
        assert int(torch.count_nonzero(ws).item()) == 0, f"call {i} left the workspace dirty"
        yr, ar = oracle_gemv(fmt, codes, scales, x)
        check_tol(y, yr, ar)


# ---------------------------------------------------------------- experts ----
def _moe_inputs(E, N, K, B, topk, seed, x_per_slot):
    cs, ss = [], []
    for e in range(E):
        c, s = oracle.quantize_q4(synth.weights_f32(synth.key(seed, 81, 0, e, synth.KIND_W), N, K))
        cs.append(c)
        ss.append(s)
    codes, scales = np.stack(cs), np.stack(ss)
    shape = (B, topk, K) if x_per_slot else (B, K)
    x = synth.activations_f16_bits(synth.key(seed, 81, 0, 0, synth.KIND_X), *shape)
    idx, r = synth.routing(synth.key(seed, 81, 0, 0, synth.KIND_IDX),
                           synth.key(seed, 81, 0, 0, synth.KIND_LOGIT), B, E, topk)
    return codes, scales, x, idx, r


def gpu_moe(codes, scales, x, x_per_slot, idx, r):
    import torch
    E, N, K2 = codes.shape
    K = 2 * K2
    B, topk = idx.shape
    c, s = dev(codes), dev(scales)
    xt, it = dev(x), dev(idx)
    rt = dev(r) if r is not None else None
    y = torch.full((B, N) if r is not None else (B, topk, N), float("nan"),
                   dtype=torch.float32, device=DEV)
    ws = bq.workspace(bq.lib().bq_moe_workspace_bytes(N, K, B, topk, E), DEV)
    st = new_status()
    bq.moe_gemv_q4(bq.qmat(c, s, N, K), E, N * K2, N * scales.shape[2], xt, x_per_slot, it, rt,
                   y, ws, st)
    torch.cuda.synchronize()
    return y.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("B,topk,E", [(1, 8, 32), (4, 8, 32), (8, 8, 32), (3, 4, 5), (8, 2, 1),
                                      (4, 2, 6)])
@pytest.mark.parametrize("x_per_slot", [False, True])
@pytest.mark.parametrize("combine", [False, True])
def test_moe_parity(B, topk, E, x_per_slot, combine):
    N, K = 96, 768
    if E < topk:
        pytest.skip("needs E >= topk for sampling without replacement")
    codes, scales, x, idx, r = _moe_inputs(E, N, K, B, topk, B * 100 + topk, x_per_slot)
    rr = r if combine else None
    y, st = gpu_moe(codes, scales, x, x_per_slot, idx, rr)
    assert st == 0
    y_ref, absy, bad = oracle.moe_gemv_q4(codes, scales, x, x_per_slot, idx, rr, nthreads=8)
    assert not bad
    check_tol(y, y_ref, absy)


def test_moe_repeated_expert_and_many_tokens():
    """All 8 tokens route all slots to a few experts (pieces of > 8 slots are
    split), including one token that lists the same expert twice."""
    N, K, B, topk, E = 64, 512, 8, 4, 6
    codes, scales, x, _, r = _moe_inputs(E, N, K, B, topk, 9, True)
    idx = np.array([[0, 1, 2, 3]] * 7 + [[5, 5, 0, 1]], dtype=np.int32)
    for rr in (None, r):
        y, st = gpu_moe(codes, scales, x, True, idx, rr)
        assert st == 0
        y_ref, absy, _ = oracle.moe_gemv_q4(codes, scales, x, True, idx, rr)
        check_tol(y, y_ref, absy)


def test_moe_out_of_range_index_sets_status_no_trap():
    N, K, B, topk, E = 32, 256, 2, 2, 4
    codes, scales, x, _, r = _moe_inputs(E, N, K, B, topk, 11, False)
    idx = np.array([[0, 4], [-3, 1]], dtype=np.int32)
    for rr in (None, r):
        y, st = gpu_moe(codes, scales, x, False, idx, rr)
        assert st == 1 << bq.BQ_ERR_EXPERT_INDEX
        y_ref, absy, bad = oracle.moe_gemv_q4(codes, scales, x, False, idx, rr)
        assert bad
        check_tol(y, y_ref, absy)


def test_moe_token_with_no_valid_slot_combines_to_zero():
    """A token whose every expert id is out of range: its combined row is 0 (the
    output starts as NaN, so every element must be written), the other tokens
    are combined normally, and the status flags the bad ids."""
    N, K, B, topk, E = 96, 512, 3, 3, 6
    codes, scales, x, _, r = _moe_inputs(E, N, K, B, topk, 13, True)
    idx = np.array([[0, 5, 2], [-1, 6, 99], [2, 2, 3]], dtype=np.int32)
    y, st = gpu_moe(codes, scales, x, True, idx, r)
    assert st == 1 << bq.BQ_ERR_EXPERT_INDEX
    assert np.all(y[1] == 0.0)
    y_ref, absy, bad = oracle.moe_gemv_q4(codes, scales, x, True, idx, r)
    assert bad
    check_tol(y, y_ref, absy)


@pytest.mark.parametrize("B", [1, 2])
def test_moe_small_batch_combine(B):
    """Combined outputs at batch 1-2: a token listing one expert twice, a token
    with no valid slot (its row must be written as 0: the output starts NaN),
    and the workspace all-zero again afterwards."""
    import torch
    N, K, topk, E = 96, 512, 4, 6
    codes, scales, x, _, r = _moe_inputs(E, N, K, B, topk, 17 + B, False)
    rows = [[5, 5, 0, 3], [-1, 6, 99, -2]][:B]
    idx = np.array(rows, dtype=np.int32)
    c, s = dev(codes), dev(scales)
    y = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = bq.workspace(bq.lib().bq_moe_workspace_bytes(N, K, B, topk, E), DEV)
    st = new_status()
    bq.moe_gemv_q4(bq.qmat(c, s, N, K), E, N * K // 2, N * scales.shape[2], dev(x), False,
                   dev(idx), dev(r), y, ws, st)
    torch.cuda.synchronize()
    yn = y.cpu().numpy()
    y_ref, absy, bad = oracle.moe_gemv_q4(codes, scales, x, False, idx, r)
    assert int(st.item()) == (1 << bq.BQ_ERR_EXPERT_INDEX if bad else 0)
    if B == 2:
        assert np.all(yn[1] == 0.0)
    check_tol(yn, y_ref, absy)
    assert int(torch.count_nonzero(ws).item()) == 0


def test_moe_single_expert_matches_dense():
    N, K, B = 200, 1024, 6
    codes, scales, x, _, _ = _moe_inputs(3, N, K, B, 1, 12, False)
    idx = np.full((B, 1), 1, dtype=np.int32)
    y, st = gpu_moe(codes, scales, x, False, idx, None)
    assert st == 0
    yd = gpu_gemv(4, codes[1], scales[1], x)
    np.testing.assert_array_equal(y[:, 0], yd)


# ------------------------------------------------------------ decode step ----
def _step_entries(fmt, specs, seed):
    """specs: list of (N, K, B, stage) -> (entries, numpy planes/x for the oracle)."""
    import torch
    entries, host = [], []
    for i, (N, K, B, stage) in enumerate(specs):
        w = synth.weights_f32(synth.key(seed, 82, i, 0, synth.KIND_W), N, K)
        codes, scales = quantize(fmt, w)
        x = synth.activations_f16_bits(synth.key(seed, 82, i, 0, synth.KIND_X), B, K)
        c, s, xt = dev(codes.view(np.uint8)), dev(scales), dev(x)
        y = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
        entries.append((bq.qmat(c, s, N, K), xt, y, stage))
        host.append((codes, scales, x))
    return entries, host


@pytest.mark.parametrize("fmt", [4, 8])
def test_step_plan_parity_and_repeat(fmt):
    import torch
    specs = [(3072, 2048, 1, 0), (512, 2048, 1, 0), (2048, 2048, 1, 1), (16384, 2048, 1, 2),
             (2048, 8192, 1, 3), (77, 288, 3, 3), (1000, 96, 8, 5), (16, 32, 2, 4),
             (4096, 4096, 8, 7), (300, 5120, 2, 6)]
    order = [5, 0, 9, 2, 7, 1, 4, 3, 8, 6]           # plan input order is irrelevant
    entries, host = _step_entries(fmt, [specs[i] for i in order], 7 + fmt)
    plan = bq.StepPlan(fmt, entries, DEV)
    assert plan.info.n_stages == 8
    st = new_status()
    plan.run(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    first = [e[2].cpu().numpy() for e in entries]
    for (W, x, y, stage), (codes, scales, xb), yg in zip(entries, host, first):
        y_ref, absy = oracle_gemv(fmt, codes, scales, xb)
        check_tol(yg, y_ref, absy)
    for _ in range(3):
        for e in entries:
            e[2].fill_(float("nan"))
        plan.run(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for e, y0 in zip(entries, first):
        assert np.array_equal(e[2].cpu().numpy(), y0)
    # barrier words (first 512 bytes) and band counters are back at zero;
    # the partial-sum area after them is scratch
    nbytes = 512 + -(-plan.info.max_stage_bands * 4 // 256) * 256
    assert int(plan.ws[:nbytes].view(torch.int32).abs().sum().item()) == 0


def test_step_barrier_orders_dependent_stages():
    """Stage 1 reads stage 0's output buffer (its fp32 bits as fp16 x).  Stage
    0 returns small integers (one-hot x, unit scales), whose fp32 bits are
    known, so stage 1's exact input is known; without the grid barrier stage 1
    would read the NaN fill."""
    import torch
    N0, K0 = 256, 64
    r = np.random.default_rng(3)
    q0 = r.integers(0, 16, size=(N0, K0))
    codes0 = np.zeros((N0, K0 // 2), dtype=np.uint8)
    for j in range(K0 // 32):
        for i in range(16):
            codes0[:, 16 * j + i] = q0[:, 32 * j + i] | (q0[:, 32 * j + i + 16] << 4)
    scales0 = np.zeros((N0, 8), dtype=np.uint16)
    scales0[:, :2] = 0x3C00
    x0 = np.zeros((1, K0), dtype=np.float16)
    x0[0, 0] = 1.0
    y0_expect = (q0[:, 0] - 8).astype(np.float32)
    x1_expect = y0_expect.view(np.uint16).reshape(1, 2 * N0)    # little-endian halves
    N1, K1 = 3000, 2 * N0
    w1 = synth.weights_f32(synth.key(0, 83, 1, 0, synth.KIND_W), N1, K1)
    codes1, scales1 = oracle.quantize_q4(w1)
    c0, s0, xt0 = dev(codes0), dev(scales0), dev(x0.view(np.uint16))
    y0 = torch.full((1, N0), float("nan"), dtype=torch.float32, device=DEV)
    c1, s1 = dev(codes1), dev(scales1)
    y1 = torch.full((1, N1), float("nan"), dtype=torch.float32, device=DEV)
    x1_alias = y0.view(torch.int16)                             # [1, 2*N0] fp16 bits
    plan = bq.StepPlan(4, [(bq.qmat(c0, s0, N0, K0), xt0, y0, 0),
                           (bq.qmat(c1, s1, N1, K1), x1_alias, y1, 1)], DEV)
    st = new_status()
    for _ in range(3):
        y0.fill_(float("nan"))
        y1.fill_(float("nan"))
        plan.run(st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert np.array_equal(y0.cpu().numpy()[0], y0_expect)
        y_ref, absy = oracle.gemv_q4(codes1, scales1, x1_expect)
        check_tol(y1.cpu().numpy(), y_ref, absy)


def test_step_reread_buffer_sees_later_writes():
    """A buffer is read as x by stage 0, overwritten (as y) by stage 1 and read
    again as x by stage 2, all in one launch: stage 2 must see stage 1's
    values, not a stale copy cached while stage 0 read it."""
    import torch
    N1, K1 = 256, 64
    r = np.random.default_rng(5)
    q1 = r.integers(0, 16, size=(N1, K1))
    codes1 = np.zeros((N1, K1 // 2), dtype=np.uint8)
    for j in range(K1 // 32):
        for i in range(16):
            codes1[:, 16 * j + i] = q1[:, 32 * j + i] | (q1[:, 32 * j + i + 16] << 4)
    scales1 = np.zeros((N1, 8), dtype=np.uint16)
    scales1[:, :2] = 0x3C00
    x1 = np.zeros((1, K1), dtype=np.float16)
    x1[0, 5] = 1.0
    y1_expect = (q1[:, 5] - 8).astype(np.float32)               # small integers
    X = torch.full((1, N1), 0.5, dtype=torch.float32, device=DEV)  # shared buffer
    K0 = 2 * N1                                                  # its fp16 view
    before = np.full((1, N1), 0.5, dtype=np.float32).view(np.uint16).reshape(1, K0)
    after = y1_expect.view(np.uint16).reshape(1, K0)
    w0 = synth.weights_f32(synth.key(0, 85, 0, 0, synth.KIND_W), 1024, K0)
    w2 = synth.weights_f32(synth.key(0, 85, 2, 0, synth.KIND_W), 2048, K0)
    c0, s0 = oracle.quantize_q4(w0)
    c2, s2 = oracle.quantize_q4(w2)
    y0 = torch.empty((1, 1024), dtype=torch.float32, device=DEV)
    y2 = torch.empty((1, 2048), dtype=torch.float32, device=DEV)
    tc0, ts0, tc1, ts1, tc2, ts2 = dev(c0), dev(s0), dev(codes1), dev(scales1), dev(c2), dev(s2)
    xt1 = dev(x1.view(np.uint16))
    plan = bq.StepPlan(4, [(bq.qmat(tc0, ts0, 1024, K0), X.view(torch.int16), y0, 0),
                           (bq.qmat(tc1, ts1, N1, K1), xt1, X, 1),
                           (bq.qmat(tc2, ts2, 2048, K0), X.view(torch.int16), y2, 2)], DEV)
    st = new_status()
    for _ in range(3):
        X.fill_(0.5)
        plan.run(st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        r0, a0 = oracle.gemv_q4(c0, s0, before)
        r2, a2 = oracle.gemv_q4(c2, s2, after)
        check_tol(y0.cpu().numpy(), r0, a0)
        assert np.array_equal(X.cpu().numpy()[0], y1_expect)
        check_tol(y2.cpu().numpy(), r2, a2)

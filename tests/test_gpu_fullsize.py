"""Parity at the full workload sizes, in the launch configuration bench.py
times (the whole decode step as one plan, resident weights quantised on the
device).

The oracle cannot redo multi-GB steps, so each test checks every output row
of the first and the last layer and a seeded sample of rows of every other
matrix (for the fused feed-forward stage: of its SwiGLU output h).  For each checked row the fp32 weights are regenerated from the same
seeded generator, quantised by the oracle, compared bit-for-bit with the
device-quantised planes the kernel streamed, and multiplied by the oracle in
fp64 against the same activations.  No oracle input comes from the CUDA path:
weights and activations come from the input generators; the planes the GPU
used are only *compared* with the oracle's.
"""
import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import DEV, check_swiglu, check_tol, dev, new_status

pytestmark = pytest.mark.gpu


def _rows_for(layer, layers, N, every, rng):
    if layer in (0, layers - 1) or every <= 1:
        return np.arange(N)
    k = max(1, N // every)
    return np.sort(rng.choice(N, size=k, replace=False))


def _regen_rows(wl, seed, layer, m, rows, K, N_mat):
    """fp32 rows of matrix m of a layer, regenerated from its seed key on the GPU."""
    import torch
    w = synth.weights_f32_torch(synth.key(seed, wl.wid, layer, wl.mats.index(m), synth.KIND_W),
                                N_mat, K, DEV)
    out = w[torch.as_tensor(rows, device=DEV)].cpu().numpy()
    del w
    return out


def _quant(fmt, w):
    return oracle.quantize_q4(w) if fmt == 4 else oracle.quantize_q8(w)


def _gemv(fmt, codes, scales, xb):
    return (oracle.gemv_q4 if fmt == 4 else oracle.gemv_q8)(codes, scales, xb, nthreads=8)


def _check_step(wl, every, seed=0):
    """Run the decode step once; check sampled rows of every matrix.  The fused
    feed-forward stage (gate|up in SwiGLU pair order) is checked on its fp16
    output h against the oracle's SwiGLU of the oracle's gate and up GEMVs;
    the down stage then reads the h the GPU produced."""
    import torch
    import bench
    step = bench.DenseStep(wl, torch.device(DEV), seed=seed)
    step.build_plan()
    st = new_status()
    step.plan.run(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(step.status.item()) == 0
    rng = np.random.default_rng([seed, wl.wid, 12345])
    stages = bench.fused_stages(wl)
    worst = 0.0
    li = 0
    for layer in range(wl.layers):
        for s, group in stages:
            q, x, y, label, _, epi = step.launches[li]
            li += 1
            codes_d, scales_d = q._refs
            K = group[0].K
            xb = x.cpu().numpy().view(np.uint16)
            if epi == bq.BQ_EPI_SWIGLU:
                F = sum(m.N for m in group) // 2
                rows = _rows_for(layer, wl.layers, F, every, rng)
                if len(group) == 2:
                    wg = _regen_rows(wl, seed, layer, group[0], rows, K, F)
                    wu = _regen_rows(wl, seed, layer, group[1], rows, K, F)
                else:
                    wg = _regen_rows(wl, seed, layer, group[0], rows, K, 2 * F)
                    wu = _regen_rows(wl, seed, layer, group[0], rows + F, K, 2 * F)
                (cg, sg), (cu, su) = _quant(wl.fmt, wg), _quant(wl.fmt, wu)
                rg = torch.as_tensor(16 * (rows // 8) + rows % 8, device=DEV)   # pair order
                for r_dev, c_ref, s_ref, what in ((rg, cg, sg, "gate"), (rg + 8, cu, su, "up")):
                    assert np.array_equal(codes_d[r_dev].cpu().numpy(), c_ref.view(np.uint8)), \
                        f"{label} L{layer}: {what} codes differ"
                    assert np.array_equal(scales_d[r_dev].cpu().numpy().view(np.uint16), s_ref), \
                        f"{label} L{layer}: {what} scales differ"
                g, ag = _gemv(wl.fmt, cg, sg, xb)
                u, au = _gemv(wl.fmt, cu, su, xb)
                hb = y.cpu().numpy().view(np.uint16)[:, rows]
                worst = max(worst, check_swiglu(hb, g, ag, u, au))
                continue
            yg = y.cpu().numpy()
            r0 = 0
            for m in group:
                rows = _rows_for(layer, wl.layers, m.N, every, rng)
                wr = _regen_rows(wl, seed, layer, m, rows, m.K, m.N)
                oc, os_ = _quant(wl.fmt, wr)
                sel = torch.as_tensor(rows + r0, device=DEV)
                gc = codes_d[sel].cpu().numpy()
                gs = scales_d[sel].cpu().numpy().view(np.uint16)
                assert np.array_equal(gc, oc.view(np.uint8)), f"{label} L{layer}: codes differ"
                assert np.array_equal(gs, os_), f"{label} L{layer}: scales differ"
                yr, ar = _gemv(wl.fmt, oc, os_, xb)
                worst = max(worst, check_tol(yg[:, rows + r0], yr, ar))
                r0 += m.N
    return worst


def test_single_q8_2048_all_rows():
    """One 2048 x 2048 Q8 matrix, batch 1: every row."""
    import torch
    wl = synth.SINGLE_Q8
    N, K = 2048, 2048
    w = synth.weights_f32(synth.key(0, wl.wid, 0, 0, synth.KIND_W), N, K)
    codes, scales = oracle.quantize_q8(w)
    x = synth.activations_f16_bits(synth.key(0, wl.wid, 0, 0, synth.KIND_X), 1, K)
    c, s, xt = dev(codes.view(np.uint8)), dev(scales), dev(x)
    y = torch.empty((1, N), dtype=torch.float32, device=DEV)
    ws = bq.workspace(bq.lib().bq_gemv_workspace_bytes(N, K), DEV)
    st = new_status()
    bq.gemv(8, bq.qmat(c, s, N, K), xt, y, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    yr, ar = oracle.gemv_q8(codes, scales, x, nthreads=8)
    check_tol(y.cpu().numpy(), yr, ar)


def test_dense16_h2048_step():
    """16-layer decoder (hidden 2048, FFN 8192), Q4, batch 1, as one plan."""
    _check_step(synth.DENSE_H2048, every=16)


@pytest.mark.parametrize("fmt", [4, 8])
def test_dense36_h4096_step_batch8(fmt):
    """36 distinct copies of a hidden-4096 layer, batch 8, as one plan."""
    _check_step(synth.dense_h4096(fmt, 8), every=128)


def test_dense64_h5120_step():
    """64-layer decoder (hidden 5120, FFN 25600, ~16 GB Q4), batch 1, as one plan."""
    _check_step(synth.DENSE_H5120, every=1024)


@pytest.mark.parametrize("B", [1, 8])
def test_moe_layer_full(B):
    """One routed-expert layer: 128 experts, gate|up 1536 x 2048 per expert
    (per-slot outputs) and down 2048 x 768 (combined with the routing
    weights), top-8, every output row of every routed slot."""
    import torch
    wl = synth.moe_h2048(B)
    E, topk, layer = wl.E, wl.topk, 0
    idx, r = synth.routing(synth.key(0, wl.wid, layer, 0, synth.KIND_IDX),
                           synth.key(0, wl.wid, layer, 0, synth.KIND_LOGIT), B, E, topk)
    st = new_status()
    for part, (N, K) in (("gateup", wl.gateup()), ("down", wl.down())):
        mid = 0 if part == "gateup" else 1
        ldS = bq.scales_ld(K)
        codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=DEV)
        scales = torch.empty((E, N, ldS), dtype=torch.int16, device=DEV)
        for e in range(E):
            w = synth.weights_f32_torch(synth.key(0, wl.wid, layer, mid * 1000 + e, synth.KIND_W),
                                        N, K, DEV)
            bq.quantize_dev(4, w, codes[e], scales[e], st)
        if part == "gateup":
            x = synth.activations_f16_torch(synth.key(0, wl.wid, layer, 0, synth.KIND_X), (B, K), DEV)
            per_slot, rr = False, None
            y = torch.empty((B, topk, N), dtype=torch.float32, device=DEV)
        else:
            x = synth.activations_f16_torch(synth.key(0, wl.wid, layer, 1, synth.KIND_H),
                                            (B, topk, K), DEV)
            per_slot, rr = True, r
            y = torch.empty((B, N), dtype=torch.float32, device=DEV)
        ws = bq.workspace(bq.lib().bq_moe_workspace_bytes(N, K, B, topk, E), DEV)
        it, rt = dev(idx), dev(rr) if rr is not None else None
        bq.moe_gemv_q4(bq.qmat(codes, scales, N, K), E, N * K // 2, N * ldS, x, per_slot, it, rt,
                       y, ws, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        used = sorted(set(idx.ravel().tolist()))
        oc = np.zeros((E, N, K // 2), dtype=np.uint8)
        os_ = np.zeros((E, N, ldS), dtype=np.uint16)
        for e in used:
            w = synth.weights_f32_torch(synth.key(0, wl.wid, layer, mid * 1000 + e, synth.KIND_W),
                                        N, K, DEV).cpu().numpy()
            oc[e], os_[e] = oracle.quantize_q4(w)
            assert np.array_equal(codes[e].cpu().numpy(), oc[e])
            assert np.array_equal(scales[e].cpu().numpy().view(np.uint16), os_[e])
        xb = x.cpu().numpy().view(np.uint16)
        yr, ar, bad = oracle.moe_gemv_q4(oc, os_, xb, per_slot, idx, rr, nthreads=8)
        assert not bad
        check_tol(y.cpu().numpy(), yr, ar)

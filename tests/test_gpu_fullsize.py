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
from tests.gpu_helpers import DEV, check_swiglu, check_tol, dev, new_status, pair_order

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
    return {2: oracle.quantize_q2, 3: oracle.quantize_q3, 4: oracle.quantize_q4,
            5: oracle.quantize_q5, 6: oracle.quantize_q6, 8: oracle.quantize_q8}[fmt](w)


def _gemv(fmt, codes, scales, xb):
    fn = {2: oracle.gemv_q2, 3: oracle.gemv_q3, 4: oracle.gemv_q4, 5: oracle.gemv_q5,
          6: oracle.gemv_q6, 8: oracle.gemv_q8}[fmt]
    return fn(codes, scales, xb, nthreads=8)


def _check_step(wl, every, seed=0, engines=("step",)):
    """Run the decode step once per engine; check sampled rows of every
    matrix after each.  The fused feed-forward stage (gate|up in SwiGLU pair
    order) is checked on its fp16 output h against the oracle's SwiGLU of the
    oracle's gate and up GEMVs; the down stage then reads the h the GPU
    produced.  Every output buffer is filled with NaN before each engine runs,
    so each engine must write every output itself.  engines: "step" (one plan,
    a single cooperative launch) and/or "graph" (the per-matrix launch chain
    with static weights that bench.py times)."""
    import torch
    import bench
    step = bench.DenseStep(wl, torch.device(DEV), seed=seed)
    worst = 0.0
    for engine in engines:
        step.y_all.fill_(float("nan"))
        step.h_all.fill_(float("nan"))
        if engine == "step":
            step.build_plan()
            st = new_status()
            step.plan.run(st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
        else:       # the per-matrix launch chain bench.py's graph engine times
            step.launch(torch.cuda.current_stream())
            torch.cuda.synchronize()
        assert int(step.status.item()) == 0
        worst = max(worst, _check_outputs(wl, step, every, seed))
    return worst


def _check_outputs(wl, step, every, seed):
    import torch
    import bench
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


def test_dense16_h2048_step_every_row():
    """16-layer decoder (hidden 2048, FFN 8192), Q4, batch 1: every output row
    of every layer, as one plan and as the chain of per-matrix launches with
    static weights."""
    _check_step(synth.DENSE_H2048, every=1, engines=("step", "graph"))


@pytest.mark.parametrize("fmt", [6, 5, 3, 2])
def test_dense16_h2048_other_formats_chain(fmt):
    """The 16-layer hidden-2048 decoder in Q6, Q5, Q3 and Q2, as the launch chain."""
    _check_step(synth.dense_h2048(fmt), every=16, engines=("graph",))


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("B", [1, 2, 4, 8])
def test_dense36_h4096_step(fmt, B):
    """36 distinct copies of a hidden-4096 layer at batch 1, 2, 4 and 8, in Q4
    and Q8, as the launch chain: every row of the first and last layer, 1/128
    of the rows of every other matrix."""
    _check_step(synth.dense_h4096(fmt, B), every=128, engines=("graph",))


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("B", [16, 32])
def test_verify36_h4096_step(fmt, B):
    """The hidden-4096 layer's matrices (36 distinct copies) as a batched
    verification step at B = 16 and 32 through the tensor-core GEMM: every row
    of the first and last layer, 1/128 of the rows of every other matrix."""
    _check_step(synth.verify_h4096(fmt, B), every=128, engines=("graph",))


def test_dense64_h5120_step():
    """64-layer decoder (hidden 5120, FFN 25600, ~16 GB Q4), batch 1: as the
    launch chain bench.py times, and as one plan."""
    _check_step(synth.DENSE_H5120, every=1024, engines=("graph", "step"))


@pytest.mark.parametrize("B,layers", [(1, None), (8, (0, 47))])
def test_moe_step_full(B, layers):
    """The routed-expert decode step built exactly as the benchmark builds it
    (48 layers of 128 experts, gate|up 1536 x 2048 per expert in SwiGLU pair
    order, down 2048 x 768, top-8), run once as the benchmark's launch
    sequence: per-slot h = silu(gate) * up of every routed slot, and y =
    down(h) combined with the routing weights, against the oracle on every
    routed expert -- of all 48 layers at batch 1, of the first and last layer
    at batch 8 (52 distinct experts a layer)."""
    import torch
    import bench
    wl = synth.moe_h2048(B)
    step = bench.MoEStep(wl, torch.device(DEV))
    step.h_all.fill_(float("nan"))
    step.y_all.fill_(0xFF)               # NaN bit patterns in every fp32 output
    step.launch(torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    for layer in (range(wl.layers) if layers is None else layers):
        _check_moe_layer(wl, step, layer)


def _check_moe_layer(wl, step, layer, seed=0):
    import torch
    E, topk = wl.E, wl.topk
    (Ng, Kg), (Nd, Kd) = wl.gateup(), wl.down()
    F = Ng // 2
    stacks, idx_d, r_d, x_d, h_d, y_d = step.layers[layer]
    idx, r = idx_d.cpu().numpy(), r_d.cpu().numpy()
    used = sorted(set(idx.ravel().tolist()))
    planes = []
    for mid, (N, K) in ((0, (Ng, Kg)), (1, (Nd, Kd))):
        w = synth.weights_f32_torch(synth.key(seed, wl.wid, layer, mid, synth.KIND_W), E * N, K, DEV)
        rows = np.concatenate([np.arange(e * N, (e + 1) * N) for e in used])
        wu = w[torch.as_tensor(rows, device=DEV)].cpu().numpy().reshape(len(used), N, K)
        del w
        ldS = bq.scales_ld(K)
        codes_d, scales_d = stacks[mid][0]._refs
        parts = []
        for half in ((0, F), (F, 2 * F)) if mid == 0 else ((0, N),):
            c = np.zeros((E, half[1] - half[0], K // 2), dtype=np.uint8)
            sc = np.zeros((E, half[1] - half[0], ldS), dtype=np.uint16)
            for j, e in enumerate(used):
                c[e], sc[e] = oracle.quantize_q4(wu[j, half[0]:half[1]])
            parts.append((c, sc))
        for j, e in enumerate(used):        # the device planes are the oracle's, bit for bit
            if mid == 0:
                want_c = pair_order(parts[0][0][e], parts[1][0][e])
                want_s = pair_order(parts[0][1][e], parts[1][1][e])
            else:
                want_c, want_s = parts[0][0][e], parts[0][1][e]
            assert np.array_equal(codes_d[e].cpu().numpy(), want_c), f"L{layer} expert {e} codes"
            assert np.array_equal(scales_d[e].cpu().numpy().view(np.uint16), want_s), \
                f"L{layer} expert {e} scales"
        planes.append(parts)
    xb = x_d.cpu().numpy().view(np.uint16)
    (cg, sg), (cu, su) = planes[0]
    g, ag, bad = oracle.moe_gemv_q4(cg, sg, xb, False, idx, nthreads=8)
    u, au, _ = oracle.moe_gemv_q4(cu, su, xb, False, idx, nthreads=8)
    assert not bad
    hb = h_d.cpu().numpy().view(np.uint16)
    check_swiglu(hb, g, ag, u, au)
    (cd, sd), = planes[1]
    yr, ar, _ = oracle.moe_gemv_q4(cd, sd, hb, True, idx, r, nthreads=8)
    check_tol(y_d.cpu().numpy(), yr, ar)

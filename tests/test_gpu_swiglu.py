"""The fused feed-forward path: a gate|up GEMV in SwiGLU pair order whose
epilogue writes h = silu(gate) * up as fp16, and the down GEMV reading h,
against the oracle (gate / up / down GEMVs in fp64, SwiGLU in fp64 rounded
once to fp16)."""
import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import (DEV, check_swiglu, check_tol, dev, new_status, oracle_gemv,
                               pair_order)

pytestmark = pytest.mark.gpu


def _quant(fmt, w):
    return oracle.quantize_q4(w) if fmt == 4 else oracle.quantize_q8(w)


def _ffn_inputs(fmt, F, K, B, seed):
    wg = synth.weights_f32(synth.key(seed, 82, 0, 0, synth.KIND_W), F, K)
    wu = synth.weights_f32(synth.key(seed, 82, 0, 1, synth.KIND_W), F, K)
    (cg, sg), (cu, su) = _quant(fmt, wg), _quant(fmt, wu)
    x = synth.activations_f16_bits(synth.key(seed, 82, 0, 0, synth.KIND_X), B, K)
    return cg, sg, cu, su, x


@pytest.mark.parametrize("fmt,flags", [(4, 0), (4, bq.BQ_GEMV_ROWS16), (4, bq.BQ_GEMV_ROWS32),
                                       (8, 0)])
@pytest.mark.parametrize("F,K", [(8, 256), (24, 800), (200, 2048), (1024, 512)])
@pytest.mark.parametrize("B", [1, 3, 4, 8])
def test_gemv_swiglu_epilogue(fmt, flags, F, K, B):
    """The SwiGLU epilogue with either Q4 chunk height (a 16-row tile holds 8
    gate and the same 8 up rows in both)."""
    import torch
    cg, sg, cu, su, x = _ffn_inputs(fmt, F, K, B, 5)
    codes, scales = pair_order(cg, cu), pair_order(sg, su)
    N = 2 * F
    c, s, xt = dev(codes.view(np.uint8)), dev(scales), dev(x)
    h = torch.full((B, F), float("nan"), dtype=torch.float16, device=DEV)
    ws = bq.workspace(bq.lib().bq_gemv_workspace_bytes(N, K), DEV)
    st = new_status()
    bq.gemv(fmt, bq.qmat(c, s, N, K), xt, h, ws, st, epilogue=bq.BQ_EPI_SWIGLU, flags=flags)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g, ag = oracle_gemv(fmt, cg, sg, x)
    u, au = oracle_gemv(fmt, cu, su, x)
    check_swiglu(h.cpu().numpy().view(np.uint16), g, ag, u, au)


@pytest.mark.parametrize("fmt", [4, 8])
def test_launch_chain_fused_ffn_static_weights(fmt):
    """The feed-forward block as two back-to-back bq_gemv_ex launches with the
    static-weights flag (each launch loads weights before waiting for the
    previous one): down must still read the h gate|up wrote.  Three rounds
    with different inputs, no host sync in between."""
    import torch
    F, H, B = 512, 1024, 3
    cg, sg, cu, su, _ = _ffn_inputs(fmt, F, H, B, 8)
    wd = synth.weights_f32(synth.key(8, 82, 0, 2, synth.KIND_W), H, F)
    cd, sd = _quant(fmt, wd)
    W1 = bq.qmat(dev(pair_order(cg, cu).view(np.uint8)), dev(pair_order(sg, su)), 2 * F, H)
    W2 = bq.qmat(dev(cd.view(np.uint8)), dev(sd), H, F)
    ws = bq.workspace(bq.lib().bq_gemv_workspace_bytes(2 * F, max(H, F)) * 2, DEV)
    st = new_status()
    xs = [synth.activations_f16_bits(synth.key(8 + r, 82, 1, 0, synth.KIND_X), B, H) for r in range(3)]
    hs = [torch.full((B, F), float("nan"), dtype=torch.float16, device=DEV) for _ in range(3)]
    ys = [torch.full((B, H), float("nan"), dtype=torch.float32, device=DEV) for _ in range(3)]
    for r in range(3):
        bq.gemv(fmt, W1, dev(xs[r]), hs[r], ws, st, epilogue=bq.BQ_EPI_SWIGLU,
                flags=bq.BQ_GEMV_STATIC_WEIGHTS)
        bq.gemv(fmt, W2, hs[r], ys[r], ws, st, flags=bq.BQ_GEMV_STATIC_WEIGHTS)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for r in range(3):
        g, ag = oracle_gemv(fmt, cg, sg, xs[r])
        u, au = oracle_gemv(fmt, cu, su, xs[r])
        hb = hs[r].cpu().numpy().view(np.uint16)
        check_swiglu(hb, g, ag, u, au)
        yr, ar = oracle_gemv(fmt, cd, sd, hb)
        check_tol(ys[r].cpu().numpy(), yr, ar)


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("F,H", [(256, 512), (768, 2048)])
def test_step_fused_ffn(fmt, F, H):
    """One feed-forward block as a two-stage plan: gate|up + SwiGLU (stage 0)
    writes h, down (stage 1) reads it; run twice (the plan is reusable)."""
    import torch
    B = 2
    cg, sg, cu, su, x = _ffn_inputs(fmt, F, H, B, 6)
    wd = synth.weights_f32(synth.key(6, 82, 0, 2, synth.KIND_W), H, F)
    cd, sd = _quant(fmt, wd)
    c1, s1 = dev(pair_order(cg, cu).view(np.uint8)), dev(pair_order(sg, su))
    c2, s2 = dev(cd.view(np.uint8)), dev(sd)
    xt = dev(x)
    h = torch.full((B, F), float("nan"), dtype=torch.float16, device=DEV)
    y = torch.full((B, H), float("nan"), dtype=torch.float32, device=DEV)
    plan = bq.StepPlan(fmt, [(bq.qmat(c1, s1, 2 * F, H), xt, h, 0, bq.BQ_EPI_SWIGLU),
                             (bq.qmat(c2, s2, H, F), h, y, 1)], DEV)
    st = new_status()
    for _ in range(2):
        plan.run(st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        hb = h.cpu().numpy().view(np.uint16)
        g, ag = oracle_gemv(fmt, cg, sg, x)
        u, au = oracle_gemv(fmt, cu, su, x)
        check_swiglu(hb, g, ag, u, au)
        yr, ar = oracle_gemv(fmt, cd, sd, hb)      # down on the h the GPU produced
        check_tol(y.cpu().numpy(), yr, ar)


def _expert_ffn(E, F, H, seed):
    """Per expert: gate / up (F x H) and down (H x F) Q4 planes."""
    cg, sg, cu, su, cd, sd = [], [], [], [], [], []
    for e in range(E):
        for lst_c, lst_s, mid, n, k in ((cg, sg, 0, F, H), (cu, su, 1, F, H), (cd, sd, 2, H, F)):
            c, s = oracle.quantize_q4(synth.weights_f32(synth.key(seed, 83, e, mid, synth.KIND_W), n, k))
            lst_c.append(c)
            lst_s.append(s)
    return [np.stack(a) for a in (cg, sg, cu, su, cd, sd)]


@pytest.mark.parametrize("B,topk,E", [(1, 8, 16), (4, 8, 16), (8, 8, 32), (3, 2, 5)])
def test_moe_expert_ffn_fused(B, topk, E):
    """Routed-expert feed-forward block: per-slot gate|up with the SwiGLU
    epilogue writes h [B][topk][F] (fp16), then down reads it per slot and
    combines with the routing weights.  One slot id is out of range: its h is
    zero and the status flags it."""
    import torch
    F, H = 96, 512
    cg, sg, cu, su, cd, sd = _expert_ffn(E, F, H, 7)
    codes_gu = np.stack([pair_order(cg[e], cu[e]) for e in range(E)])
    scales_gu = np.stack([pair_order(sg[e], su[e]) for e in range(E)])
    x = synth.activations_f16_bits(synth.key(7, 83, 0, 0, synth.KIND_X), B, H)
    idx, r = synth.routing(synth.key(7, 83, 0, 0, synth.KIND_IDX),
                           synth.key(7, 83, 0, 0, synth.KIND_LOGIT), B, E, topk)
    idx[B - 1, topk - 1] = E + 3
    ldS_h, ldS_f = scales_gu.shape[2], sd.shape[2]
    c1, s1, c2, s2 = (dev(codes_gu.view(np.uint8)), dev(scales_gu), dev(cd.view(np.uint8)), dev(sd))
    xt, it, rt = dev(x), dev(idx), dev(r)
    h = torch.full((B, topk, F), float("nan"), dtype=torch.float16, device=DEV)
    y = torch.full((B, H), float("nan"), dtype=torch.float32, device=DEV)
    ws1 = bq.workspace(bq.lib().bq_moe_workspace_bytes(2 * F, H, B, topk, E), DEV)
    ws2 = bq.workspace(bq.lib().bq_moe_workspace_bytes(H, F, B, topk, E), DEV)
    st = new_status()
    bq.moe_gemv_q4(bq.qmat(c1, s1, 2 * F, H), E, 2 * F * H // 2, 2 * F * ldS_h, xt, False, it,
                   None, h, ws1, st, epilogue=bq.BQ_EPI_SWIGLU)
    bq.moe_gemv_q4(bq.qmat(c2, s2, H, F), E, H * F // 2, H * ldS_f, h, True, it, rt, y, ws2, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 1 << bq.BQ_ERR_EXPERT_INDEX
    hb = h.cpu().numpy().view(np.uint16)
    assert np.all(hb[B - 1, topk - 1] == 0)
    g, ag, bad = oracle.moe_gemv_q4(cg, sg, x, False, idx)
    u, au, _ = oracle.moe_gemv_q4(cu, su, x, False, idx)
    assert bad
    check_swiglu(hb, g, ag, u, au)
    yr, ar, _ = oracle.moe_gemv_q4(cd, sd, hb, True, idx, r)      # down on the GPU's h
    check_tol(y.cpu().numpy(), yr, ar)

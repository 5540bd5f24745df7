"""Shared helpers of the GPU parity tests: upload numpy planes, call the CUDA
path through the C ABI binding, and check the tolerance

    |y - y_ref| <= 1e-3 * sum_k |deq(w) x| + 1e-5      (per output element)

against the fp64 oracle.  For the SwiGLU epilogue, h = silu(g) * u is checked
against the oracle's fp16 h with that tolerance carried through silu(g) * u
(|d silu / dz| <= 1.1 everywhere) plus one fp16 unit in the last place for
the two roundings to fp16."""
import numpy as np

import oracle
from quantised_weight_gemv_b200 import bq

DEV = "cuda:0"
REL, ABS = 1e-3, 1e-5


def dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(DEV)


def new_status():
    import torch
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def gpu_gemv(fmt, codes, scales, x_bits, ws=None, status=None, flags=0):
    """Run bq_gemv_q{fmt} (bq_gemv_ex when flags are given) on numpy planes /
    fp16 bits; returns fp32 [B, N]."""
    import torch
    N = codes.shape[0]
    K = {2: codes.shape[1] * 4, 3: codes.shape[1] * 8 // 3, 4: codes.shape[1] * 2,
         5: codes.shape[1] * 8 // 5, 6: codes.shape[1] * 4 // 3, 8: codes.shape[1]}[fmt]
    x_bits = np.atleast_2d(x_bits)
    B = x_bits.shape[0]
    c, s, x = dev(codes.view(np.uint8)), dev(scales), dev(x_bits)
    y = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = ws if ws is not None else bq.workspace(bq.lib().bq_gemv_workspace_bytes(N, K), DEV)
    st = status if status is not None else new_status()
    bq.gemv(fmt, bq.qmat(c, s, N, K), x, y, ws, st, flags=flags)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item()):#x}"
    return y.cpu().numpy()


def check_tol(y, y_ref, absy):
    """Assert the per-element tolerance; return the max error/bound ratio."""
    y = np.asarray(y, dtype=np.float64)
    assert np.all(np.isfinite(y))
    err = np.abs(y - y_ref)
    bound = REL * absy + ABS
    ratio = float(np.max(err / bound)) if err.size else 0.0
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{len(bad)} outputs out of tolerance, first {bad[:5].tolist()}, max ratio {ratio}"
    return ratio


def oracle_gemv(fmt, codes, scales, x_bits, nthreads=8):
    fn = {2: oracle.gemv_q2, 3: oracle.gemv_q3, 4: oracle.gemv_q4, 5: oracle.gemv_q5,
          6: oracle.gemv_q6, 8: oracle.gemv_q8}[fmt]
    return fn(codes, scales, x_bits, nthreads=nthreads)


def quantize(fmt, w):
    return {2: oracle.quantize_q2, 3: oracle.quantize_q3, 4: oracle.quantize_q4,
            5: oracle.quantize_q5, 6: oracle.quantize_q6, 8: oracle.quantize_q8}[fmt](w)


def pair_order(gate, up):
    """Rows of the gate and up projections (each [F, ...], F a multiple of 8)
    interleaved 8 at a time: SwiGLU pair order."""
    F = gate.shape[0]
    assert F % 8 == 0 and up.shape == gate.shape
    g = gate.reshape(F // 8, 8, *gate.shape[1:])
    u = up.reshape(F // 8, 8, *up.shape[1:])
    return np.stack([g, u], axis=1).reshape(2 * F, *gate.shape[1:])


def check_swiglu(h_bits, g, absg, u, absu):
    """Assert the SwiGLU output h (fp16 bits [B, F]) against the oracle."""
    h = np.asarray(h_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    h_ref = oracle.swiglu_f16(g, u).view(np.float16).astype(np.float64)
    assert np.all(np.isfinite(h))
    tol_g = REL * absg + ABS
    tol_u = REL * absu + ABS
    sil = np.array([oracle.silu(z) for z in np.ravel(g)]).reshape(g.shape)
    bound = 1.1 * np.abs(u) * tol_g + np.abs(sil) * tol_u + tol_g * tol_u \
        + 2.0 ** -10 * np.abs(h_ref) + 2.0 ** -24
    err = np.abs(h - h_ref)
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{len(bad)} h out of tolerance, first {bad[:5].tolist()}"
    return float(np.max(err / bound)) if err.size else 0.0

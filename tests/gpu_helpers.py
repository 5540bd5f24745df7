"""Shared helpers of the GPU parity tests: upload numpy planes, call the CUDA
path through the C ABI binding, and check the tolerance

    |y - y_ref| <= 1e-3 * sum_k |deq(w) x| + 1e-5      (per output element)

against the fp64 oracle."""
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


def gpu_gemv(fmt, codes, scales, x_bits, ws=None, status=None):
    """Run bq_gemv_q{fmt} on numpy planes / fp16 bits; returns fp32 [B, N]."""
    import torch
    N = codes.shape[0]
    K = codes.shape[1] * (2 if fmt == 4 else 1)
    x_bits = np.atleast_2d(x_bits)
    B = x_bits.shape[0]
    c, s, x = dev(codes.view(np.uint8)), dev(scales), dev(x_bits)
    y = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = ws if ws is not None else bq.workspace(bq.lib().bq_gemv_workspace_bytes(N, K), DEV)
    st = status if status is not None else new_status()
    bq.gemv(fmt, bq.qmat(c, s, N, K), x, y, ws, st)
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
    return (oracle.gemv_q4 if fmt == 4 else oracle.gemv_q8)(codes, scales, x_bits, nthreads=nthreads)


def quantize(fmt, w):
    return oracle.quantize_q4(w) if fmt == 4 else oracle.quantize_q8(w)

"""GPU parity of the Q6 and Q5 formats (fp16 scale absmax/31 or absmax/15,
6- or 5-bit codes as a low-nibble plane plus a 2- or 1-bit plane) against
the fp64 oracle, through bq_gemv_ex and the device quantisers.  Tolerance as
for Q4/Q8: |y - y_ref| <= 1e-3 * sum_k |deq(w) x| + 1e-5 per output; packing
bit-exact."""
import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import (DEV, check_swiglu, check_tol, dev, gpu_gemv, new_status,
                               oracle_gemv, pair_order, quantize)

pytestmark = pytest.mark.gpu

# Q6: K a multiple of 64 (rows of 3K/4 bytes stay 16-byte aligned); Q5: of
# 128 (rows of 5K/8 bytes).  Several chunks, ragged bands and a ragged last
# chunk along K; 1024 x 8192 sums its bands across CTAs in clusters.
SHAPES = {6: [(1, 64), (15, 64), (16, 256), (17, 320), (33, 832), (100, 2048), (257, 4160),
              (1000, 128), (4, 25600), (48, 768), (1024, 8192)],
          5: [(1, 128), (15, 128), (16, 256), (17, 384), (33, 896), (100, 2048), (257, 4224),
              (1000, 128), (4, 25600), (48, 768), (1024, 8192)]}
CASES = [(f, n, k) for f in (6, 5) for n, k in SHAPES[f]]


@pytest.mark.parametrize("fmt,N,K", CASES)
@pytest.mark.parametrize("B", [1, 3, 8])
@pytest.mark.parametrize("flags", [0, bq.BQ_GEMV_STATIC_WEIGHTS])
def test_gemv_parity(fmt, N, K, B, flags):
    w = synth.weights_f32(synth.key(fmt, 84, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(fmt, 84, N, K, synth.KIND_X), B, K)
    y = gpu_gemv(fmt, codes, scales, x, flags=flags)
    y_ref, absy = oracle_gemv(fmt, codes, scales, x)
    check_tol(y, y_ref, absy)


@pytest.mark.parametrize("fmt", [6, 5])
def test_one_hot_is_exact_column(fmt):
    """x = e_k returns column k of deq(W) exactly (one product, fp32-exact)."""
    N, K = 64, 256
    w = synth.weights_f32(synth.key(fmt, 85, 0, 0, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    deq = (oracle.dequantize_q6 if fmt == 6 else oracle.dequantize_q5)(codes, scales)
    one = np.float16(1.0).view(np.uint16)
    for k0 in range(0, K, 8):
        x = np.zeros((8, K), dtype=np.uint16)
        x[np.arange(8), k0 + np.arange(8)] = one
        y = gpu_gemv(fmt, codes, scales, x)
        assert np.array_equal(y.astype(np.float64), deq[:, k0:k0 + 8].T)


@pytest.mark.parametrize("fmt", [6, 5])
def test_device_quantiser_bit_exact(fmt):
    import torch
    N, K = 300, 1024
    w = synth.weights_f32(synth.key(fmt, 86, 0, 0, synth.KIND_W), N, K)
    w[0, :32] = 0.0
    w[1, :32] = 1e-9
    oc, os_ = quantize(fmt, w)
    wd = torch.from_numpy(w).to(DEV)
    c = torch.zeros(oc.shape, dtype=torch.uint8, device=DEV)
    s = torch.zeros((N, bq.scales_ld(K)), dtype=torch.int16, device=DEV)
    st = new_status()
    bq.quantize_dev(fmt, wd, c, s, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(c.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), os_)


@pytest.mark.parametrize("fmt", [6, 5])
@pytest.mark.parametrize("F,K,B", [(8, 256, 1), (200, 2048, 3), (1024, 512, 8)])
def test_swiglu_epilogue(fmt, F, K, B):
    import torch
    wg = synth.weights_f32(synth.key(1, 87, F, K, synth.KIND_W), F, K)
    wu = synth.weights_f32(synth.key(2, 87, F, K, synth.KIND_W), F, K)
    (cg, sg), (cu, su) = quantize(fmt, wg), quantize(fmt, wu)
    x = synth.activations_f16_bits(synth.key(1, 87, F, K, synth.KIND_X), B, K)
    codes, scales = pair_order(cg, cu), pair_order(sg, su)
    N = 2 * F
    h = torch.full((B, F), float("nan"), dtype=torch.float16, device=DEV)
    ws = bq.workspace(bq.lib().bq_gemv_workspace_bytes(N, K), DEV)
    st = new_status()
    bq.gemv(fmt, bq.qmat(dev(codes), dev(scales), N, K), dev(x), h, ws, st,
            epilogue=bq.BQ_EPI_SWIGLU)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g, ag = oracle_gemv(fmt, cg, sg, x)
    u, au = oracle_gemv(fmt, cu, su, x)
    check_swiglu(h.cpu().numpy().view(np.uint16), g, ag, u, au)

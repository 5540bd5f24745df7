"""GPU parity of the Q6, Q5, Q3 and Q2 formats against the fp64 oracle,
through bq_gemv_ex and the device quantisers.  Q6 / Q5: fp16 scale absmax/31
or absmax/15, 6- or 5-bit codes as a low-nibble plane plus a 2- or 1-bit
plane; Q3 / Q2: absmax/3 or absmax/1, 3- or 2-bit codes as a 2-bit plane
(plus a 1-bit plane for Q3).  Tolerance as for Q4/Q8: |y - y_ref| <= 1e-3 *
sum_k |deq(w) x| + 1e-5 per output; packing bit-exact."""
import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import (DEV, check_swiglu, check_tol, dev, gpu_gemv, new_status,
                               oracle_gemv, pair_order, quantize)

pytestmark = pytest.mark.gpu

# Q6 and Q2: K a multiple of 64 (rows of 3K/4 or K/4 bytes stay 16-byte
# aligned); Q5 and Q3: of 128 (rows of 5K/8 or 3K/8 bytes).  Several chunks,
# ragged bands and a ragged last chunk along K; 1024 x 8192 sums its bands
# across CTAs in clusters.
_K64 = [(1, 64), (15, 64), (16, 256), (17, 320), (33, 832), (100, 2048), (257, 4160),
        (1000, 128), (4, 25600), (48, 768), (1024, 8192)]
_K128 = [(1, 128), (15, 128), (16, 256), (17, 384), (33, 896), (100, 2048), (257, 4224),
         (1000, 128), (4, 25600), (48, 768), (1024, 8192)]
SHAPES = {6: _K64, 5: _K128, 3: _K128, 2: _K64}
FMTS = [6, 5, 3, 2]
CASES = [(f, n, k) for f in FMTS for n, k in SHAPES[f]]
_DEQ = {2: oracle.dequantize_q2, 3: oracle.dequantize_q3, 5: oracle.dequantize_q5,
        6: oracle.dequantize_q6}


@pytest.mark.parametrize("fmt,N,K", CASES)
@pytest.mark.parametrize("B", [1, 3, 4, 8])
@pytest.mark.parametrize("flags", [0, bq.BQ_GEMV_STATIC_WEIGHTS])
def test_gemv_parity(fmt, N, K, B, flags):
    w = synth.weights_f32(synth.key(fmt, 84, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(fmt, 84, N, K, synth.KIND_X), B, K)
    y = gpu_gemv(fmt, codes, scales, x, flags=flags)
    y_ref, absy = oracle_gemv(fmt, codes, scales, x)
    check_tol(y, y_ref, absy)


@pytest.mark.parametrize("fmt", FMTS)
def test_one_hot_is_exact_column(fmt):
    """x = e_k returns column k of deq(W) exactly (one product, fp32-exact)."""
    N, K = 64, 256
    w = synth.weights_f32(synth.key(fmt, 85, 0, 0, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    deq = _DEQ[fmt](codes, scales)
    one = np.float16(1.0).view(np.uint16)
    for k0 in range(0, K, 8):
        x = np.zeros((8, K), dtype=np.uint16)
        x[np.arange(8), k0 + np.arange(8)] = one
        y = gpu_gemv(fmt, codes, scales, x)
        assert np.array_equal(y.astype(np.float64), deq[:, k0:k0 + 8].T)


@pytest.mark.parametrize("fmt", FMTS)
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


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("F,K,B", [(8, 256, 1), (200, 2048, 3), (512, 1024, 4), (1024, 512, 8)])
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


_ZERO = {2: 2, 3: 4, 5: 16, 6: 32}


def _pack_rows(fmt, q):
    """Code rows [N, K] -> packed rows, from the format text (not from the
    library): Q2 / Q3 2-bit plane byte 8j+i = low 2 bits of elements i, i+8,
    i+16, i+24 of block j; Q3 1-bit plane byte K/4+4j+i = bit 2 of element
    i+4p in bit p; Q5 / Q6 low-nibble plane byte 16j+i = element i | element
    i+16 << 4, then Q5 bit 4 of element i+4p in bit p of byte K/2+4j+i, or Q6
    bits 4-5 of element i+8p in bit pair p of byte K/2+8j+i."""
    N, K = q.shape
    b = q.reshape(N, K // 32, 32).astype(np.int64)
    if fmt in (2, 3):
        lo = b & 3
        first = lo[..., 0:8] | (lo[..., 8:16] << 2) | (lo[..., 16:24] << 4) | (lo[..., 24:32] << 6)
        planes = [first.reshape(N, K // 4)]
        if fmt == 3:
            top = (b >> 2).reshape(N, K // 32, 8, 4)
            planes.append(sum(top[:, :, p, :] << p for p in range(8)).reshape(N, K // 8))
    else:
        lo = b & 15
        planes = [(lo[..., :16] | (lo[..., 16:] << 4)).reshape(N, K // 2)]
        if fmt == 5:
            top = (b >> 4).reshape(N, K // 32, 8, 4)
            planes.append(sum(top[:, :, p, :] << p for p in range(8)).reshape(N, K // 8))
        else:
            top = (b >> 4).reshape(N, K // 32, 4, 8)
            planes.append(sum(top[:, :, p, :] << (2 * p) for p in range(4)).reshape(N, K // 4))
    return np.concatenate(planes, axis=1).astype(np.uint8)


@pytest.mark.parametrize("fmt", FMTS)
def test_bit_positions_exhaustive_on_gpu(fmt):
    """Row r = 32*c + p holds code c at element p of block 0 (every other code
    is the zero point; block 0's scale is 1, the others' 0): with x = e_p the
    GPU must return c - zero exactly at row 32*c + p and 0 elsewhere, and the
    packed rows must be what the oracle's quantiser lays out for them."""
    ncode = 1 << {2: 2, 3: 3, 5: 5, 6: 6}[fmt]
    z = _ZERO[fmt]
    N, K = 32 * ncode, 128
    q = np.full((N, K), z, dtype=np.int64)
    for c in range(ncode):
        for p in range(32):
            q[32 * c + p, p] = c
    codes = _pack_rows(fmt, q)
    scales = np.zeros((N, 8), dtype=np.uint16)
    scales[:, 0] = 0x3C00
    assert np.array_equal(_DEQ[fmt](codes, scales)[:, :32],
                          (q[:, :32] - z).astype(np.float64))     # the packer reads as the oracle does
    for p0 in range(0, 32, 8):
        x = np.zeros((8, K), dtype=np.float16)
        for b in range(8):
            x[b, p0 + b] = 1.0
        y = gpu_gemv(fmt, codes, scales, x.view(np.uint16))
        for b in range(8):
            p = p0 + b
            expect = np.zeros(N, dtype=np.float32)
            for c in range(ncode):
                expect[32 * c + p] = c - z
            assert np.array_equal(y[b], expect), (p, np.nonzero(y[b] != expect)[0][:8])

"""GPU parity of the batched-verification GEMM (bq_verify_gemm: Q4 / Q8
weights, batch 1..32, tcgen05 tensor cores) against the fp64 oracle.

Same operation and tolerance as the decode GEMV: per output element
|y - y_ref| <= 1e-3 * sum_k |deq(w) x| + 1e-5.  (The kernel rounds each
dequantised weight once to fp16 -- relative error <= 2^-11 -- after a per-row
power-of-two prescale, so the bound holds for any scale; the extreme-scale
case below checks that.)  Planes come from the oracle's quantiser and
activations from the seeded generators: no oracle input comes from the CUDA
path."""
import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import DEV, check_tol, dev, new_status, oracle_gemv, quantize

pytestmark = pytest.mark.gpu

# tiles of 128 rows (ragged N), units of 256 weights (ragged K), tiles split
# across CTAs (1000 x 8192: 8 tiles x 32 units over the SMs) and whole tiles
# per CTA (tiny K)
SHAPES = [(1, 32), (128, 256), (129, 288), (300, 800), (1000, 8192), (2048, 2048),
          (100, 4128), (4096, 1024), (7, 96), (6144, 4096)]


def gpu_verify(fmt, codes, scales, x_bits, ws=None, status=None):
    import torch
    N = codes.shape[0]
    K = codes.shape[1] * (2 if fmt == 4 else 1)
    x_bits = np.atleast_2d(x_bits)
    B = x_bits.shape[0]
    c, s, x = dev(codes.view(np.uint8)), dev(scales), dev(x_bits)
    y = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = ws if ws is not None else bq.workspace(bq.lib().bq_verify_workspace_bytes(N, K, B), DEV)
    st = status if status is not None else new_status()
    bq.verify_gemm(fmt, bq.qmat(c, s, N, K), x, y, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item()):#x}"
    return y.cpu().numpy()


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("B", [1, 8, 16, 17, 32])
def test_verify_gemm_parity(fmt, N, K, B):
    w = synth.weights_f32(synth.key(fmt, 86, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(fmt, 86, N, K, synth.KIND_X), B, K)
    y = gpu_verify(fmt, codes, scales, x)
    y_ref, absy = oracle_gemv(fmt, codes, scales, x)
    check_tol(y, y_ref, absy)


@pytest.mark.parametrize("fmt", [4, 8])
def test_verify_gemm_extreme_scales(fmt):
    """Rows whose blocks span 2^-20 .. 2^10 of scale (and rows entirely of tiny
    or of large weights): the per-row power-of-two prescale keeps every fp16
    weight normal and finite, so the tolerance still holds."""
    N, K, B = 384, 2048, 24
    rng = np.random.default_rng([fmt, 8687])
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    blk = w.reshape(N, K // 32, 32)
    blk *= (2.0 ** rng.uniform(-20, 10, size=(N, K // 32, 1))).astype(np.float32)
    blk[:128] *= np.float32(2.0 ** -12)           # a tile of tiny rows
    blk[128:160] *= np.float32(2.0 ** 4)          # rows of large weights
    w = blk.reshape(N, K)
    codes, scales = quantize(fmt, w)
    x = synth.activations_f16_bits(synth.key(fmt, 87, N, K, synth.KIND_X), B, K)
    y = gpu_verify(fmt, codes, scales, x)
    y_ref, absy = oracle_gemv(fmt, codes, scales, x)
    check_tol(y, y_ref, absy)


@pytest.mark.parametrize("fmt", [4, 8])
def test_verify_gemm_one_hot_columns(fmt):
    """x = e_k for 32 distinct k: y[b] is column k_b of deq(W) up to the one
    fp16 rounding of each weight (relative 2^-11)."""
    N, K = 256, 1024
    w = synth.weights_f32(synth.key(fmt, 88, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(fmt, w)
    ks = np.random.default_rng(88).choice(K, size=32, replace=False)
    x = np.zeros((32, K), dtype=np.float16)
    x[np.arange(32), ks] = 1.0
    y = gpu_verify(fmt, codes, scales, x.view(np.uint16))
    deq = {4: oracle.dequantize_q4, 8: oracle.dequantize_q8}[fmt](codes, scales)
    col = deq[:, ks].T
    assert np.all(np.abs(y - col) <= 2.0 ** -11 * np.abs(col) + 1e-30)


@pytest.mark.parametrize("fmt", [4, 8])
def test_verify_gemm_deterministic_and_workspace_returns_to_zero(fmt):
    """Two calls give bit-identical y; the workspace is all-zero after each, so
    one workspace serves calls of different shapes."""
    import torch
    shapes = [(1000, 8192, 32), (4096, 4096, 16), (300, 800, 9)]
    ws = bq.workspace(max(bq.lib().bq_verify_workspace_bytes(n, k, b) for n, k, b in shapes), DEV)
    for N, K, B in shapes:
        w = synth.weights_f32(synth.key(fmt, 89, N, K, synth.KIND_W), N, K)
        codes, scales = quantize(fmt, w)
        x = synth.activations_f16_bits(synth.key(fmt, 89, N, K, synth.KIND_X), B, K)
        y1 = gpu_verify(fmt, codes, scales, x, ws=ws)
        assert int(ws.view(torch.int32).abs().sum().item()) == 0
        y2 = gpu_verify(fmt, codes, scales, x, ws=ws)
        assert np.array_equal(y1, y2)
        y_ref, absy = oracle_gemv(fmt, codes, scales, x)
        check_tol(y1, y_ref, absy)


def test_verify_gemm_agrees_with_decode_gemv_at_batch_8():
    """At B = 8 both paths run: each within the tolerance of the oracle, and of
    each other."""
    N, K, B = 2048, 8192, 8
    from tests.gpu_helpers import gpu_gemv
    w = synth.weights_f32(synth.key(4, 90, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(4, w)
    x = synth.activations_f16_bits(synth.key(4, 90, N, K, synth.KIND_X), B, K)
    yv = gpu_verify(4, codes, scales, x)
    yg = gpu_gemv(4, codes, scales, x)
    y_ref, absy = oracle_gemv(4, codes, scales, x)
    check_tol(yv, y_ref, absy)
    check_tol(yg, y_ref, absy)
    assert np.all(np.abs(yv.astype(np.float64) - yg) <= 2e-3 * absy + 2e-5)

"""The Python binding refuses arguments the C library cannot check itself
(it takes raw pointers and sizes): host tensors where device memory is
meant, an x whose width is not K, planes or outputs too small for the shape.
Every refusal happens before any library call or launch, so these run on the
CPU; `_Dev` stands in for a device tensor of the right shape."""
import numpy as np
import pytest
import torch

from quantised_weight_gemv_b200 import bq


class _Dev:
    """A CPU tensor that reports itself as a CUDA tensor (for the shape checks)."""

    def __init__(self, t):
        self._t = t
        self.is_cuda = True
        self.shape = t.shape
        self.dtype = t.dtype
        self.device = "cuda:0"

    def __getattr__(self, name):
        return getattr(self._t, name)


def _planes(fmt, N, K, rows=None):
    width = {2: K // 4, 3: 3 * K // 8, 4: K // 2, 5: 5 * K // 8, 6: 3 * K // 4, 8: K}[fmt]
    rows = N if rows is None else rows
    return (_Dev(torch.zeros((rows, width), dtype=torch.uint8)),
            _Dev(torch.zeros((rows, bq.scales_ld(K)), dtype=torch.int16)))


def test_gemv_refuses_host_tensors():
    c, s = _planes(4, 64, 256)
    W = bq.qmat(c, s, 64, 256)
    x = torch.zeros((1, 256), dtype=torch.float16)                  # host memory
    y = _Dev(torch.zeros((1, 64), dtype=torch.float32))
    ws = _Dev(torch.zeros(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        bq.gemv(4, W, x, y, ws)
    with pytest.raises(ValueError, match="codes must be a CUDA tensor"):
        bq.gemv(4, bq.qmat(torch.zeros((64, 128), dtype=torch.uint8), s, 64, 256), _Dev(x), y, ws)


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
def test_gemv_refuses_wrong_shapes(fmt):
    N, K, B = 64, 256, 2
    c, s = _planes(fmt, N, K)
    W = bq.qmat(c, s, N, K)
    ws = _Dev(torch.zeros(1 << 20, dtype=torch.uint8))
    y = _Dev(torch.zeros((B, N), dtype=torch.float32))
    x_bad = _Dev(torch.zeros((B, K + 32), dtype=torch.float16))     # width is not K
    with pytest.raises(ValueError, match="x must be a contiguous"):
        bq.gemv(fmt, W, x_bad, y, ws)
    x = _Dev(torch.zeros((B, K), dtype=torch.float16))
    with pytest.raises(ValueError, match="y must be contiguous"):
        bq.gemv(fmt, W, x, _Dev(torch.zeros((B, N - 1), dtype=torch.float32)), ws)
    h = _Dev(torch.zeros((B, N // 2 - 1), dtype=torch.float16))      # SwiGLU: fp16 [B][N/2]
    with pytest.raises(ValueError, match="y must be contiguous"):
        bq.gemv(fmt, W, x, h, ws, epilogue=bq.BQ_EPI_SWIGLU)
    c_short, s_short = _planes(fmt, N, K, rows=N - 1)
    with pytest.raises(ValueError, match="codes hold"):
        bq.gemv(fmt, bq.qmat(c_short, s, N, K), x, y, ws)
    with pytest.raises(ValueError, match="scales hold"):
        bq.gemv(fmt, bq.qmat(c, s_short, N, K), x, y, ws)


def test_quantize_dev_refuses_host_tensors_and_small_planes():
    N, K = 32, 256
    w = torch.zeros((N, K), dtype=torch.float32)
    c, s = _planes(4, N, K)
    with pytest.raises(ValueError, match="w must be a CUDA tensor"):
        bq.quantize_dev(4, w, c, s)
    c_short, _ = _planes(4, N, K, rows=N - 1)
    with pytest.raises(ValueError, match="planes too small"):
        bq.quantize_dev(4, _Dev(w), c_short, s)
    with pytest.raises(ValueError, match="w must be contiguous fp32"):
        bq.quantize_dev(4, _Dev(w.half()), c, s)


def test_moe_and_step_plan_refuse_host_tensors():
    N, K, E, B, topk = 64, 256, 4, 2, 2
    c = _Dev(torch.zeros((E, N, K // 2), dtype=torch.uint8))
    s = _Dev(torch.zeros((E, N, bq.scales_ld(K)), dtype=torch.int16))
    idx = torch.zeros((B, topk), dtype=torch.int32)                # host memory
    with pytest.raises(ValueError, match="expert_idx must be a CUDA tensor"):
        bq.moe_gemv_q4(bq.qmat(c, s, N, K), E, N * K // 2, N * bq.scales_ld(K),
                       _Dev(torch.zeros((B, K), dtype=torch.float16)), False, idx, None,
                       _Dev(torch.zeros((B, topk, N), dtype=torch.float32)),
                       _Dev(torch.zeros(1 << 20, dtype=torch.uint8)))
    c2, s2 = _planes(4, N, K)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        bq.StepPlan(4, [(bq.qmat(c2, s2, N, K), torch.zeros((1, K), dtype=torch.float16),
                         _Dev(torch.zeros((1, N), dtype=torch.float32)), 0)], "cuda:0")


def test_verify_gemm_refuses_host_tensors_and_wrong_shapes():
    N, K, B = 256, 512, 16
    c, s = _planes(4, N, K)
    W = bq.qmat(c, s, N, K)
    ws = _Dev(torch.zeros(1 << 20, dtype=torch.uint8))
    y = _Dev(torch.zeros((B, N), dtype=torch.float32))
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        bq.verify_gemm(4, W, torch.zeros((B, K), dtype=torch.float16), y, ws)
    with pytest.raises(ValueError, match="x must be a contiguous"):
        bq.verify_gemm(4, W, _Dev(torch.zeros((B, K + 32), dtype=torch.float16)), y, ws)
    with pytest.raises(ValueError, match="y must be contiguous"):
        bq.verify_gemm(4, W, _Dev(torch.zeros((B, K), dtype=torch.float16)),
                       _Dev(torch.zeros((B, N - 1), dtype=torch.float32)), ws)
    small = bq.qmat(*_planes(4, N, K, rows=N - 1), N, K)            # planes short of N rows
    with pytest.raises(ValueError):
        bq.verify_gemm(4, small, _Dev(torch.zeros((B, K), dtype=torch.float16)), y, ws)


def _cache(B, Hkv, T, D=128):
    return (_Dev(torch.zeros((B, Hkv, T, D), dtype=torch.int8)),
            _Dev(torch.zeros((B, Hkv, T, D // 32), dtype=torch.int16)),
            _Dev(torch.zeros((B, Hkv, D, T), dtype=torch.int8)),
            _Dev(torch.zeros((B, Hkv, T, D // 32), dtype=torch.int16)))


def test_attention_refuses_host_tensors_and_wrong_shapes():
    B, Hkv, G, T, D = 2, 4, 5, 256, 128
    kc, ks, vt, vs = _cache(B, Hkv, T)
    with pytest.raises(ValueError, match="k_codes must be a CUDA tensor"):
        bq.kv_cache(torch.zeros((B, Hkv, T, D), dtype=torch.int8), ks, vt, vs)
    with pytest.raises(ValueError, match="do not match the cache layout"):
        bq.kv_cache(kc, ks, _Dev(torch.zeros((B, Hkv, T, D), dtype=torch.int8)), vs)   # not transposed
    kv = bq.kv_cache(kc, ks, vt, vs)
    q = _Dev(torch.zeros((B, Hkv * G, D), dtype=torch.float16))
    lens = _Dev(torch.zeros(B, dtype=torch.int32))
    o = _Dev(torch.zeros((B, Hkv * G, D), dtype=torch.float32))
    ws = _Dev(torch.zeros(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        bq.attn_decode_q8(kv, torch.zeros((B, Hkv * G, D), dtype=torch.float16), lens, G, 0.1, o, ws)
    with pytest.raises(ValueError, match="q must be contiguous"):
        bq.attn_decode_q8(kv, _Dev(torch.zeros((B, Hkv * (G + 1), D), dtype=torch.float16)), lens, G,
                          0.1, o, ws)
    with pytest.raises(ValueError, match="lens must be int32"):
        bq.attn_decode_q8(kv, q, _Dev(torch.zeros(B, dtype=torch.int64)), G, 0.1, o, ws)
    with pytest.raises(ValueError, match="o too small"):
        bq.attn_decode_q8(kv, q, lens, G, 0.1, _Dev(torch.zeros((B, Hkv * G, D - 1),
                                                               dtype=torch.float32)), ws)

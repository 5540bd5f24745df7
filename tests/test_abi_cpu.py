"""C ABI checks that need no GPU: the library loads and exports every entry
point include/bq.h declares, the host-side quantiser and unpacker agree
bit-for-bit with the oracle, the plane <-> block converters round-trip, and
every GPU entry point rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from quantised_weight_gemv_b200 import bq, synth
from tests.conftest import ROOT, read_golden

FAKE = 0x7f0000000000          # a 16-byte aligned address that is never dereferenced


def _declared():
    with open(os.path.join(ROOT, "include", "bq.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"BQ_API[^;(]*?\b(bq_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 17
    L = bq.lib()
    for n in names:
        assert hasattr(L, n), n
        assert n in bq._SIGS, f"binding lacks {n}"


def test_status_strings_and_scales_ld():
    assert bq.bq_status_string(0) == "ok"
    assert bq.bq_status_string(bq.BQ_ERR_TIMEOUT) == "bounded wait timed out"
    for K in (32, 64, 96, 256, 288, 768, 2048, 25600):
        assert bq.scales_ld(K) == oracle.scales_ld(K) == -(-(K // 32) // 8) * 8
    assert bq.scales_ld(33) == 0 and bq.scales_ld(0) == 0


_ORQ = {2: lambda w: oracle.quantize_q2(w), 3: lambda w: oracle.quantize_q3(w),
        4: lambda w: oracle.quantize_q4(w), 5: lambda w: oracle.quantize_q5(w),
        6: lambda w: oracle.quantize_q6(w), 8: lambda w: oracle.quantize_q8(w)}


def _host_quantize(fmt, w):
    N, K = w.shape
    width = {2: K // 4, 3: 3 * K // 8, 4: K // 2, 5: 5 * K // 8, 6: 3 * K // 4, 8: K}[fmt]
    codes = np.zeros((N, width), dtype=np.int8 if fmt == 8 else np.uint8)
    scales = np.zeros((N, bq.scales_ld(K)), dtype=np.uint16)
    fn = {2: bq.lib().bq_quantize_q2, 3: bq.lib().bq_quantize_q3, 4: bq.lib().bq_quantize_q4,
          5: bq.lib().bq_quantize_q5, 6: bq.lib().bq_quantize_q6, 8: bq.lib().bq_quantize_q8}[fmt]
    rc = fn(w.ctypes.data, N, K, codes.ctypes.data, scales.ctypes.data)
    return rc, codes, scales


def _edge_weights():
    w = synth.weights_f32(synth.key(0, 93, 0, 0, 0), 24, 320)
    w[0, :32] = 0.0                                   # zero block
    w[1, :32] = 1e-9                                  # scale rounds to zero
    w[2, :32] = np.float32(2.0 ** -20)                # subnormal fp16 scale
    w[3, 0], w[3, 1] = 0.7, -0.7                      # symmetric absmax tie
    d = np.float32(0.1) / np.float32(7.0)
    w[4, 32:64] = np.float32(2.5) * np.float32(2.0 ** -6)
    w[4, 32] = 7 * 2.0 ** -6                          # exact half-way codes
    w[5] *= 1000.0                                    # large but finite scales
    return w


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
def test_host_quantiser_bit_exact_vs_oracle(fmt):
    w = _edge_weights()
    rc, codes, scales = _host_quantize(fmt, w)
    assert rc == 0
    oc, os_ = _ORQ[fmt](w)
    assert np.array_equal(codes.view(np.uint8), oc.view(np.uint8))
    assert np.array_equal(scales, os_)


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
def test_host_quantiser_rejects_out_of_range(fmt):
    w = np.zeros((1, 32), dtype=np.float32)
    w[0, 3] = np.nan
    assert _host_quantize(fmt, w)[0] == bq.BQ_ERR_RANGE
    w[0, 3] = 1.0e7                                    # absmax/levels overflows fp16
    assert _host_quantize(fmt, w)[0] == bq.BQ_ERR_RANGE


@pytest.mark.parametrize("fmt", [2, 3, 4, 5, 6, 8])
def test_host_dequantize_matches_oracle(fmt):
    w = synth.weights_f32(synth.key(1, 93, 0, 0, 0), 9, 128)
    codes, scales = _ORQ[fmt](w)
    out = np.zeros(w.shape, dtype=np.float32)
    fn = {2: bq.lib().bq_dequantize_q2, 3: bq.lib().bq_dequantize_q3, 4: bq.lib().bq_dequantize_q4,
          5: bq.lib().bq_dequantize_q5, 6: bq.lib().bq_dequantize_q6, 8: bq.lib().bq_dequantize_q8}[fmt]
    assert fn(codes.ctypes.data, scales.ctypes.data, 9, 128, out.ctypes.data) == 0
    ref = {2: oracle.dequantize_q2, 3: oracle.dequantize_q3, 4: oracle.dequantize_q4,
           5: oracle.dequantize_q5, 6: oracle.dequantize_q6, 8: oracle.dequantize_q8}[fmt](codes, scales)
    assert np.array_equal(out.astype(np.float64), ref)


def test_blocks_layout_matches_golden_and_round_trips():
    g = read_golden("q4_block_worked.txt")
    codes = np.array([[int(t, 16) for t in g["packed"]]], dtype=np.uint8)
    scales = np.zeros((1, 8), dtype=np.uint16)
    scales[0, 0] = int(g["scale_bits"][0], 16)
    blk = np.zeros(18, dtype=np.uint8)
    assert bq.lib().bq_planes_to_blocks_q4(codes.ctypes.data, scales.ctypes.data, 1, 32,
                                           blk.ctypes.data) == 0
    assert list(blk[:2]) == [0x00, 0x20]              # little-endian fp16 scale first
    assert np.array_equal(blk[2:], codes[0])
    r = np.random.default_rng(5)
    for fmt, rec in ((4, 18), (8, 34)):
        N, K = 7, 160
        blocks = r.integers(0, 256, size=N * (K // 32) * rec, dtype=np.uint8)
        c = np.zeros((N, K // 2 if fmt == 4 else K), dtype=np.uint8)
        s = np.zeros((N, bq.scales_ld(K)), dtype=np.uint16)
        to_p = bq.lib().bq_blocks_to_planes_q4 if fmt == 4 else bq.lib().bq_blocks_to_planes_q8
        to_b = bq.lib().bq_planes_to_blocks_q4 if fmt == 4 else bq.lib().bq_planes_to_blocks_q8
        assert to_p(blocks.ctypes.data, N, K, c.ctypes.data, s.ctypes.data) == 0
        back = np.zeros_like(blocks)
        assert to_b(c.ctypes.data, s.ctypes.data, N, K, back.ctypes.data) == 0
        assert np.array_equal(back, blocks)
        assert np.all(s[:, K // 32:] == 0)


def test_workspace_sizes():
    assert bq.lib().bq_gemv_workspace_bytes(0, 32) == 0
    assert bq.lib().bq_gemv_workspace_bytes(16, 48) == 0
    a = bq.lib().bq_gemv_workspace_bytes(2048, 2048)
    b = bq.lib().bq_gemv_workspace_bytes(51200, 5120)
    assert 0 < a < b < (64 << 20)
    assert bq.lib().bq_moe_workspace_bytes(2048, 768, 8, 8, 128) > 0
    assert bq.lib().bq_moe_workspace_bytes(2048, 768, 9, 8, 128) == 0
    assert bq.lib().bq_moe_workspace_bytes(2048, 768, 8, 9, 128) == 0


def _gemv_rc(fmt=4, W=None, x=FAKE, B=1, y=FAKE, ws=FAKE, ws_bytes=1 << 30):
    W = W if W is not None else bq.bq_qmat(FAKE, FAKE, 64, 256)
    fn = bq.lib().bq_gemv_q4 if fmt == 4 else bq.lib().bq_gemv_q8
    return fn(ctypes.byref(W), x, B, y, ws, ws_bytes, None, None)


@pytest.mark.parametrize("fmt", [4, 8])
def test_gemv_argument_validation_before_launch(fmt):
    assert bq.lib().bq_gemv_q4(None, FAKE, 1, FAKE, FAKE, 1 << 30, None, None) == bq.BQ_ERR_NULL
    assert _gemv_rc(fmt, W=bq.bq_qmat(None, FAKE, 64, 256)) == bq.BQ_ERR_NULL
    assert _gemv_rc(fmt, x=None) == bq.BQ_ERR_NULL
    assert _gemv_rc(fmt, ws=None) == bq.BQ_ERR_NULL
    assert _gemv_rc(fmt, W=bq.bq_qmat(FAKE, FAKE, 64, 48)) == bq.BQ_ERR_SHAPE
    assert _gemv_rc(fmt, W=bq.bq_qmat(FAKE, FAKE, 0, 256)) == bq.BQ_ERR_SHAPE
    assert _gemv_rc(fmt, B=0) == bq.BQ_ERR_BATCH
    assert _gemv_rc(fmt, B=9) == bq.BQ_ERR_BATCH
    assert _gemv_rc(fmt, x=FAKE + 8) == bq.BQ_ERR_ALIGN
    assert _gemv_rc(fmt, W=bq.bq_qmat(FAKE + 4, FAKE, 64, 256)) == bq.BQ_ERR_ALIGN
    assert _gemv_rc(fmt, ws_bytes=1024) == bq.BQ_ERR_WORKSPACE


def test_gemv_ex_epilogue_validation_before_launch():
    f = bq.lib().bq_gemv_ex

    def rc(fmt=4, N=64, epi=bq.BQ_EPI_SWIGLU, flags=0):
        W = bq.bq_qmat(FAKE, FAKE, N, 256)
        return f(fmt, ctypes.byref(W), FAKE, 1, FAKE, epi, flags, FAKE, 1 << 30, None, None)

    assert rc(fmt=7) == bq.BQ_ERR_SHAPE
    assert rc(fmt=1) == bq.BQ_ERR_SHAPE
    assert rc(fmt=9) == bq.BQ_ERR_SHAPE
    assert rc(flags=8) == bq.BQ_ERR_SHAPE           # unknown flag bit
    assert rc(flags=bq.BQ_GEMV_ROWS16 | bq.BQ_GEMV_ROWS32) == bq.BQ_ERR_SHAPE
    assert rc(fmt=8, flags=bq.BQ_GEMV_ROWS32) == bq.BQ_ERR_SHAPE   # Q8 chunks are 16 rows
    assert rc(fmt=6, flags=bq.BQ_GEMV_ROWS32) == bq.BQ_ERR_SHAPE   # so are Q6 chunks
    W6 = bq.bq_qmat(FAKE, FAKE, 64, 96)                            # Q6 needs K % 64 == 0
    assert f(6, ctypes.byref(W6), FAKE, 1, FAKE, bq.BQ_EPI_NONE, 0, FAKE, 1 << 30, None,
             None) == bq.BQ_ERR_SHAPE
    W5 = bq.bq_qmat(FAKE, FAKE, 64, 192)                           # Q5 needs K % 128 == 0
    assert f(5, ctypes.byref(W5), FAKE, 1, FAKE, bq.BQ_EPI_NONE, 0, FAKE, 1 << 30, None,
             None) == bq.BQ_ERR_SHAPE
    assert rc(fmt=5, flags=bq.BQ_GEMV_ROWS32) == bq.BQ_ERR_SHAPE
    W2 = bq.bq_qmat(FAKE, FAKE, 64, 96)                            # Q2 needs K % 64 == 0
    assert f(2, ctypes.byref(W2), FAKE, 1, FAKE, bq.BQ_EPI_NONE, 0, FAKE, 1 << 30, None,
             None) == bq.BQ_ERR_SHAPE
    W3 = bq.bq_qmat(FAKE, FAKE, 64, 192)                           # Q3 needs K % 128 == 0
    assert f(3, ctypes.byref(W3), FAKE, 1, FAKE, bq.BQ_EPI_NONE, 0, FAKE, 1 << 30, None,
             None) == bq.BQ_ERR_SHAPE
    assert rc(fmt=3, flags=bq.BQ_GEMV_ROWS32) == bq.BQ_ERR_SHAPE
    assert rc(fmt=2, flags=bq.BQ_GEMV_ROWS32) == bq.BQ_ERR_SHAPE
    assert rc(flags=bq.BQ_GEMV_STATIC_WEIGHTS, N=40) == bq.BQ_ERR_SHAPE
    assert rc(epi=2) == bq.BQ_ERR_SHAPE
    assert rc(epi=-1) == bq.BQ_ERR_SHAPE
    assert rc(N=40) == bq.BQ_ERR_SHAPE            # SwiGLU needs whole 16-row gate|up tiles
    W = bq.bq_qmat(FAKE, FAKE, 64, 256)
    assert f(4, ctypes.byref(W), None, 1, FAKE, bq.BQ_EPI_SWIGLU, 0, FAKE, 1 << 30, None, None) == bq.BQ_ERR_NULL
    assert f(8, ctypes.byref(W), FAKE, 9, FAKE, bq.BQ_EPI_SWIGLU, 1, FAKE, 1 << 30, None, None) == bq.BQ_ERR_BATCH


def test_moe_argument_validation_before_launch():
    W = bq.bq_qmat(FAKE, FAKE, 64, 256)
    f = bq.lib().bq_moe_gemv_q4
    cs, ss = 64 * 128, 64 * 8

    def rc(**kw):
        a = dict(W=W, E=16, cs=cs, ss=ss, x=FAKE, xps=0, idx=FAKE, rw=None, B=2, topk=4, y=FAKE,
                 ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return f(ctypes.byref(a["W"]), a["E"], a["cs"], a["ss"], a["x"], a["xps"], a["idx"],
                 a["rw"], a["B"], a["topk"], a["y"], a["ws"], a["wsb"], None, None)

    assert rc(idx=None) == bq.BQ_ERR_NULL
    assert rc(B=9) == bq.BQ_ERR_BATCH
    assert rc(B=8, topk=9) == bq.BQ_ERR_BATCH
    assert rc(E=0) == bq.BQ_ERR_SHAPE
    assert rc(cs=cs - 16) == bq.BQ_ERR_SHAPE
    assert rc(ss=ss + 4) == bq.BQ_ERR_ALIGN
    assert rc(wsb=4096) == bq.BQ_ERR_WORKSPACE


def test_device_quantiser_argument_validation():
    assert bq.lib().bq_quantize_q3_dev(FAKE, 4, 192, FAKE, FAKE, None, None) == bq.BQ_ERR_SHAPE
    assert bq.lib().bq_quantize_q2_dev(FAKE, 4, 60, FAKE, FAKE, None, None) == bq.BQ_ERR_SHAPE
    f = bq.lib().bq_quantize_q4_dev
    assert f(None, 4, 64, FAKE, FAKE, None, None) == bq.BQ_ERR_NULL
    assert f(FAKE, 4, 60, FAKE, FAKE, None, None) == bq.BQ_ERR_SHAPE
    assert f(FAKE + 4, 4, 64, FAKE, FAKE, None, None) == bq.BQ_ERR_ALIGN


def test_product_path_has_no_oracle_or_fallback():
    """The library and its binding never reference the oracle, and the binding
    raises instead of falling back when the library is absent."""
    pkg = os.path.join(ROOT, "quantised_weight_gemv_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                with open(os.path.join(dirpath, fn)) as f:
                    src = f.read()
                assert "import oracle" not in src and "from oracle" not in src, fn
                assert "oracle.c" not in src and "liboracle" not in src, fn


def test_binding_raises_when_the_library_is_missing(monkeypatch, tmp_path):
    """No fallback: with libbq.so absent, loading it and every wrapper raise."""
    monkeypatch.setattr(bq, "_lib", None)
    monkeypatch.setattr(bq, "LIB_PATH", str(tmp_path / "libbq.so"))
    with pytest.raises(RuntimeError, match="missing"):
        bq.lib()
    with pytest.raises(RuntimeError, match="missing"):
        bq.bq_scales_ld(256)
    with pytest.raises(RuntimeError, match="missing"):
        bq.lib().bq_gemv_workspace_bytes(64, 256)


def test_oracle_shares_nothing_with_the_library():
    """The oracle is plain C over the C standard library: it includes no header
    of the package or the CUDA toolkit, and its Python wrapper imports nothing
    from the package."""
    import re
    with open(os.path.join(ROOT, "oracle", "oracle.c")) as f:
        src = f.read()
    includes = re.findall(r'#include\s*[<"]([^>"]+)[>"]', src)
    assert set(includes) <= {"math.h", "pthread.h", "stdint.h", "stdlib.h", "string.h"}, includes
    with open(os.path.join(ROOT, "oracle", "__init__.py")) as f:
        py = f.read()
    assert "quantised_weight_gemv_b200" not in py and "libbq" not in py


def test_step_argument_validation_before_launch():
    L = bq.lib()
    assert L.bq_step_plan_bytes(0) == 0 and L.bq_step_plan_bytes(3) > 3 * 320
    info = bq.bq_step_info()
    arr = (bq.bq_step_mat * 2)()
    for i in range(2):
        arr[i] = bq.bq_step_mat(bq.bq_qmat(FAKE, FAKE, 64, 256), FAKE, FAKE, 1, i)
    nb = L.bq_step_plan_bytes(2)
    assert L.bq_step_plan(4, None, 2, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_NULL
    assert L.bq_step_plan(5, arr, 2, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_SHAPE
    assert L.bq_step_plan(4, arr, 0, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_SHAPE
    assert L.bq_step_plan(4, arr, 2, FAKE, nb - 1, ctypes.byref(info)) == bq.BQ_ERR_WORKSPACE
    assert L.bq_step_plan(4, arr, 2, FAKE + 16, nb, ctypes.byref(info)) == bq.BQ_ERR_ALIGN
    arr[1].B = 9
    assert L.bq_step_plan(4, arr, 2, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_BATCH
    arr[1].B = 1
    arr[1].stage = -1
    assert L.bq_step_plan(4, arr, 2, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_SHAPE
    arr[1].stage = 1
    arr[1].epilogue = 3
    assert L.bq_step_plan(4, arr, 2, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_SHAPE
    arr[1].epilogue = bq.BQ_EPI_SWIGLU
    arr[1].W.N = 24                                   # not whole 16-row gate|up tiles
    assert L.bq_step_plan(4, arr, 2, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_SHAPE
    arr[1].W.N = 64
    arr[0].W.K = 40
    assert L.bq_step_plan(4, arr, 2, FAKE, nb, ctypes.byref(info)) == bq.BQ_ERR_SHAPE
    info = bq.bq_step_info(4, 2, 2, 296, 10, 0, 64, 128, 1 << 20)
    assert L.bq_step_run(None, FAKE, FAKE, 1 << 20, None, None) == bq.BQ_ERR_NULL
    assert L.bq_step_run(ctypes.byref(info), FAKE, FAKE, 1024, None, None) == bq.BQ_ERR_WORKSPACE
    assert L.bq_step_run(ctypes.byref(info), FAKE + 16, FAKE, 1 << 20, None, None) == bq.BQ_ERR_ALIGN


def test_step_run_ex_rejects_negative_options():
    """Host-side checks of the bounded-wait options: nothing is launched."""
    import ctypes
    info = bq.bq_step_info()
    info.fmt, info.n_stages, info.grid = 4, 1, 1
    w = bq.bq_step_wait(-1, 0, 0)
    fake = 0x7f0000000000
    assert bq.lib().bq_step_run_ex(ctypes.byref(info), fake, fake, 1 << 30, ctypes.byref(w),
                                   None, None) == bq.BQ_ERR_SHAPE
    w = bq.bq_step_wait(0, -1, 0)
    assert bq.lib().bq_step_run_ex(ctypes.byref(info), fake, fake, 1 << 30, ctypes.byref(w),
                                   None, None) == bq.BQ_ERR_SHAPE


def test_verify_and_attention_workspace_sizes():
    f = bq.lib().bq_verify_workspace_bytes
    assert f(0, 256, 8) == 0 and f(128, 48, 8) == 0 and f(128, 256, 0) == 0 and f(128, 256, 33) == 0
    a, b = f(128, 4096, 32), f(24576, 4096, 32)
    assert 0 < a < b
    g = bq.lib().bq_attn_workspace_bytes
    assert g(0, 8) == 0 and g(1, 0) == 0
    assert 0 < g(1, 8) <= g(8, 8)


def _verify_rc(fmt=4, W=None, x=FAKE, B=16, y=FAKE, ws=FAKE, ws_bytes=1 << 30):
    W = W if W is not None else bq.bq_qmat(FAKE, FAKE, 256, 512)
    return bq.lib().bq_verify_gemm(fmt, ctypes.byref(W), x, B, y, ws, ws_bytes, None, None)


def test_verify_gemm_argument_validation_before_launch():
    """Every host-detectable error of bq_verify_gemm is returned before any
    device call (fake pointers are never dereferenced)."""
    assert bq.lib().bq_verify_gemm(4, None, FAKE, 16, FAKE, FAKE, 1 << 30, None, None) == bq.BQ_ERR_NULL
    assert _verify_rc(W=bq.bq_qmat(None, FAKE, 256, 512)) == bq.BQ_ERR_NULL
    assert _verify_rc(fmt=5) == bq.BQ_ERR_SHAPE                  # Q4 or Q8 only
    assert _verify_rc(W=bq.bq_qmat(FAKE, FAKE, 256, 48)) == bq.BQ_ERR_SHAPE
    assert _verify_rc(x=None) == bq.BQ_ERR_NULL
    assert _verify_rc(ws=None) == bq.BQ_ERR_NULL
    assert _verify_rc(B=0) == bq.BQ_ERR_BATCH
    assert _verify_rc(B=33) == bq.BQ_ERR_BATCH
    assert _verify_rc(y=FAKE + 4) == bq.BQ_ERR_ALIGN
    assert _verify_rc(ws_bytes=1024) == bq.BQ_ERR_WORKSPACE


def _attn_rc(kv=None, q=FAKE, lens=FAKE, B=2, Hkv=4, G=5, scale=0.088, o=FAKE, ws=FAKE,
             ws_bytes=1 << 30):
    kv = kv if kv is not None else bq.bq_kv_cache(FAKE, FAKE, FAKE, FAKE, 128, 1024)
    return bq.lib().bq_attn_decode_q8(ctypes.byref(kv), q, lens, B, Hkv, G, scale, o, ws, ws_bytes,
                                      None, None)


def test_attention_argument_validation_before_launch():
    """Every host-detectable error of bq_attn_decode_q8 is returned before any
    device call: null planes, a head dimension other than 128, a cache length
    that is not a multiple of 128 positions, G outside 1..8, a NaN scale, the
    batch, 16-byte alignment and the workspace size."""
    assert bq.lib().bq_attn_decode_q8(None, FAKE, FAKE, 2, 4, 5, 0.1, FAKE, FAKE, 1 << 30,
                                      None, None) == bq.BQ_ERR_NULL
    assert _attn_rc(kv=bq.bq_kv_cache(FAKE, None, FAKE, FAKE, 128, 1024)) == bq.BQ_ERR_NULL
    assert _attn_rc(lens=None) == bq.BQ_ERR_NULL
    assert _attn_rc(kv=bq.bq_kv_cache(FAKE, FAKE, FAKE, FAKE, 64, 1024)) == bq.BQ_ERR_SHAPE
    assert _attn_rc(kv=bq.bq_kv_cache(FAKE, FAKE, FAKE, FAKE, 128, 1000)) == bq.BQ_ERR_SHAPE
    assert _attn_rc(G=0) == bq.BQ_ERR_SHAPE and _attn_rc(G=9) == bq.BQ_ERR_SHAPE
    assert _attn_rc(scale=float("nan")) == bq.BQ_ERR_SHAPE
    assert _attn_rc(B=0) == bq.BQ_ERR_BATCH
    assert _attn_rc(q=FAKE + 2) == bq.BQ_ERR_ALIGN
    assert _attn_rc(ws_bytes=16) == bq.BQ_ERR_WORKSPACE


def _prototypes():
    """name -> (return type, [parameter types]) for every BQ_API function of
    include/bq.h, comments removed and `const` dropped."""
    with open(os.path.join(ROOT, "include", "bq.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    out = {}
    for ret, name, params in re.findall(r"BQ_API\s+([^;(]*?)\b(bq_\w+)\s*\(([^)]*)\)\s*;", src):
        def norm(t):
            t = re.sub(r"\bconst\b", " ", t)
            t = re.sub(r"\s*\*", " *", t)
            return " ".join(t.split())
        types = []
        for p in params.split(","):
            p = norm(p)
            # drop the parameter name: the last identifier after the type
            m = re.match(r"^(.*?)(\w+)$", p)
            assert m, (name, p)
            types.append(norm(m.group(1)))
        out[name] = (norm(ret), types)
    return out


def _ctype_of(c):
    scalars = {"int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "uint64_t": ctypes.c_uint64,
               "size_t": ctypes.c_size_t, "float": ctypes.c_float}
    if c in scalars:
        return scalars[c]
    if c == "char *":
        return ctypes.c_char_p
    if c == "void * *":
        return ctypes.POINTER(ctypes.c_void_p)
    if c == "size_t *":
        return ctypes.POINTER(ctypes.c_size_t)
    m = re.match(r"^(bq_\w+) \*$", c)
    if m:
        return ctypes.POINTER(getattr(bq, m.group(1)))
    assert c.endswith("*"), c
    return ctypes.c_void_p


def test_binding_signatures_match_the_header():
    """Every ctypes signature the binding declares has the header's parameter
    count, scalar widths and pointer kinds (a struct pointer as that struct),
    so an argument can neither shift nor be truncated."""
    protos = _prototypes()
    assert set(protos) == set(_declared())
    assert set(bq._SIGS) == set(protos), set(bq._SIGS) ^ set(protos)
    for name, (ret, params) in protos.items():
        res, args = bq._SIGS[name]
        assert res == _ctype_of(ret), (name, ret, res)
        assert len(args) == len(params), (name, params, args)
        for i, (c, a) in enumerate(zip(params, args)):
            assert a == _ctype_of(c), (name, i, c, a)


def test_binding_structs_match_the_header_layout(tmp_path):
    """Size and field offsets of every structure the binding mirrors, as gcc
    lays them out from include/bq.h."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    structs = [bq.bq_qmat, bq.bq_step_mat, bq.bq_step_info, bq.bq_step_wait, bq.bq_kv_cache,
               bq.bq_gemv_geometry]
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "bq.h"', "int main(void) {"]
    for s in structs:
        n = s.__name__
        lines.append(f'printf("{n} sizeof %zu\\n", sizeof({n}));')
        for f, _ in s._fields_:
            lines.append(f'printf("{n} {f} %zu\\n", offsetof({n}, {f}));')
    lines += ["return 0;", "}"]
    c = tmp_path / "layout.c"
    c.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([gcc, "-std=c11", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)],
                   check=True, capture_output=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n"):
        if line:
            n, f, v = line.split()
            got[(n, f)] = int(v)
    for s in structs:
        n = s.__name__
        assert got[(n, "sizeof")] == ctypes.sizeof(s), n
        for f, _ in s._fields_:
            assert got[(n, f)] == getattr(s, f).offset, (n, f)

"""fp64 CPU oracle for block-quantised weight GEMV -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and the
two share no code: this wraps ``oracle.c`` (plain C, compiled with gcc) through
ctypes, and ``oracle.c`` has its own fp16 conversions, quantisers and
unpackers.

What the oracle computes is the plain definition of a decode GEMV with the
dequantisation fused into the inner loop (BaseRT, gist.science technical
summary, "Methodologie" / "Specialisatie"): ``y[b][n] = sum_k deq(W)[n][k] *
x[b][k]`` in fp64, plus ``sum_k |deq(W)[n][k] * x[b][k]|`` for the tolerance
bound.  Every entry point is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 32

_c_u8p = ctypes.POINTER(ctypes.c_uint8)
_c_i8p = ctypes.POINTER(ctypes.c_int8)
_c_u16p = ctypes.POINTER(ctypes.c_uint16)
_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_f32p = ctypes.POINTER(ctypes.c_float)
_c_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no fast-math, no FP contraction)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
               "-fno-fast-math", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            L.oracle_half_to_double.restype = ctypes.c_double
            L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_double_to_half.restype = ctypes.c_uint16
            L.oracle_double_to_half.argtypes = [ctypes.c_double]
            L.oracle_scales_ld.restype = ctypes.c_int
            L.oracle_scales_ld.argtypes = [ctypes.c_int]
            L.oracle_quantize_q4.restype = ctypes.c_int
            L.oracle_quantize_q4.argtypes = [_c_f32p, ctypes.c_int, ctypes.c_int, _c_u8p, _c_u16p]
            for f in ("q2", "q3"):
                getattr(L, f"oracle_quantize_{f}").restype = ctypes.c_int
                getattr(L, f"oracle_quantize_{f}").argtypes = [
                    _c_f32p, ctypes.c_int, ctypes.c_int, _c_u8p, _c_u16p]
                getattr(L, f"oracle_dequantize_{f}").restype = None
                getattr(L, f"oracle_dequantize_{f}").argtypes = [
                    _c_u8p, _c_u16p, ctypes.c_int, ctypes.c_int, _c_f64p]
            L.oracle_quantize_q5.restype = ctypes.c_int
            L.oracle_quantize_q5.argtypes = [_c_f32p, ctypes.c_int, ctypes.c_int, _c_u8p, _c_u16p]
            L.oracle_dequantize_q5.restype = None
            L.oracle_dequantize_q5.argtypes = [_c_u8p, _c_u16p, ctypes.c_int, ctypes.c_int, _c_f64p]
            L.oracle_quantize_q6.restype = ctypes.c_int
            L.oracle_quantize_q6.argtypes = [_c_f32p, ctypes.c_int, ctypes.c_int, _c_u8p, _c_u16p]
            L.oracle_dequantize_q6.restype = None
            L.oracle_dequantize_q6.argtypes = [_c_u8p, _c_u16p, ctypes.c_int, ctypes.c_int, _c_f64p]
            L.oracle_quantize_q8.restype = ctypes.c_int
            L.oracle_quantize_q8.argtypes = [_c_f32p, ctypes.c_int, ctypes.c_int, _c_i8p, _c_u16p]
            L.oracle_dequantize_q4.restype = None
            L.oracle_dequantize_q4.argtypes = [_c_u8p, _c_u16p, ctypes.c_int, ctypes.c_int, _c_f64p]
            L.oracle_dequantize_q8.restype = None
            L.oracle_dequantize_q8.argtypes = [_c_i8p, _c_u16p, ctypes.c_int, ctypes.c_int, _c_f64p]
            gemv_args = [ctypes.c_void_p, _c_u16p, ctypes.c_int, ctypes.c_int, _c_u16p,
                         ctypes.c_int, ctypes.c_int, _c_f64p, _c_f64p, ctypes.c_int]
            L.oracle_gemv_q4.restype = ctypes.c_int
            L.oracle_gemv_q4.argtypes = gemv_args
            L.oracle_gemv_q2.restype = ctypes.c_int
            L.oracle_gemv_q2.argtypes = gemv_args
            L.oracle_gemv_q3.restype = ctypes.c_int
            L.oracle_gemv_q3.argtypes = gemv_args
            L.oracle_gemv_q5.restype = ctypes.c_int
            L.oracle_gemv_q5.argtypes = gemv_args
            L.oracle_gemv_q6.restype = ctypes.c_int
            L.oracle_gemv_q6.argtypes = gemv_args
            L.oracle_gemv_q8.restype = ctypes.c_int
            L.oracle_gemv_q8.argtypes = gemv_args
            L.oracle_moe_gemv_q4.restype = ctypes.c_int
            L.oracle_moe_gemv_q4.argtypes = [
                _c_u8p, _c_u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_longlong, ctypes.c_longlong, _c_u16p, ctypes.c_int, _c_i32p,
                _c_f32p, ctypes.c_int, ctypes.c_int, _c_f64p, _c_f64p, ctypes.c_int]
            L.oracle_silu.restype = ctypes.c_double
            L.oracle_silu.argtypes = [ctypes.c_double]
            L.oracle_swiglu_f16.restype = None
            L.oracle_swiglu_f16.argtypes = [_c_f64p, _c_f64p, ctypes.c_int, _c_u16p]
            L.oracle_attn_decode_q8.restype = ctypes.c_int
            L.oracle_attn_decode_q8.argtypes = [
                _c_i8p, _c_u16p, _c_i8p, _c_u16p, _c_u16p, _c_i32p, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _c_f64p, _c_f64p]
            _lib = L
        return _lib


def _p(a: np.ndarray, ct):
    return a.ctypes.data_as(ct)


def scales_ld(K: int) -> int:
    """Entries per scale-plane row: K/32 rounded up to a multiple of 8."""
    return int(lib().oracle_scales_ld(int(K)))


# ---------------------------------------------------------------- fp16 ----
def half_to_double(bits) -> np.ndarray:
    """binary16 bit patterns -> float64, element by element."""
    b = np.asarray(bits, dtype=np.uint16).ravel()
    f = lib().oracle_half_to_double
    return np.array([f(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def double_to_half(vals) -> np.ndarray:
    """float64 -> nearest binary16 bit pattern (ties to even)."""
    v = np.asarray(vals, dtype=np.float64).ravel()
    f = lib().oracle_double_to_half
    return np.array([f(float(t)) for t in v], dtype=np.uint16).reshape(np.shape(vals))


# ----------------------------------------------------------- quantisers ----
def quantize_q4(w: np.ndarray):
    """fp32 [N, K] -> (codes uint8 [N, K/2], scales fp16-bits uint16 [N, ldS])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, scales_ld(K)), dtype=np.uint16)
    rc = lib().oracle_quantize_q4(_p(w, _c_f32p), N, K, _p(codes, _c_u8p), _p(scales, _c_u16p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_q4 failed ({rc})")
    return codes, scales


def quantize_q2(w: np.ndarray):
    """fp32 [N, K] -> (codes uint8 [N, K/4]: the 2-bit plane, scales
    fp16-bits uint16 [N, ldS])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros((N, K // 4), dtype=np.uint8)
    scales = np.zeros((N, scales_ld(K)), dtype=np.uint16)
    rc = lib().oracle_quantize_q2(_p(w, _c_f32p), N, K, _p(codes, _c_u8p), _p(scales, _c_u16p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_q2 failed ({rc})")
    return codes, scales


def quantize_q3(w: np.ndarray):
    """fp32 [N, K] -> (codes uint8 [N, 3K/8]: 2-bit plane then 1-bit plane,
    scales fp16-bits uint16 [N, ldS])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros((N, 3 * K // 8), dtype=np.uint8)
    scales = np.zeros((N, scales_ld(K)), dtype=np.uint16)
    rc = lib().oracle_quantize_q3(_p(w, _c_f32p), N, K, _p(codes, _c_u8p), _p(scales, _c_u16p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_q3 failed ({rc})")
    return codes, scales


def quantize_q5(w: np.ndarray):
    """fp32 [N, K] -> (codes uint8 [N, 5K/8]: low-nibble plane then 1-bit
    plane, scales fp16-bits uint16 [N, ldS])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros((N, 5 * K // 8), dtype=np.uint8)
    scales = np.zeros((N, scales_ld(K)), dtype=np.uint16)
    rc = lib().oracle_quantize_q5(_p(w, _c_f32p), N, K, _p(codes, _c_u8p), _p(scales, _c_u16p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_q5 failed ({rc})")
    return codes, scales


def quantize_q6(w: np.ndarray):
    """fp32 [N, K] -> (codes uint8 [N, 3K/4]: low-nibble plane then 2-bit
    plane, scales fp16-bits uint16 [N, ldS])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros((N, 3 * K // 4), dtype=np.uint8)
    scales = np.zeros((N, scales_ld(K)), dtype=np.uint16)
    rc = lib().oracle_quantize_q6(_p(w, _c_f32p), N, K, _p(codes, _c_u8p), _p(scales, _c_u16p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_q6 failed ({rc})")
    return codes, scales


def quantize_q8(w: np.ndarray):
    """fp32 [N, K] -> (codes int8 [N, K], scales fp16-bits uint16 [N, ldS])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros((N, K), dtype=np.int8)
    scales = np.zeros((N, scales_ld(K)), dtype=np.uint16)
    rc = lib().oracle_quantize_q8(_p(w, _c_f32p), N, K, _p(codes, _c_i8p), _p(scales, _c_u16p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_q8 failed ({rc})")
    return codes, scales


def dequantize_q4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K = codes.shape[0], codes.shape[1] * 2
    assert scales.shape == (N, scales_ld(K))
    out = np.zeros((N, K), dtype=np.float64)
    lib().oracle_dequantize_q4(_p(codes, _c_u8p), _p(scales, _c_u16p), N, K, _p(out, _c_f64p))
    return out


def dequantize_q2(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K = codes.shape[0], codes.shape[1] * 4
    assert scales.shape == (N, scales_ld(K))
    out = np.zeros((N, K), dtype=np.float64)
    lib().oracle_dequantize_q2(_p(codes, _c_u8p), _p(scales, _c_u16p), N, K, _p(out, _c_f64p))
    return out


def dequantize_q3(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K = codes.shape[0], codes.shape[1] * 8 // 3
    assert scales.shape == (N, scales_ld(K))
    out = np.zeros((N, K), dtype=np.float64)
    lib().oracle_dequantize_q3(_p(codes, _c_u8p), _p(scales, _c_u16p), N, K, _p(out, _c_f64p))
    return out


def dequantize_q5(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K = codes.shape[0], codes.shape[1] * 8 // 5
    assert scales.shape == (N, scales_ld(K))
    out = np.zeros((N, K), dtype=np.float64)
    lib().oracle_dequantize_q5(_p(codes, _c_u8p), _p(scales, _c_u16p), N, K, _p(out, _c_f64p))
    return out


def dequantize_q6(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K = codes.shape[0], codes.shape[1] * 4 // 3
    assert scales.shape == (N, scales_ld(K))
    out = np.zeros((N, K), dtype=np.float64)
    lib().oracle_dequantize_q6(_p(codes, _c_u8p), _p(scales, _c_u16p), N, K, _p(out, _c_f64p))
    return out


def dequantize_q8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K = codes.shape
    assert scales.shape == (N, scales_ld(K))
    out = np.zeros((N, K), dtype=np.float64)
    lib().oracle_dequantize_q8(_p(codes, _c_i8p), _p(scales, _c_u16p), N, K, _p(out, _c_f64p))
    return out


# ----------------------------------------------------------------- GEMV ----
def _gemv(fn, codes, scales, K, x_bits, nthreads):
    x_bits = np.ascontiguousarray(np.atleast_2d(x_bits), dtype=np.uint16)
    B = x_bits.shape[0]
    assert x_bits.shape[1] == K
    N = codes.shape[0]
    assert scales.shape == (N, scales_ld(K))
    y = np.zeros((B, N), dtype=np.float64)
    absy = np.zeros((B, N), dtype=np.float64)
    rc = fn(codes.ctypes.data_as(ctypes.c_void_p), _p(scales, _c_u16p), N, K,
            _p(x_bits, _c_u16p), B, K, _p(y, _c_f64p), _p(absy, _c_f64p), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle gemv failed ({rc})")
    return y, absy


def gemv_q4(codes, scales, x_bits, nthreads: int = 1):
    """y[b][n] = sum_k deq(W)[n][k] * x[b][k] in fp64; returns (y, sum|terms|), both [B, N]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    return _gemv(lib().oracle_gemv_q4, codes, scales, codes.shape[1] * 2, x_bits, nthreads)


def gemv_q2(codes, scales, x_bits, nthreads: int = 1):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    return _gemv(lib().oracle_gemv_q2, codes, scales, codes.shape[1] * 4, x_bits, nthreads)


def gemv_q3(codes, scales, x_bits, nthreads: int = 1):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    return _gemv(lib().oracle_gemv_q3, codes, scales, codes.shape[1] * 8 // 3, x_bits, nthreads)


def gemv_q5(codes, scales, x_bits, nthreads: int = 1):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    return _gemv(lib().oracle_gemv_q5, codes, scales, codes.shape[1] * 8 // 5, x_bits, nthreads)


def gemv_q6(codes, scales, x_bits, nthreads: int = 1):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    return _gemv(lib().oracle_gemv_q6, codes, scales, codes.shape[1] * 4 // 3, x_bits, nthreads)


def gemv_q8(codes, scales, x_bits, nthreads: int = 1):
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    return _gemv(lib().oracle_gemv_q8, codes, scales, codes.shape[1], x_bits, nthreads)


def moe_gemv_q4(codes, scales, x_bits, x_per_slot: bool, expert_idx, route_w=None,
                nthreads: int = 1):
    """Routed-expert Q4 GEMV over an expert stack.

    codes: uint8 [E, N, K/2]; scales: uint16 [E, N, ldS]; x_bits: uint16 [B, K]
    (or [B, topk, K] when x_per_slot); expert_idx: int32 [B, topk];
    route_w: float32 [B, topk] or None.  Returns (y, absy, had_bad_index) with
    y [B, N] when route_w is given, else [B, topk, N].
    """
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    E, N, K2 = codes.shape
    K = K2 * 2
    idx = np.ascontiguousarray(expert_idx, dtype=np.int32)
    B, topk = idx.shape
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    assert x_bits.shape == ((B, topk, K) if x_per_slot else (B, K))
    if route_w is not None:
        route_w = np.ascontiguousarray(route_w, dtype=np.float32)
        assert route_w.shape == (B, topk)
        y = np.zeros((B, N), dtype=np.float64)
    else:
        y = np.zeros((B, topk, N), dtype=np.float64)
    absy = np.zeros_like(y)
    rc = lib().oracle_moe_gemv_q4(
        _p(codes, _c_u8p), _p(scales, _c_u16p), E, N, K, N * K2, N * scales.shape[2],
        _p(x_bits, _c_u16p), 1 if x_per_slot else 0, _p(idx, _c_i32p),
        _p(route_w, _c_f32p) if route_w is not None else None, B, topk,
        _p(y, _c_f64p), _p(absy, _c_f64p), int(nthreads))
    if rc not in (0, 2):
        raise ValueError(f"oracle moe gemv failed ({rc})")
    return y, absy, rc == 2


def silu(z: float) -> float:
    """silu(z) = z / (1 + e^-z) in fp64."""
    return float(lib().oracle_silu(float(z)))


def swiglu_f16(g, u) -> np.ndarray:
    """fp16 bits of silu(g) * u, evaluated in fp64 and rounded once (ties to
    even).  g, u: float arrays of the same shape (fp64 sums of the gate and up
    projections)."""
    g = np.ascontiguousarray(g, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    assert g.shape == u.shape
    h = np.empty(g.shape, dtype=np.uint16)
    lib().oracle_swiglu_f16(_p(g, _c_f64p), _p(u, _c_f64p), int(g.size), _p(h, _c_u16p))
    return h


def attn_decode_q8(k_codes, k_scales, vt_codes, v_scales, q_bits, lens, scale: float):
    """Decode attention over a Q8 KV cache (fp64).

    k_codes int8 [B, Hkv, Tmax, D]; k_scales uint16 [B, Hkv, Tmax, D/32];
    vt_codes int8 [B, Hkv, D, Tmax] (values transposed); v_scales uint16
    [B, Hkv, Tmax, D/32]; q_bits uint16 [B, Hkv*G, D]; lens int32 [B].
    Returns (o, abso, had_empty) with o, abso float64 [B, Hkv*G, D]."""
    k_codes = np.ascontiguousarray(k_codes, dtype=np.int8)
    k_scales = np.ascontiguousarray(k_scales, dtype=np.uint16)
    vt_codes = np.ascontiguousarray(vt_codes, dtype=np.int8)
    v_scales = np.ascontiguousarray(v_scales, dtype=np.uint16)
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    B, Hkv, Tmax, D = k_codes.shape
    H = q_bits.shape[1]
    assert H % Hkv == 0 and q_bits.shape == (B, H, D) and lens.shape == (B,)
    assert k_scales.shape == (B, Hkv, Tmax, D // 32) and v_scales.shape == k_scales.shape
    assert vt_codes.shape == (B, Hkv, D, Tmax)
    o = np.zeros((B, H, D), dtype=np.float64)
    abso = np.zeros_like(o)
    rc = lib().oracle_attn_decode_q8(
        _p(k_codes, _c_i8p), _p(k_scales, _c_u16p), _p(vt_codes, _c_i8p), _p(v_scales, _c_u16p),
        _p(q_bits, _c_u16p), _p(lens, _c_i32p), B, Hkv, H // Hkv, D, Tmax, float(scale),
        _p(o, _c_f64p), _p(abso, _c_f64p))
    if rc not in (0, 2):
        raise ValueError(f"oracle attention failed ({rc})")
    return o, abso, rc == 2

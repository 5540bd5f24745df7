"""ctypes binding of libbq.so -- same names as the C ABI in include/bq.h.

Argument marshalling only: every step of the GEMV runs in the CUDA library.
The raw functions take integer addresses (device or host, as the header says)
and return the bq_status code.  The helpers at the bottom accept torch tensors
(torch is used for device memory and streams only) and raise on a non-zero
status.  There is no fallback: if the library is missing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbq.so")

BQ_OK, BQ_ERR_NULL, BQ_ERR_SHAPE, BQ_ERR_ALIGN, BQ_ERR_BATCH = 0, 1, 2, 3, 4
BQ_ERR_EXPERT_INDEX, BQ_ERR_CUDA, BQ_ERR_TIMEOUT, BQ_ERR_WORKSPACE, BQ_ERR_RANGE = 5, 6, 7, 8, 9
BQ_EPI_NONE, BQ_EPI_SWIGLU = 0, 1
BQ_GEMV_STATIC_WEIGHTS, BQ_GEMV_ROWS16, BQ_GEMV_ROWS32 = 1, 2, 4


class bq_qmat(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("N", ctypes.c_int32), ("K", ctypes.c_int32)]


class bq_step_mat(ctypes.Structure):
    _fields_ = [("W", bq_qmat), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("B", ctypes.c_int32), ("stage", ctypes.c_int32),
                ("epilogue", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class bq_step_info(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("n_mats", ctypes.c_int32),
                ("n_stages", ctypes.c_int32), ("grid", ctypes.c_int32),
                ("max_stage_bands", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("stages_off", ctypes.c_uint64), ("mats_off", ctypes.c_uint64),
                ("ws_bytes", ctypes.c_uint64)]


class bq_step_wait(ctypes.Structure):
    _fields_ = [("wait_cycles", ctypes.c_int64), ("extra_arrivals", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class bq_kv_cache(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
                ("vt_codes", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("D", ctypes.c_int32), ("Tmax", ctypes.c_int32)]


class bq_gemv_geometry(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("rows", "chunks", "chunks_per_band",
                                               "chunks_per_worker", "grid", "cluster",
                                               "cross_cta_bands", "reserved")]


class BQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {bq_status_string(status)} ({status})")
        self.status = status


_lib = None
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_QP = ctypes.POINTER(bq_qmat)
_SMP = ctypes.POINTER(bq_step_mat)
_SIP = ctypes.POINTER(bq_step_info)

# name -> (restype, argtypes); mirrors include/bq.h
_SIGS = {
    "bq_status_string": (ctypes.c_char_p, [_i32]),
    "bq_scales_ld": (_i32, [_i32]),
    "bq_gemv_workspace_bytes": (_sz, [_i32, _i32]),
    "bq_gemv_q4": (_i32, [_QP, _vp, _i32, _vp, _vp, _sz, _vp, _vp]),
    "bq_gemv_ex": (_i32, [_i32, _QP, _vp, _i32, _vp, _i32, _i32, _vp, _sz, _vp, _vp]),
    "bq_gemv_q8": (_i32, [_QP, _vp, _i32, _vp, _vp, _sz, _vp, _vp]),
    "bq_gemv_q4_noalloc": (_i32, [_QP, _vp, _i32, _vp, _vp, _vp]),
    "bq_gemv_q4_noalloc_scratch": (_i32, [ctypes.POINTER(_vp), ctypes.POINTER(_sz)]),
    "bq_step_plan_bytes": (_sz, [_i32]),
    "bq_gemv_geometry_of": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32,
                                    ctypes.POINTER(bq_gemv_geometry)]),
    "bq_step_plan": (_i32, [_i32, _SMP, _i32, _vp, _sz, _SIP]),
    "bq_step_run": (_i32, [_SIP, _vp, _vp, _sz, _vp, _vp]),
    "bq_step_run_ex": (_i32, [_SIP, _vp, _vp, _sz, ctypes.POINTER(bq_step_wait), _vp, _vp]),
    "bq_moe_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "bq_verify_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "bq_attn_workspace_bytes": (_sz, [_i32, _i32]),
    "bq_attn_decode_q8": (_i32, [ctypes.POINTER(bq_kv_cache), _vp, _vp, _i32, _i32, _i32,
                                 ctypes.c_float, _vp, _vp, _sz, _vp, _vp]),
    "bq_verify_gemm": (_i32, [_i32, _QP, _vp, _i32, _vp, _vp, _sz, _vp, _vp]),
    "bq_moe_gemv_q4": (_i32, [_QP, _i32, _i64, _i64, _vp, _i32, _vp, _vp, _i32, _i32, _vp,
                              _vp, _sz, _vp, _vp]),
    "bq_moe_gemv_ex": (_i32, [_QP, _i32, _i64, _i64, _vp, _i32, _vp, _vp, _i32, _i32, _vp, _i32,
                              _vp, _sz, _vp, _vp]),
    "bq_quantize_q8": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_quantize_q4": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_dequantize_q8": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_dequantize_q4": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_quantize_q2": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_quantize_q3": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_dequantize_q2": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_dequantize_q3": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_quantize_q6": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_quantize_q5": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_dequantize_q5": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_dequantize_q6": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_planes_to_blocks_q4": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_planes_to_blocks_q8": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "bq_blocks_to_planes_q4": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_blocks_to_planes_q8": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "bq_quantize_q4_dev": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "bq_quantize_q8_dev": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "bq_quantize_q2_dev": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "bq_quantize_q3_dev": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "bq_quantize_q6_dev": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "bq_quantize_q5_dev": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
}


def lib() -> ctypes.CDLL:
    """Load libbq.so; raises if it has not been built (no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m quantised_weight_gemv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def __getattr__(name):
    # module-level access to the raw C functions: bq.bq_gemv_q4(...)
    if name in _SIGS:
        return getattr(lib(), name)
    raise AttributeError(name)


def bq_status_string(status: int) -> str:
    return lib().bq_status_string(int(status)).decode()


def check(fn: str, status: int) -> None:
    if status != BQ_OK:
        raise BQError(fn, status)


# ------------------------------------------------------- torch helpers ----
def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


_ROW_BYTES = {2: lambda K: K // 4, 3: lambda K: 3 * K // 8, 4: lambda K: K // 2,
              5: lambda K: 5 * K // 8, 6: lambda K: 3 * K // 4, 8: lambda K: K}


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _on_device(fn: str, **tensors) -> None:
    """The C library takes raw device pointers and cannot tell a host
    pointer from a device one: refuse host tensors before any launch."""
    for name, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise ValueError(f"{fn}: {name} must be a CUDA tensor (got device {t.device})")


def _check_planes(fn: str, fmt: int, W: bq_qmat) -> None:
    """Device planes behind a bq_qmat made by qmat(): on the GPU and large
    enough for N rows of the format (the kernel reads them through TMA maps
    built from N and K alone)."""
    refs = getattr(W, "_refs", None)
    if refs is None:
        return
    codes, scales = refs
    _on_device(fn, codes=codes, scales=scales)
    if fmt in _ROW_BYTES and W.K % 32 == 0:
        if _nbytes(codes) < W.N * _ROW_BYTES[fmt](W.K):
            raise ValueError(f"{fn}: codes hold {_nbytes(codes)} bytes, "
                             f"{W.N} rows of Q{fmt} need {W.N * _ROW_BYTES[fmt](W.K)}")
        if _nbytes(scales) < W.N * scales_ld(W.K) * 2:
            raise ValueError(f"{fn}: scales hold {_nbytes(scales)} bytes, "
                             f"need {W.N * scales_ld(W.K) * 2}")


def qmat(codes, scales, N: int, K: int) -> bq_qmat:
    """bq_qmat over two tensors (device planes for GEMV, host for pack calls).

    The struct keeps references to both tensors, so their memory stays
    allocated for as long as the bq_qmat is alive."""
    m = bq_qmat(codes.data_ptr(), scales.data_ptr(), int(N), int(K))
    m._refs = (codes, scales)
    return m


def gemv_geometry(fmt: int, N: int, K: int, B: int, flags: int = 0, sm_count: int = 0) -> dict:
    """The launch geometry bq_gemv_ex chooses (bq_gemv_geometry_of); with
    sm_count > 0 computed for such a device without touching one."""
    g = bq_gemv_geometry()
    check("bq_gemv_geometry_of",
          lib().bq_gemv_geometry_of(fmt, N, K, B, flags, sm_count, ctypes.byref(g)))
    return {n: getattr(g, n) for n, _ in bq_gemv_geometry._fields_ if n != "reserved"}


def scales_ld(K: int) -> int:
    return int(lib().bq_scales_ld(int(K)))


def workspace(nbytes: int, device):
    """A zero-filled caller-owned workspace of nbytes (torch allocation)."""
    import torch
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def gemv(fmt: int, W: bq_qmat, x, y, ws, status=None, stream=None, epilogue: int = BQ_EPI_NONE,
         flags: int = 0) -> None:
    """y[B, N] (fp32) = deq(W) . x[B, K] (fp16), through bq_gemv_q4 / bq_gemv_q8;
    Q6, an epilogue (BQ_EPI_SWIGLU: y is fp16 [B, N/2]) or flags go through
    bq_gemv_ex."""
    _on_device("gemv", x=x, y=y, ws=ws, status=status)
    _check_planes("gemv", fmt, W)
    if x.dim() != 2 or x.shape[1] != W.K or x.element_size() != 2 or not x.is_contiguous():
        raise ValueError(f"gemv: x must be a contiguous [B, {W.K}] tensor of fp16 bits, got "
                         f"{tuple(x.shape)} {x.dtype}")
    B = x.shape[0]
    need = B * W.N * (4 if epilogue == BQ_EPI_NONE else 1)      # fp32 [B][N] or fp16 [B][N/2]
    if not y.is_contiguous() or _nbytes(y) < need:
        raise ValueError(f"gemv: y must be contiguous with at least {need} bytes")
    if epilogue == BQ_EPI_NONE and flags == 0 and fmt in (4, 8):   # (Q2, Q3, Q5, Q6: bq_gemv_ex)
        fn = lib().bq_gemv_q4 if fmt == 4 else lib().bq_gemv_q8
        rc = fn(ctypes.byref(W), x.data_ptr(), B, y.data_ptr(), ws.data_ptr(),
                ws.numel() * ws.element_size(), _ptr(status), _stream_ptr(stream))
        check(f"bq_gemv_q{fmt}", rc)
        return
    rc = lib().bq_gemv_ex(int(fmt), ctypes.byref(W), x.data_ptr(), B, y.data_ptr(), int(epilogue),
                          int(flags), ws.data_ptr(), ws.numel() * ws.element_size(), _ptr(status),
                          _stream_ptr(stream))
    check("bq_gemv_ex", rc)


def verify_gemm(fmt: int, W: bq_qmat, x, y, ws, status=None, stream=None) -> None:
    """y[B, N] (fp32) = deq(W) . x[B, K] (fp16) for a verification batch of
    B = 1..32 rows, through bq_verify_gemm (Q4 or Q8; tensor cores)."""
    _on_device("verify_gemm", x=x, y=y, ws=ws, status=status)
    _check_planes("verify_gemm", fmt, W)
    if x.dim() != 2 or x.shape[1] != W.K or x.element_size() != 2 or not x.is_contiguous():
        raise ValueError(f"verify_gemm: x must be a contiguous [B, {W.K}] tensor of fp16 bits, got "
                         f"{tuple(x.shape)} {x.dtype}")
    B = x.shape[0]
    if not y.is_contiguous() or _nbytes(y) < B * W.N * 4:
        raise ValueError(f"verify_gemm: y must be contiguous with at least {B * W.N * 4} bytes")
    check("bq_verify_gemm", lib().bq_verify_gemm(int(fmt), ctypes.byref(W), x.data_ptr(), B,
                                                 y.data_ptr(), ws.data_ptr(),
                                                 ws.numel() * ws.element_size(), _ptr(status),
                                                 _stream_ptr(stream)))


def kv_cache(k_codes, k_scales, vt_codes, v_scales) -> bq_kv_cache:
    """A bq_kv_cache over device tensors: k_codes int8 [B, Hkv, Tmax, D],
    k_scales fp16 bits [B, Hkv, Tmax, D/32], vt_codes int8 [B, Hkv, D, Tmax],
    v_scales fp16 bits [B, Hkv, Tmax, D/32] (the tensors stay owned by the
    caller; the struct keeps references)."""
    _on_device("kv_cache", k_codes=k_codes, k_scales=k_scales, vt_codes=vt_codes, v_scales=v_scales)
    B, Hkv, Tmax, D = k_codes.shape
    if (tuple(vt_codes.shape) != (B, Hkv, D, Tmax) or tuple(k_scales.shape) != (B, Hkv, Tmax, D // 32)
            or tuple(v_scales.shape) != (B, Hkv, Tmax, D // 32)
            or any(not t.is_contiguous() for t in (k_codes, k_scales, vt_codes, v_scales))
            or k_codes.element_size() != 1 or vt_codes.element_size() != 1
            or k_scales.element_size() != 2 or v_scales.element_size() != 2):
        raise ValueError("kv_cache: shapes/dtypes/contiguity do not match the cache layout")
    kv = bq_kv_cache(k_codes.data_ptr(), k_scales.data_ptr(), vt_codes.data_ptr(),
                     v_scales.data_ptr(), int(D), int(Tmax))
    kv._refs = (k_codes, k_scales, vt_codes, v_scales)
    kv.B, kv.Hkv = int(B), int(Hkv)
    return kv


def attn_decode_q8(kv: bq_kv_cache, q, lens, G: int, scale: float, o, ws, status=None,
                   stream=None) -> None:
    """o[B, Hkv*G, D] (fp32) = softmax(scale q K^T) V over the Q8 cache, per
    sequence over its first lens[b] positions (bq_attn_decode_q8)."""
    _on_device("attn_decode_q8", q=q, lens=lens, o=o, ws=ws, status=status)
    B, Hkv = kv.B, kv.Hkv
    if tuple(q.shape) != (B, Hkv * G, kv.D) or q.element_size() != 2 or not q.is_contiguous():
        raise ValueError(f"attn_decode_q8: q must be contiguous fp16 bits [{B}, {Hkv * G}, {kv.D}]")
    if lens.numel() != B or lens.element_size() != 4 or not lens.is_contiguous():
        raise ValueError(f"attn_decode_q8: lens must be int32 [{B}]")
    if not o.is_contiguous() or _nbytes(o) < B * Hkv * G * kv.D * 4:
        raise ValueError("attn_decode_q8: o too small")
    check("bq_attn_decode_q8", lib().bq_attn_decode_q8(
        ctypes.byref(kv), q.data_ptr(), lens.data_ptr(), B, Hkv, int(G), float(scale), o.data_ptr(),
        ws.data_ptr(), ws.numel() * ws.element_size(), _ptr(status), _stream_ptr(stream)))


def moe_gemv_q4(Wstack: bq_qmat, E: int, codes_stride: int, scales_stride: int, x,
                x_per_slot: bool, expert_idx, route_w, y, ws, status=None, stream=None,
                epilogue: int = BQ_EPI_NONE) -> None:
    """Routed-expert Q4 GEMV (bq_moe_gemv_q4); with epilogue BQ_EPI_SWIGLU,
    per-slot fp16 h (bq_moe_gemv_ex)."""
    _on_device("moe_gemv_q4", x=x, expert_idx=expert_idx, route_w=route_w, y=y, ws=ws,
               status=status)
    refs = getattr(Wstack, "_refs", None)
    if refs is not None:
        _on_device("moe_gemv_q4", codes=refs[0], scales=refs[1])
    B, topk = expert_idx.shape
    rc = lib().bq_moe_gemv_ex(ctypes.byref(Wstack), int(E), int(codes_stride), int(scales_stride),
                              x.data_ptr(), 1 if x_per_slot else 0, expert_idx.data_ptr(),
                              _ptr(route_w), B, topk, y.data_ptr(), int(epilogue), ws.data_ptr(),
                              ws.numel() * ws.element_size(), _ptr(status), _stream_ptr(stream))
    check("bq_moe_gemv_ex", rc)


class StepPlan:
    """A decode-step plan: device plan buffer + host info + workspace (torch
    allocations owned by this object), built once by bq_step_plan."""

    def __init__(self, fmt: int, entries, device):
        """entries: iterable of (bq_qmat, x, y, stage) or (bq_qmat, x, y, stage,
        epilogue) with device tensors."""
        import torch
        entries = list(entries)
        arr = (bq_step_mat * len(entries))()
        self._refs = []
        for i, e in enumerate(entries):
            W, x, y, stage = e[:4]
            epi = e[4] if len(e) > 4 else BQ_EPI_NONE
            _on_device("StepPlan", x=x, y=y)
            _check_planes("StepPlan", fmt, W)
            arr[i] = bq_step_mat(W, x.data_ptr(), y.data_ptr(), int(x.shape[0]), int(stage),
                                 int(epi), 0)
            self._refs += [W, x, y]
        nbytes = lib().bq_step_plan_bytes(len(entries))
        self.plan = torch.empty(nbytes + 64, dtype=torch.uint8, device=device)
        off = (-self.plan.data_ptr()) % 64
        self.plan_ptr = self.plan.data_ptr() + off
        self.info = bq_step_info()
        check("bq_step_plan", lib().bq_step_plan(int(fmt), arr, len(entries), self.plan_ptr,
                                                 nbytes, ctypes.byref(self.info)))
        self.ws = workspace(self.info.ws_bytes, device)

    def run(self, status=None, stream=None, wait_cycles: int | None = None,
            extra_arrivals: int = 0) -> None:
        """One step.  wait_cycles / extra_arrivals: bounded-wait options
        (bq_step_run_ex); None / 0 are the defaults."""
        if wait_cycles is None and extra_arrivals == 0:
            check("bq_step_run", lib().bq_step_run(ctypes.byref(self.info), self.plan_ptr,
                                                   self.ws.data_ptr(), self.ws.numel(),
                                                   _ptr(status), _stream_ptr(stream)))
            return
        w = bq_step_wait(int(wait_cycles or 0), int(extra_arrivals), 0)
        check("bq_step_run_ex", lib().bq_step_run_ex(ctypes.byref(self.info), self.plan_ptr,
                                                     self.ws.data_ptr(), self.ws.numel(),
                                                     ctypes.byref(w), _ptr(status),
                                                     _stream_ptr(stream)))


def quantize_dev(fmt: int, w, codes, scales, status=None, stream=None) -> None:
    _on_device("quantize_dev", w=w, codes=codes, scales=scales, status=status)
    N, K = w.shape
    if (w.element_size() != 4 or not w.is_contiguous() or not codes.is_contiguous()
            or not scales.is_contiguous()):
        raise ValueError("quantize_dev: w must be contiguous fp32 [N, K]; codes and scales contiguous")
    if fmt in _ROW_BYTES and K % 32 == 0 and (_nbytes(codes) < N * _ROW_BYTES[fmt](K)
                                              or _nbytes(scales) < N * scales_ld(K) * 2):
        raise ValueError(f"quantize_dev: planes too small for {N} rows of Q{fmt} with K = {K}")
    fn = {2: lib().bq_quantize_q2_dev, 3: lib().bq_quantize_q3_dev, 4: lib().bq_quantize_q4_dev,
          5: lib().bq_quantize_q5_dev, 6: lib().bq_quantize_q6_dev, 8: lib().bq_quantize_q8_dev}[fmt]
    check(f"bq_quantize_q{fmt}_dev",
          fn(w.data_ptr(), N, K, codes.data_ptr(), scales.data_ptr(), _ptr(status),
             _stream_ptr(stream)))

"""bq_gemv_q4_noalloc: the Q4 GEMV for callers that cannot allocate device
memory (frameworks that own every allocation, decode loops that must not call
cudaMalloc).  Its scratch is a fixed array inside the library, so the checks
here are that two calls in a row agree with the workspace entry point and the
oracle (the array keeps the previous call's contents), and that a matrix too
large for the array is refused before anything is launched.

A third check poisons the fixed array (non-zero band counters, NaN partial
sums, as a call killed mid-way or a stray writer could leave it) before a
call whose bands are summed across CTAs: the call must clear the counters it
uses itself, so its result must still match.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest

from quantised_weight_gemv_b200 import bq, synth
from tests.gpu_helpers import DEV, REL, ABS, check_tol, dev, gpu_gemv, new_status, oracle_gemv, quantize

FAKE = 0x7f0000000000


def test_noalloc_rejects_oversized_before_launch():
    W = bq.bq_qmat(FAKE, FAKE, (1 << 20) + 1, 256)
    assert bq.lib().bq_gemv_q4_noalloc(ctypes.byref(W), FAKE, 1, FAKE, None, None) == bq.BQ_ERR_WORKSPACE
    W = bq.bq_qmat(FAKE, FAKE, 64, 256)
    assert bq.lib().bq_gemv_q4_noalloc(ctypes.byref(W), FAKE, 9, FAKE, None, None) == bq.BQ_ERR_BATCH
    assert bq.lib().bq_gemv_q4_noalloc(ctypes.byref(W), None, 1, FAKE, None, None) == bq.BQ_ERR_NULL


@pytest.mark.gpu
@pytest.mark.parametrize("N,K,B", [(1000, 3072, 3), (16384, 2048, 1), (33, 288, 8)])
def test_noalloc_two_calls_match_workspace_entry_point(N, K, B):
    import torch
    w = synth.weights_f32(synth.key(0, 84, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(4, w)
    x = synth.activations_f16_bits(synth.key(0, 84, N, K, synth.KIND_X), B, K)
    y_ws = gpu_gemv(4, codes, scales, x)                       # existing entry point
    y_ref, absy = oracle_gemv(4, codes, scales, x)
    c, s, xt = dev(codes), dev(scales), dev(x)
    W = bq.qmat(c, s, N, K)
    for _ in range(2):
        y = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
        st = new_status()
        rc = bq.lib().bq_gemv_q4_noalloc(ctypes.byref(W), xt.data_ptr(), B, y.data_ptr(),
                                         st.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == bq.BQ_OK
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        yn = y.cpu().numpy()
        check_tol(yn, y_ref, absy)
        assert np.all(np.abs(yn.astype(np.float64) - y_ws) <= REL * absy + ABS)


class _DevView:
    """A raw device range as a torch tensor (no copy), through the CUDA array
    interface."""

    def __init__(self, ptr, nbytes):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1",
                                         "data": (ptr, False), "version": 3}


@pytest.mark.gpu
@pytest.mark.parametrize("N,K,B", [(1000, 3072, 3), (4096, 4096, 1)])
def test_noalloc_result_does_not_depend_on_what_the_array_held(N, K, B):
    import torch
    p, nb = ctypes.c_void_p(), ctypes.c_size_t()
    assert bq.lib().bq_gemv_q4_noalloc_scratch(ctypes.byref(p), ctypes.byref(nb)) == bq.BQ_OK
    assert nb.value == 917504 and p.value
    scratch = torch.as_tensor(_DevView(p.value, nb.value), device=DEV)
    assert scratch.numel() == nb.value
    w = synth.weights_f32(synth.key(0, 85, N, K, synth.KIND_W), N, K)
    codes, scales = quantize(4, w)
    x = synth.activations_f16_bits(synth.key(0, 85, N, K, synth.KIND_X), B, K)
    y_ref, absy = oracle_gemv(4, codes, scales, x)
    c, s, xt = dev(codes), dev(scales), dev(x)
    W = bq.qmat(c, s, N, K)
    for poison in (0x01, 0xFF):          # counters 0x01010101 / -1, partials tiny / NaN
        scratch.fill_(poison)
        torch.cuda.synchronize()
        y = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
        st = new_status()
        rc = bq.lib().bq_gemv_q4_noalloc(ctypes.byref(W), xt.data_ptr(), B, y.data_ptr(),
                                         st.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == bq.BQ_OK
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        check_tol(y.cpu().numpy(), y_ref, absy)

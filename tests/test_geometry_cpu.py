"""Host-side launch geometry (bq_gemv_geometry_of, computed for a given SM
count without a device), checked against brute-force definitions: the chunk
counts, the stream-K split, whether some band's chunks span CTAs, and -- when
the launch runs as thread-block clusters -- that every band lies inside one
cluster, so that its cross-CTA sum can go through the cluster's shared
memory."""
import ctypes

import pytest

from quantised_weight_gemv_b200 import bq

WARPS = 8            # worker warps per CTA
CHUNK_K = 256        # weights along K per chunk


def _cdiv(a, b):
    return -(-a // b)


def _brute(N, K, rows, cpw):
    """(some band spans CTAs, first CTA of each band, last CTA of each band),
    walking every band."""
    cpb = _cdiv(K, CHUNK_K)
    nbands = _cdiv(N, rows)
    first_cta = [(b * cpb // cpw) // WARPS for b in range(nbands)]
    last_cta = [(((b + 1) * cpb - 1) // cpw) // WARPS for b in range(nbands)]
    crosses = any(f != l for f, l in zip(first_cta, last_cta))
    return crosses, first_cta, last_cta


SHAPES = [(1, 32), (16, 256), (40, 2048), (777, 3072), (2048, 2048), (3072, 2048),
          (16384, 2048), (2048, 8192), (4096, 4096), (6144, 4096), (24576, 4096),
          (4096, 12288), (5120, 5120), (7168, 5120), (51200, 5120), (5120, 25600),
          (1024, 16384), (1000, 1792), (12345, 800)]


@pytest.mark.parametrize("sm_count", [148, 132, 100])
@pytest.mark.parametrize("fmt,flags", [(4, 0), (4, bq.BQ_GEMV_ROWS16), (4, bq.BQ_GEMV_ROWS32),
                                       (8, 0), (4, bq.BQ_GEMV_STATIC_WEIGHTS), (6, 0),
                                       (5, 0), (3, 0), (2, 0)])
@pytest.mark.parametrize("B", [1, 8])
def test_geometry_matches_brute_force(sm_count, fmt, flags, B):
    cap = min(2 * sm_count, 512)
    for N, K in SHAPES:
        if (fmt in (2, 6) and K % 64) or (fmt in (3, 5) and K % 128):
            continue
        g = bq.gemv_geometry(fmt, N, K, B, flags, sm_count=sm_count)
        rows = g["rows"]
        if fmt != 4 or flags == bq.BQ_GEMV_ROWS16:
            assert rows == 16
        elif flags == bq.BQ_GEMV_ROWS32:
            assert rows == 32
        else:
            assert rows in (16, 32)
        cpb = _cdiv(K, CHUNK_K)
        T = _cdiv(N, rows) * cpb
        assert g["chunks_per_band"] == cpb and g["chunks"] == T
        G0 = min(cap, T)
        cpw = max(1, _cdiv(T, G0 * WARPS))
        assert g["chunks_per_worker"] == cpw, (N, K)
        # every chunk has a worker in the launched grid
        assert g["grid"] * WARPS * cpw >= T and g["grid"] <= cap
        crosses, first_cta, last_cta = _brute(N, K, rows, cpw)
        assert g["cross_cta_bands"] == int(crosses), (N, K, rows)
        C = g["cluster"]
        if C == 1:
            continue
        assert crosses and C in (2, 4, 8) and g["grid"] % C == 0, (N, K, C)
        assert all(f // C == l // C for f, l in zip(first_cta, last_cta)), (N, K, C)


def test_geometry_examples_on_148_sms():
    """A few launches of the 16-layer hidden-2048 decoder and others, on 148
    SMs: which work units and which cross-CTA sums they get."""
    g = lambda *a, **k: bq.gemv_geometry(*a, sm_count=148, **k)
    down = g(4, 2048, 8192, 1)       # 64 bands of 32 chunks: each band spans 4 CTAs
    assert down["cross_cta_bands"] == 1 and down["cluster"] == 4 and down["grid"] == 256
    sq = g(4, 4096, 4096, 1, bq.BQ_GEMV_ROWS32)   # 32-row bands span 2 CTAs ...
    assert sq["cross_cta_bands"] == 1 and sq["cluster"] == 2
    sq16 = g(4, 4096, 4096, 1, bq.BQ_GEMV_ROWS16)  # ... 16-row bands fit in one
    assert sq16["cross_cta_bands"] == 0 and sq16["cluster"] == 1
    k5120 = g(4, 5120, 5120, 1, bq.BQ_GEMV_ROWS32)  # 20 chunks per band: would need 5
    assert k5120["cross_cta_bands"] == 1 and k5120["cluster"] == 1


def test_geometry_validation():
    f = lambda *a: bq.lib().bq_gemv_geometry_of(*a, None)
    out = bq.bq_gemv_geometry()
    call = lambda fmt, N, K, B, flags, sm: bq.lib().bq_gemv_geometry_of(
        fmt, N, K, B, flags, sm, ctypes.byref(out))
    assert f(4, 64, 256, 1, 0, 148) == bq.BQ_ERR_NULL
    assert call(7, 64, 256, 1, 0, 148) == bq.BQ_ERR_SHAPE
    assert call(5, 64, 192, 1, 0, 148) == bq.BQ_ERR_SHAPE          # Q5: K % 128
    assert call(6, 64, 96, 1, 0, 148) == bq.BQ_ERR_SHAPE           # Q6: K % 64
    assert call(3, 64, 192, 1, 0, 148) == bq.BQ_ERR_SHAPE          # Q3: K % 128
    assert call(2, 64, 96, 1, 0, 148) == bq.BQ_ERR_SHAPE           # Q2: K % 64
    assert call(1, 64, 256, 1, 0, 148) == bq.BQ_ERR_SHAPE
    assert call(3, 64, 256, 1, 0, 148) == bq.BQ_OK and out.rows == 16
    assert call(2, 64, 256, 1, bq.BQ_GEMV_ROWS32, 148) == bq.BQ_ERR_SHAPE
    assert call(4, 64, 48, 1, 0, 148) == bq.BQ_ERR_SHAPE
    assert call(4, 0, 256, 1, 0, 148) == bq.BQ_ERR_SHAPE
    assert call(4, 64, 256, 0, 0, 148) == bq.BQ_ERR_BATCH
    assert call(4, 64, 256, 9, 0, 148) == bq.BQ_ERR_BATCH
    assert call(4, 64, 256, 1, 8, 148) == bq.BQ_ERR_SHAPE
    assert call(4, 64, 256, 1, bq.BQ_GEMV_ROWS16 | bq.BQ_GEMV_ROWS32, 148) == bq.BQ_ERR_SHAPE
    assert call(8, 64, 256, 1, bq.BQ_GEMV_ROWS32, 148) == bq.BQ_ERR_SHAPE
    assert call(4, 64, 256, 1, 0, -1) == bq.BQ_ERR_SHAPE
    assert call(4, 64, 256, 1, 0, 148) == bq.BQ_OK

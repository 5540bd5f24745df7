"""Failure detection on the GPU without a fault: every wait in the kernels is
bounded, and a wait that runs out reports BQ_ERR_TIMEOUT in the caller's
status word, stops the kernel and leaves the context usable.

The test makes a decode-step plan's grid barrier wait for one arrival more
than the grid makes (bq_step_run_ex, extra_arrivals = 1 -- a flag nothing
sets) with a short limit of about a millisecond.  Every CTA's first barrier
then runs out: the run must report the timeout, the stage before the barrier
must be complete and correct, the stages after it untouched, and after the
workspace is zero-filled again a normal run of the same plan must match the
oracle.  Nothing faults, traps or hangs: the waits end by their own limit."""
import time

import numpy as np
import pytest

from quantised_weight_gemv_b200 import bq
from tests.gpu_helpers import DEV, check_tol, new_status, oracle_gemv
from tests.test_gpu_parity import _step_entries

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 1 << 7          # 1 << BQ_ERR_TIMEOUT
SHORT = 2_000_000             # SM cycles: about 1 ms at 1.9 GHz


@pytest.mark.parametrize("fmt", [4, 8])
def test_grid_barrier_wait_runs_out_and_reports_timeout(fmt):
    import torch
    assert bq.BQ_ERR_TIMEOUT == 7
    specs = [(2048, 2048, 1, 0), (77, 288, 3, 0), (1000, 96, 3, 1), (4096, 4096, 8, 2)]
    entries, host = _step_entries(fmt, specs, 31 + fmt)
    plan = bq.StepPlan(fmt, entries, DEV)
    st = new_status()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    plan.run(st, wait_cycles=SHORT, extra_arrivals=1)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(st.item()) & TIMEOUT_BIT, f"status {int(st.item()):#x}"
    assert elapsed < 1.0, f"the run took {elapsed:.3f} s: the short limit was not applied"
    for (W, x, y, stage), (codes, scales, xb) in zip(entries, host):
        yg = y.cpu().numpy()
        if stage == 0:          # finished before the failed barrier
            y_ref, absy = oracle_gemv(fmt, codes, scales, xb)
            check_tol(yg, y_ref, absy)
        else:                   # never started
            assert np.all(np.isnan(yg)), f"stage {stage} was written after a failed barrier"
    # the context is usable: zero-fill the workspace again and run normally
    plan.ws.zero_()
    st.zero_()
    for e in entries:
        e[2].fill_(float("nan"))
    plan.run(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for (W, x, y, stage), (codes, scales, xb) in zip(entries, host):
        y_ref, absy = oracle_gemv(fmt, codes, scales, xb)
        check_tol(y.cpu().numpy(), y_ref, absy)


def test_short_limit_alone_does_not_fire():
    """A millisecond is far longer than a real grid barrier (about a
    microsecond): with no extra arrivals the short limit never runs out."""
    import torch
    specs = [(3072, 2048, 1, 0), (2048, 2048, 1, 1), (2048, 8192, 1, 2), (16384, 2048, 1, 3)]
    entries, host = _step_entries(4, specs, 77)
    plan = bq.StepPlan(4, entries, DEV)
    st = new_status()
    for _ in range(5):
        plan.run(st, wait_cycles=SHORT)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for (W, x, y, stage), (codes, scales, xb) in zip(entries, host):
        y_ref, absy = oracle_gemv(4, codes, scales, xb)
        check_tol(y.cpu().numpy(), y_ref, absy)

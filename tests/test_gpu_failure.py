"""Failure detection on the GPU without a GPU fault: a bounded device wait that
nothing completes gives up after its limit, the host reads DG_ERR_TIMEOUT, and
the same process then runs a denoise step normally (the context is usable)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from token_canvas_denoising_b200 import inputs as fx

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    from token_canvas_denoising_b200 import _lib as L
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    lib = L.load()
    st = lib.dg_selftest_wait_timeout(None)
    assert st == L.DG_ERR_TIMEOUT, (st, lib.dg_last_error())
    cv, keep = from_workload(fx.make_workload(fx.CONFIGS["tiny"]))
    try:
        out = cv.step(schedule(8, 0.05, True), debug=True)
        cv.sync()
        assert np.all(np.isfinite(out["ent"].cpu().numpy()))
    finally:
        cv.close()

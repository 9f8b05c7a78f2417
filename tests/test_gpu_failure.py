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


def test_workspace_cap_reports_oom_before_any_allocation(monkeypatch):
    """DG_WORKSPACE_LIMIT_MB caps the context's workspace: a cap below what the
    workload needs makes dg_canvas_init return DG_ERR_OOM (checked on the host
    before the allocation); without the cap the same workload initialises."""
    from token_canvas_denoising_b200 import _lib as L
    from token_canvas_denoising_b200.canvas import from_workload
    wl = fx.make_workload(fx.CONFIGS["tiny"])
    monkeypatch.setenv("DG_WORKSPACE_LIMIT_MB", "0.01")
    with pytest.raises(L.DgError) as e:
        from_workload(wl)
    assert e.value.status == L.DG_ERR_OOM
    assert "DG_WORKSPACE_LIMIT_MB" in str(e.value)
    monkeypatch.delenv("DG_WORKSPACE_LIMIT_MB")
    cv, keep = from_workload(wl)
    cv.close()


@pytest.mark.parametrize("noalloc", [False, True])
def test_op_entry_points_report_a_nan_entropy(noalloc):
    """The single-operation entry points return after queuing their kernels;
    dg_ops_check then reports what the kernels found. A hidden state of NaNs
    gives NaN logits, which the entropy merge flags (no memory access depends
    on the values); the check reports DG_ERR_DEVICE_CHECK once and clears the
    word, after which a normal call checks clean."""
    import ctypes as C
    from token_canvas_denoising_b200 import _lib as L
    lib = L.load()
    M, d, V = 64, 128, 4096
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    w = torch.randn(V, d, device="cuda").to(torch.bfloat16)
    ent = torch.empty(M, dtype=torch.float32, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    fn = lib.dg_lmhead_entropy_noalloc if noalloc else lib.dg_lmhead_entropy
    p = lambda t: C.c_void_p(t.data_ptr())
    assert lib.dg_ops_check(s) == L.DG_OK
    hs = torch.full((M, d), float("nan"), device="cuda").to(torch.bfloat16)
    assert fn(L.DG_BF16, p(hs), p(w), None, M, d, V, p(ent), p(am), s) == L.DG_OK
    assert lib.dg_ops_check(s) == L.DG_ERR_DEVICE_CHECK
    assert lib.dg_ops_check(s) == L.DG_OK  # cleared
    hs = torch.randn(M, d, device="cuda").to(torch.bfloat16)
    assert fn(L.DG_BF16, p(hs), p(w), None, M, d, V, p(ent), p(am), s) == L.DG_OK
    assert lib.dg_ops_check(s) == L.DG_OK
    assert torch.isfinite(ent).all()

"""The allocation-free LM head (dg_lmhead_entropy_noalloc) against the regular
one (dg_lmhead_entropy), through the C ABI.

Callers that may not allocate device memory while they run this step (for
example while their stream is being recorded into a CUDA graph, or under a
framework that reserves all device memory itself) use the allocation-free
entry point; its results must be the regular entry point's. Two calls in a row
check that the shared, library-owned scratch array carries nothing over from
one call to the next. Collected last so that a failure here comes after every
other test has run."""
import ctypes as C
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from token_canvas_denoising_b200 import inputs as fx

pytestmark = pytest.mark.gpu

ENT_TOL = 1e-3  # nats, as in the oracle parity tests


def _dev(arr, dtype):
    from token_canvas_denoising_b200.canvas import to_device
    return to_device(arr, dtype, "cuda")


def _call(fn, dtype_code, hs, w, invT, M, d, V):
    ent = torch.empty(M, dtype=torch.float32, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    p = lambda t: C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)
    st = fn(dtype_code, p(hs), p(w), p(invT), M, d, V, p(ent), p(am),
            C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    return ent.cpu().numpy(), am.cpu().numpy()


@pytest.mark.parametrize("dtype,M,d,V", [("bf16", 256, 512, 32768), ("bf16", 300, 256, 8192),
                                         ("f32", 40, 64, 2048)])
def test_noalloc_matches_regular_entry_point_twice(dtype, M, d, V):
    from token_canvas_denoising_b200 import _lib
    lib = _lib.load()
    code = _lib.DG_BF16 if dtype == "bf16" else _lib.DG_F32
    invT = torch.from_numpy(np.exp(np.random.default_rng(M).uniform(-1.5, 1.5, M)).astype(np.float32)).cuda()
    for call in range(2):  # a second call on different data reuses the same scratch
        hs = _dev(fx.normal(61 + call, 1, (M, d), 1.0, dtype), dtype)
        w = _dev(fx.normal(61 + call, 2, (V, d), 1.0 / math.sqrt(d), dtype), dtype)
        e_ref, a_ref = _call(lib.dg_lmhead_entropy, code, hs, w, invT, M, d, V)
        e_na, a_na = _call(lib.dg_lmhead_entropy_noalloc, code, hs, w, invT, M, d, V)
        assert np.max(np.abs(e_na - e_ref)) <= ENT_TOL
        assert np.array_equal(a_na, a_ref)


def test_noalloc_rejects_problems_beyond_its_scratch():
    from token_canvas_denoising_b200 import _lib
    lib = _lib.load()
    cap = lib.dg_lmhead_entropy_noalloc_max_records()
    assert cap == 65536
    M, d, V = 65536 + 256, 64, 65536  # M rows with at least one partition each exceed the cap
    hs = torch.zeros(M, d, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(V, d, dtype=torch.bfloat16, device="cuda")
    ent = torch.empty(M, dtype=torch.float32, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    st = lib.dg_lmhead_entropy_noalloc(_lib.DG_BF16, C.c_void_p(hs.data_ptr()), C.c_void_p(w.data_ptr()),
                                       None, M, d, V, C.c_void_p(ent.data_ptr()), C.c_void_p(am.data_ptr()),
                                       C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.DG_ERR_UNSUPPORTED
    assert b"scratch" in lib.dg_last_error()

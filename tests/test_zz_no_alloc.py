"""The allocation-free LM head (dg_lmhead_entropy_noalloc) against the regular
one (dg_lmhead_entropy), through the C ABI.

Some callers of this library cannot allocate device memory where they run the
LM head: an application whose own allocator reserves the device's memory up
front, or a host that gives a plug-in only the buffers it passes. They call
the allocation-free entry point, which keeps its temporary results in a
fixed array inside the library. It runs the same kernels with the same vocab
partitions as the regular entry point, so its entropies and argmax must equal
the regular one's bit for bit. Two calls in a row on different data check that
the shared array carries nothing over from one call to the next, and the free
device memory and torch's allocator statistics must not change across them.
Collected last so that a failure here comes after every other test has run."""
import ctypes as C
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from token_canvas_denoising_b200 import inputs as fx

pytestmark = pytest.mark.gpu


def _dev(arr, dtype):
    from token_canvas_denoising_b200.canvas import to_device
    return to_device(arr, dtype, "cuda")


def _p(t):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def _call(fn, code, hs, w, invT, M, d, V, ent, am):
    st = fn(code, _p(hs), _p(w), _p(invT), M, d, V, _p(ent), _p(am),
            C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0


@pytest.mark.parametrize("dtype,M,d,V", [("bf16", 256, 512, 32768), ("bf16", 300, 256, 8192),
                                         ("f32", 40, 64, 2048)])
def test_noalloc_matches_regular_entry_point_twice(dtype, M, d, V):
    from token_canvas_denoising_b200 import _lib
    lib = _lib.load()
    code = _lib.DG_BF16 if dtype == "bf16" else _lib.DG_F32
    invT = torch.from_numpy(np.exp(np.random.default_rng(M).uniform(-1.5, 1.5, M)).astype(np.float32)).cuda()
    inputs, refs = [], []
    for call in range(2):  # the second call, on other data, reuses the same scratch
        hs = _dev(fx.normal(61 + call, 1, (M, d), 1.0, dtype), dtype)
        w = _dev(fx.normal(61 + call, 2, (V, d), 1.0 / math.sqrt(d), dtype), dtype)
        ent = torch.empty(M, dtype=torch.float32, device="cuda")
        am = torch.empty(M, dtype=torch.int32, device="cuda")
        _call(lib.dg_lmhead_entropy, code, hs, w, invT, M, d, V, ent, am)
        inputs.append((hs, w))
        refs.append((ent, am))
    outs = [(torch.full((M,), float("nan"), device="cuda"), torch.full((M,), -1, dtype=torch.int32, device="cuda"))
            for _ in range(3)]
    torch.cuda.synchronize()
    # the first call on this device and context looks up the array's address
    _call(lib.dg_lmhead_entropy_noalloc, code, *inputs[0], invT, M, d, V, *outs[0])
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    stats0 = torch.cuda.memory_stats()
    _call(lib.dg_lmhead_entropy_noalloc, code, *inputs[1], invT, M, d, V, *outs[1])
    _call(lib.dg_lmhead_entropy_noalloc, code, *inputs[0], invT, M, d, V, *outs[2])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    stats1 = torch.cuda.memory_stats()
    for k in ("allocation.all.current", "allocated_bytes.all.current", "reserved_bytes.all.current",
              "num_alloc_retries"):
        assert stats1.get(k, 0) == stats0.get(k, 0), k
    assert lib.dg_ops_check(C.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    for (ent, am), (e_ref, a_ref) in zip(outs, [refs[0], refs[1], refs[0]]):
        assert torch.equal(ent, e_ref)
        assert torch.equal(am, a_ref)


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

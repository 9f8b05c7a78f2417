"""CPU checks of the C ABI: the library loads and exports every function that
include/*.h declares; host-side argument validation rejects bad input before
any device work (no GPU needed for these calls)."""
import ctypes as C
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(dg_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from token_canvas_denoising_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from token_canvas_denoising_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("dg_canvas_init", "dg_denoise_step", "dg_decode_block", "dg_canvas_get_state",
              "dg_canvas_set_state", "dg_canvas_destroy", "dg_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from token_canvas_denoising_b200 import _lib
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no Python signature"


def test_status_strings_and_version(lib):
    from token_canvas_denoising_b200 import _lib
    assert lib.dg_abi_version() == 2
    for s in range(7):
        assert lib.dg_status_string(s)
    assert lib.dg_status_string(_lib.DG_ERR_OOM) == b"out of device memory"


def _model(**kw):
    from token_canvas_denoising_b200 import _lib
    m = _lib.dg_model_desc()
    m.d_model, m.n_q_heads, m.n_kv_heads, m.head_dim, m.vocab, m.dtype = 64, 2, 1, 32, 512, _lib.DG_F32
    for k in ("embed", "wq", "wk", "wv", "wo", "lm_head"):
        setattr(m, k, 4096)  # never dereferenced: validation fails first or no GPU
    for k, v in kw.items():
        setattr(m, k, v)
    return m


@pytest.mark.parametrize("over,status", [
    (dict(dtype=7), 1),
    (dict(n_q_heads=3, n_kv_heads=2), 1),
    (dict(lm_head=None), 1),
    (dict(embed=4097), 1),          # misaligned
    (dict(head_dim=48), 2),         # f32 head_dim must be a multiple of 32
    (dict(dtype=1, head_dim=64), 2),  # bf16 needs head_dim 128
    (dict(dtype=1, head_dim=128, vocab=1000), 2),
])
def test_init_rejects_bad_models(lib, over, status):
    m = _model(**over)
    ctx = C.c_void_p()
    plen = (C.c_int32 * 1)(0)
    seeds = (C.c_uint64 * 1)(0)
    st = lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None,
                            None, C.cast(seeds, C.c_void_p), None)
    assert st == status, lib.dg_last_error()
    assert not ctx.value


_BF16 = dict(dtype=1, head_dim=128, vocab=1024, d_model=128)
_MOE = dict(n_experts=32, top_k=4, moe_inter=128, n_shared=1, w_router=4096, w_gate=4096, w_up=4096,
            w_down=4096)


@pytest.mark.parametrize("over,status", [
    (dict(_MOE), 2),                                   # MoE needs the bf16 storage dtype
    (dict(_BF16, **dict(_MOE, n_experts=48)), 2),      # a multiple of 32 experts
    (dict(_BF16, **dict(_MOE, top_k=9, n_experts=64)), 2),
    (dict(_BF16, **dict(_MOE, top_k=33)), 1),          # top_k > n_experts
    (dict(_BF16, **dict(_MOE, moe_inter=100)), 2),
    (dict(_BF16, **dict(_MOE, n_shared=3)), 2),
    (dict(_BF16, **dict(_MOE, w_up=None)), 1),
])
def test_init_rejects_bad_moe_models(lib, over, status):
    m = _model(**over)
    ctx = C.c_void_p()
    plen = (C.c_int32 * 1)(0)
    seeds = (C.c_uint64 * 1)(0)
    st = lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None,
                            None, C.cast(seeds, C.c_void_p), None)
    assert st == status, lib.dg_last_error()
    assert not ctx.value


def test_init_rejects_moe_beyond_one_routing_block(lib):
    m = _model(**dict(_BF16, **_MOE))
    ctx = C.c_void_p()
    plen = (C.c_int32 * 2)(0, 0)
    seeds = (C.c_uint64 * 2)(0, 1)
    st = lib.dg_canvas_init(C.byref(ctx), C.byref(m), 2, 200, C.cast(plen, C.c_void_p), None, None,
                            None, C.cast(seeds, C.c_void_p), None)
    assert st == 2 and b"256" in lib.dg_last_error()
    assert not ctx.value


@pytest.mark.parametrize("batch,canvas", [(0, 16), (1, 0), (1, 1025)])
def test_init_rejects_bad_sizes(lib, batch, canvas):
    m = _model()
    ctx = C.c_void_p()
    plen = (C.c_int32 * 1)(0)
    seeds = (C.c_uint64 * 1)(0)
    st = lib.dg_canvas_init(C.byref(ctx), C.byref(m), batch, canvas, C.cast(plen, C.c_void_p), None,
                            None, None, C.cast(seeds, C.c_void_p), None)
    assert st == 1


def test_null_context_calls_fail_cleanly(lib):
    from token_canvas_denoising_b200 import _lib
    s = _lib.dg_schedule(48, 0.05, 1, 0)
    assert lib.dg_denoise_step(None, C.byref(s), None) == 1
    assert lib.dg_decode_block(None, C.byref(s), None, None) == 1
    assert lib.dg_canvas_sync(None) == 1
    mask = (C.c_uint8 * 4)()
    toks = (C.c_int32 * 4)()
    assert lib.dg_canvas_reset_fixed(None, None, C.cast(mask, C.c_void_p), C.cast(toks, C.c_void_p)) == 1
    assert lib.dg_canvas_block_kv(None, None, None) == 1
    assert lib.dg_canvas_set_prefix(None, None, None, None) == 1
    lib.dg_canvas_destroy(None)


def test_product_binding_has_no_fallback(monkeypatch, tmp_path):
    """The binding raises when the library is missing instead of computing on the CPU."""
    from token_canvas_denoising_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        _lib.load()


@pytest.mark.parametrize("field,value", [("n_layers", -1), ("n_layers", 65), ("lm_head_format", 7),
                                         ("expert_format", 3)])
def test_init_rejects_bad_model_fields(lib, field, value):
    m = _model()
    setattr(m, field, value)
    ctx = C.c_void_p()
    plen = (C.c_int32 * 1)(0)
    seeds = (C.c_uint64 * 1)(0)
    st = lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None, None,
                            C.cast(seeds, C.c_void_p), None)
    assert st == 1 and not ctx.value


def test_init_rejects_e4m3_without_scales_or_with_f32(lib):
    from token_canvas_denoising_b200 import _lib
    ctx = C.c_void_p()
    plen = (C.c_int32 * 1)(0)
    seeds = (C.c_uint64 * 1)(0)
    m = _model(**_BF16)
    m.lm_head_format = _lib.DG_LM_E4M3  # no lm_head_scale
    assert lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None, None,
                              C.cast(seeds, C.c_void_p), None) == 1
    m.lm_head_scale = 4096
    m.d_model = 192  # not a multiple of 128
    assert lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None, None,
                              C.cast(seeds, C.c_void_p), None) == 2
    m = _model()  # f32 storage
    m.lm_head_format, m.lm_head_scale = _lib.DG_LM_E4M3, 4096
    assert lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None, None,
                              C.cast(seeds, C.c_void_p), None) == 2
    m = _model(**dict(_BF16, **_MOE))
    m.expert_format = _lib.DG_LM_E4M3  # no expert scales
    assert lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None, None,
                              C.cast(seeds, C.c_void_p), None) == 1
    assert not ctx.value


def test_init_rejects_moe_with_a_layer_stack(lib):
    m = _model(**dict(_BF16, **_MOE))
    m.n_layers = 2
    ctx = C.c_void_p()
    plen = (C.c_int32 * 1)(0)
    seeds = (C.c_uint64 * 1)(0)
    st = lib.dg_canvas_init(C.byref(ctx), C.byref(m), 1, 16, C.cast(plen, C.c_void_p), None, None, None,
                            C.cast(seeds, C.c_void_p), None)
    assert st == 2 and b"single-layer" in lib.dg_last_error()


def test_op_entry_points_reject_bad_arguments(lib):
    assert lib.dg_lmhead_entropy_e4m3(None, None, None, None, 4, 128, 256, None, None, None) == 1
    buf = C.c_void_p(4096)
    assert lib.dg_lmhead_entropy_e4m3(buf, buf, buf, None, 4, 96, 256, buf, buf, None) == 2  # d % 128
    assert lib.dg_quantize_rows_e4m3(None, None, None, 4, 128, None) == 1
    assert lib.dg_quantize_rows_e4m3(buf, buf, buf, 4, 12, None) == 2  # d % 8

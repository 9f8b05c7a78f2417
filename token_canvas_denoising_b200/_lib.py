"""ctypes declarations of libdgcanvas.so (mirrors include/dg_canvas.h).

Argument marshalling only: every step of the denoise path runs in the CUDA
library. Loading fails loudly if the library is missing; there is no fallback.
"""
import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdgcanvas.so")

DG_OK, DG_ERR_INVALID_ARG, DG_ERR_UNSUPPORTED, DG_ERR_OOM, DG_ERR_CUDA, DG_ERR_TIMEOUT, \
    DG_ERR_DEVICE_CHECK = range(7)
DG_F32, DG_BF16 = 0, 1
DG_LM_STORAGE, DG_LM_E4M3 = 0, 1
DG_SCHED_CEIL = 0
DG_KERNEL_LMHEAD, DG_KERNEL_ATTENTION, DG_KERNEL_DECODE = 0, 1, 2


class dg_model_desc(C.Structure):
    _fields_ = [("d_model", C.c_int32), ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("vocab", C.c_int32), ("dtype", C.c_int32),
                ("embed", C.c_void_p), ("wq", C.c_void_p), ("wk", C.c_void_p), ("wv", C.c_void_p),
                ("wo", C.c_void_p), ("lm_head", C.c_void_p),
                ("n_experts", C.c_int32), ("top_k", C.c_int32), ("moe_inter", C.c_int32),
                ("n_shared", C.c_int32),
                ("w_router", C.c_void_p), ("w_gate", C.c_void_p), ("w_up", C.c_void_p),
                ("w_down", C.c_void_p),
                ("lm_head_format", C.c_int32), ("lm_head_scale", C.c_void_p), ("n_layers", C.c_int32),
                ("expert_format", C.c_int32), ("w_gate_scale", C.c_void_p), ("w_up_scale", C.c_void_p),
                ("w_down_scale", C.c_void_p)]


class dg_schedule(C.Structure):
    _fields_ = [("max_steps", C.c_int32), ("stop_entropy", C.c_float),
                ("adaptive_stop", C.c_int32), ("kind", C.c_int32)]


class dg_step_out(C.Structure):
    _fields_ = [("ent", C.c_void_p), ("argmax", C.c_void_p), ("freeze_mask", C.c_void_p),
                ("attn_out", C.c_void_p), ("hidden", C.c_void_p), ("hidden_attn", C.c_void_p),
                ("q", C.c_void_p), ("k_canvas", C.c_void_p), ("v_canvas", C.c_void_p), ("layer_out", C.c_void_p)]


class dg_state(C.Structure):
    _fields_ = [("tokens", C.c_void_p), ("frozen", C.c_void_p), ("step", C.c_void_p),
                ("seed", C.c_void_p), ("done", C.c_void_p)]


# name -> (restype, argtypes); every symbol declared in include/*.h
SIGNATURES = {
    "dg_canvas_init": (C.c_int, [C.POINTER(C.c_void_p), C.POINTER(dg_model_desc), C.c_int32, C.c_int32,
                                 C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                 C.c_void_p]),
    "dg_denoise_step": (C.c_int, [C.c_void_p, C.POINTER(dg_schedule), C.POINTER(dg_step_out)]),
    "dg_decode_block": (C.c_int, [C.c_void_p, C.POINTER(dg_schedule), C.c_void_p, C.c_void_p]),
    "dg_canvas_get_state": (C.c_int, [C.c_void_p, C.POINTER(dg_state)]),
    "dg_canvas_set_state": (C.c_int, [C.c_void_p, C.POINTER(dg_state)]),
    "dg_canvas_sync": (C.c_int, [C.c_void_p]),
    "dg_canvas_loop_steps": (C.c_int, [C.c_void_p, C.c_void_p]),
    "dg_canvas_reset": (C.c_int, [C.c_void_p, C.c_void_p]),
    "dg_canvas_reset_fixed": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_canvas_block_kv": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_selftest_wait_timeout": (C.c_int, [C.c_void_p]),
    "dg_canvas_set_prefix": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_canvas_set_timing_events": (C.c_int, [C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p]),
    "dg_canvas_set_kernel_timing": (C.c_int, [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p]),
    "dg_canvas_destroy": (None, [C.c_void_p]),
    "dg_status_string": (C.c_char_p, [C.c_int]),
    "dg_last_error": (C.c_char_p, []),
    "dg_abi_version": (C.c_int32, []),
    "dg_launches_per_step": (C.c_int32, [C.c_void_p]),
    # include/dg_ops.h
    "dg_lmhead_entropy": (C.c_int, [C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_int32,
                                    C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_lmhead_entropy_e4m3": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_int32,
                                         C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_quantize_rows_e4m3": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_void_p]),
    "dg_lmhead_entropy_noalloc": (C.c_int, [C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32,
                                            C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]),
    "dg_lmhead_entropy_noalloc_max_records": (C.c_size_t, []),
    "dg_attention": (C.c_int, [C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_int32,
                               C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                               C.c_void_p, C.c_void_p]),
    "dg_linear": (C.c_int, [C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32,
                            C.c_int32, C.c_int32, C.c_void_p]),
    "dg_ops_check": (C.c_int, [C.c_void_p]),
}

_lib = None


def load():
    """Load libdgcanvas.so (once) and declare its signatures. Raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libdgcanvas.so not built ({LIB_PATH}); run "
                           "`python -m token_canvas_denoising_b200.build`")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class DgError(RuntimeError):
    def __init__(self, status, where):
        lib = load()
        self.status = status
        msg = lib.dg_status_string(status).decode()
        detail = lib.dg_last_error().decode()
        super().__init__(f"{where}: {msg} ({detail})")


def check(status, where):
    if status != DG_OK:
        raise DgError(status, where)

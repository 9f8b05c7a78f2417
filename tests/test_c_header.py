"""The public headers are plain C: a C99 program that includes both compiles
with warnings as errors and links against libdgcanvas.so, and the struct
layouts it reports (sizes and field offsets) equal the Python binding's ctypes
structures, so the two sides of the boundary agree byte for byte. CPU only:
the program is built and run without touching a GPU."""
import ctypes as C
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STRUCTS = {
    "dg_model_desc": ["d_model", "vocab", "dtype", "embed", "lm_head", "n_experts", "n_shared", "w_router",
                      "w_down", "lm_head_format", "lm_head_scale", "n_layers", "expert_format",
                      "w_down_scale"],
    "dg_schedule": ["max_steps", "stop_entropy", "adaptive_stop", "kind"],
    "dg_step_out": ["ent", "argmax", "freeze_mask", "attn_out", "hidden", "hidden_attn", "q", "k_canvas",
                    "v_canvas", "layer_out"],
    "dg_state": ["tokens", "frozen", "step", "seed", "done"],
}


def _program():
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "dg_canvas.h"', '#include "dg_ops.h"',
             "typedef void (*fn)(void);",
             "int main(void) {",
             "  /* reference the entry points so that the link resolves them */",
             "  fn volatile f[] = {(fn)dg_canvas_init, (fn)dg_denoise_step, (fn)dg_decode_block,",
             "                     (fn)dg_canvas_reset_fixed, (fn)dg_canvas_block_kv, (fn)dg_canvas_set_prefix,",
             "                     (fn)dg_lmhead_entropy, (fn)dg_lmhead_entropy_e4m3,",
             "                     (fn)dg_quantize_rows_e4m3, (fn)dg_lmhead_entropy_noalloc, (fn)dg_attention,",
             "                     (fn)dg_linear, (fn)dg_ops_check, (fn)dg_selftest_wait_timeout,",
             "                     (fn)dg_canvas_loop_steps};",
             "  (void)f;"]
    for s, fields in STRUCTS.items():
        lines.append(f'  printf("{s} size %zu\\n", sizeof({s}));')
        for fd in fields:
            lines.append(f'  printf("{s}.{fd} %zu\\n", offsetof({s}, {fd}));')
    lines += ["  return 0;", "}"]
    return "\n".join(lines) + "\n"


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_headers_are_c99_and_layouts_match_the_binding(tmp_path):
    from token_canvas_denoising_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from token_canvas_denoising_b200 import build
        build.build()
    src = tmp_path / "abi.c"
    src.write_text(_program())
    exe = tmp_path / "abi"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-ldgcanvas", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = dict(line.rsplit(" ", 1) for line in out if line)
    for s, fields in STRUCTS.items():
        cls = getattr(_lib, s)
        assert int(got[f"{s} size"]) == C.sizeof(cls), s
        for fd in fields:
            assert int(got[f"{s}.{fd}"]) == getattr(cls, fd).offset, f"{s}.{fd}"

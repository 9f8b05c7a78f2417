"""Run the denoise step on a named synthetic workload, for profilers.

    python -m token_canvas_denoising_b200.profile_ops [--workload canvas256] [--steps 6]
        [--op step|lmhead|lmhead_e4m3|attention|linear]

'step' runs CUDA-graph denoise steps through the C ABI (every kernel of the
path); the other ops run the single-operation entry points on the workload's
shapes. Prints the mean device time per iteration (CUDA events) so the plain
run can be compared with a profiled one. Inputs are the seeded synthetic ones.
"""
import argparse
import math

import numpy as np
import torch

from . import inputs as fx
from . import ops
from .canvas import from_workload, schedule, to_device


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="canvas256")
    ap.add_argument("--steps", type=int, default=6)
    ap.add_argument("--op", default="step", choices=["step", "lmhead", "lmhead_e4m3", "attention", "linear"])
    a = ap.parse_args()
    cfg = fx.CONFIGS[a.workload]
    torch.cuda.set_device(0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.op == "step":
        wl = fx.make_workload(cfg)
        cv, _keep = from_workload(wl)
        s = schedule(cfg.max_steps, cfg.stop_entropy, adaptive_stop=False)
        cv.step(s)
        torch.cuda.synchronize()
        e0.record()
        for i in range(a.steps):
            if i and i % cfg.max_steps == 0:
                cv.reset()
            cv.step(s)
        e1.record()
        cv.sync()
        cv.close()
    else:
        M, d, V = cfg.B * cfg.C, cfg.d, cfg.V
        if a.op == "lmhead":
            hs = to_device(fx.normal(7, 1, (M, d), 1.0, "bf16"), "bf16", "cuda")
            w = to_device(fx.normal(7, 2, (V, d), 1.0 / math.sqrt(d), "bf16"), "bf16", "cuda")
            run = lambda: ops.lmhead_entropy(hs, w)
        elif a.op == "lmhead_e4m3":
            hs = to_device(fx.normal(7, 1, (M, d), 1.0, "bf16"), "bf16", "cuda")
            codes, scales = fx.e4m3_rows(fx.normal(7, 2, (V, d), 1.0 / math.sqrt(d), "f32"))
            w, sw = torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()
            run = lambda: ops.lmhead_entropy_e4m3(hs, w, sw)
        elif a.op == "linear":
            N = (cfg.Hq + 2 * cfg.Hk) * cfg.h
            x = to_device(fx.normal(7, 1, (M, d), 1.0, "bf16"), "bf16", "cuda")
            w = to_device(fx.normal(7, 2, (N, d), 1.0 / math.sqrt(d), "bf16"), "bf16", "cuda")
            run = lambda: ops.linear(x, w)
        else:
            h = cfg.h
            q = to_device(fx.normal(7, 1, (M, cfg.Hq * h), 1.0, "bf16"), "bf16", "cuda")
            kc = to_device(fx.normal(7, 2, (M, cfg.Hk * h), 1.0, "bf16"), "bf16", "cuda")
            vc = to_device(fx.normal(7, 3, (M, cfg.Hk * h), 1.0, "bf16"), "bf16", "cuda")
            pk = [to_device(fx.normal(7, 10 + b, (cfg.S[b], cfg.Hk, h), 1.0, "bf16"), "bf16", "cuda")
                  for b in range(cfg.B)]
            pv = [to_device(fx.normal(7, 30 + b, (cfg.S[b], cfg.Hk, h), 1.0, "bf16"), "bf16", "cuda")
                  for b in range(cfg.B)]
            run = lambda: ops.attention(q, kc, vc, pk, pv, cfg.B, cfg.C, cfg.Hq, cfg.Hk, h)
        run()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(a.steps):
            run()
        e1.record()
    torch.cuda.synchronize()
    print(f"{a.op} on {a.workload}: {e0.elapsed_time(e1) / a.steps * 1e3:.1f} us per iteration "
          f"({a.steps} iterations)")


if __name__ == "__main__":
    main()

"""Throughput of the canvas denoise step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload canvas256]

A bench step is one denoise step: every row of the hot path (embed, Q/K/V
projection, bidirectional attention over prefix + canvas, Wo + residual, LM
head with fused entropy/argmax, freeze selection, re-noise, stop test) over the
whole batch of canvases, run as one CUDA-graph launch through the C ABI. Every
48 steps (the step cap) the canvases are redrawn on the device (a new block),
so each timed step does real freezing work. Inputs are synthetic and seeded;
the weights and prefix K/V are resident in HBM before the timed region.

Multi-GPU: the canvases are independent requests, so N ranks run N replicas
with no data-path collective (weak scaling); the reported time is the max over
ranks and the value counts the steps of every rank.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

BLOCK_STEPS = 48
REF_BUDGET_S = 150.0  # target wall time of the whole reference-arm run


# ---------------------------------------------------------------- ranks
def max_over_ranks(value, world, device):
    """The largest value over the ranks (a device time: the job is as slow as
    its slowest rank). One all-reduce on `device` ('cuda' under NCCL, 'cpu'
    under gloo); every rank calls it at the same point."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, elapsed_ms):
    """Whole-job throughput: the units every rank processed / the slowest
    rank's elapsed time."""
    return world * units_per_rank / (elapsed_ms / 1e3)


def rank_canvas_seeds(seeds, rank):
    """Each rank decodes its own requests: canvas seeds offset per rank."""
    return tuple(int(s) + 1000 * rank for s in seeds)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4800)
    ap.add_argument("--warmup", type=int, default=96)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="canvas256")
    ap.add_argument("--e2e-blocks", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    return ap.parse_args()


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu = str(gpu_id)  # nvidia-smi id: "GPU-<uuid>" or an index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workload
def workload_cfg(name):
    from token_canvas_denoising_b200 import inputs as fx
    return fx.CONFIGS[name]


def flops_bytes(cfg):
    """Algorithmic flops and HBM bytes of one step and of the LM-head kernel."""
    M, d, V = cfg.B * cfg.C, cfg.d, cfg.V
    qd, kd = cfg.Hq * cfg.h, cfg.Hk * cfg.h
    es = 2 if cfg.dtype == "bf16" else 4
    S = sum(cfg.S)
    f_qkv = 2 * M * d * (qd + 2 * kd)
    f_attn = sum(4 * cfg.C * (s + cfg.C) * cfg.h * cfg.Hq for s in cfg.S)
    f_wo = 2 * M * qd * d
    f_lm = 2 * M * d * V
    b_lm = V * d * es + M * d * es + M * 32  # W once, Hs once, one 32-byte record per row... per CTA
    b_step = ((qd + 2 * kd) * d + d * qd + V * d) * es + 2 * S * kd * es + M * d * es * 6
    return {"flops_step": f_qkv + f_attn + f_wo + f_lm, "bytes_step": b_step, "flops_lm": f_lm,
            "bytes_lm_weights": V * d * es}


def cpu_cores_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def run_oracle_sample(cfg, seconds, wl=None):
    """Time the fp64 oracle's denoise steps on this host for about `seconds`.
    Returns (steps/s, steps run, sample description)."""
    from oracle import model as om
    from token_canvas_denoising_b200 import inputs as fx
    wl = wl or fx.make_workload(cfg)
    m = {"dtype": cfg.dtype, "d": cfg.d, "Hq": cfg.Hq, "Hk": cfg.Hk, "h": cfg.h, "V": cfg.V}
    m.update({k: wl.weights[k] for k in ("embed", "wq", "wk", "wv", "wo", "lm_head")})
    prefix = list(zip(wl.prefix_k, wl.prefix_v))
    sched = {"max_steps": cfg.max_steps, "stop_entropy": cfg.stop_entropy, "adaptive_stop": False}
    invT = None if cfg.inv_temp == "one" else wl.inv_temp
    st = om.init_state(wl.seeds, cfg.C, cfg.V)
    n = 0
    t0 = time.perf_counter()
    while True:
        st, _ = om.denoise_step(m, prefix, st, sched, invT)
        n += 1
        if time.perf_counter() - t0 >= seconds or bool(st["done"].all()):
            break
    dt = time.perf_counter() - t0
    return n / dt, n, f"{n} full oracle denoise steps of the {cfg.name} workload (fp64, numpy)"


# ---------------------------------------------------------------- reference arm
def bench_reference(args, rank, world):
    """The fp64 oracle on this host's cores, on the same workload and unit.

    Each reference step is a bounded sample of one denoise step: the oracle's
    full step (embed, Q/K/V, attention over the whole prefix, Wo + residual, LM
    head over the whole vocabulary, entropy/argmax, freeze, re-noise) on the
    first r canvas positions only, r chosen so that warm-up + timed steps fit
    in about REF_BUDGET_S seconds. A cost model t(r) = a + b r is calibrated
    first from one step on 1 row and one step on the whole canvas; the
    workload's step time is the measured sample step time plus (C - r) rows at
    the per-row cost b. Weights and prefix K/V are widened to fp64 once, before
    the timed region."""
    if rank != 0:
        return 0
    from oracle import model as om
    from token_canvas_denoising_b200 import inputs as fx
    cfg = workload_cfg(args.workload)
    wl = fx.make_workload(cfg)
    m = {"dtype": cfg.dtype, "d": cfg.d, "Hq": cfg.Hq, "Hk": cfg.Hk, "h": cfg.h, "V": cfg.V}
    m.update({k: wl.weights[k] for k in ("embed", "wq", "wk", "wv", "wo", "lm_head")})
    m = om.prewiden(m)
    prefix = [(om.widen(k, cfg.dtype), om.widen(v, cfg.dtype)) for k, v in zip(wl.prefix_k, wl.prefix_v)]
    sched = {"max_steps": cfg.max_steps, "stop_entropy": cfg.stop_entropy, "adaptive_stop": False}

    def run(rows, n):
        invT = None if cfg.inv_temp == "one" else wl.inv_temp[:rows]
        st = om.init_state(wl.seeds, rows, cfg.V)
        t0 = time.perf_counter()
        for _ in range(n):
            st, _ = om.denoise_step(m, prefix, st, sched, invT)
            if st["done"].all():
                st = om.init_state(wl.seeds, rows, cfg.V)
        return time.perf_counter() - t0

    # per-step cost t(r) = a + b r (a: work independent of the sampled rows,
    # such as streaming the weights; b: per row), from one step on 1 row and
    # one step on the whole canvas, so the model is exact at both ends
    tc0 = time.perf_counter()
    t1 = run(1, 2) / 2
    tC = run(cfg.C, 1) if cfg.C > 1 else t1
    b = max(0.0, (tC - t1) / max(1, cfg.C - 1))
    a = max(1e-4, t1 - b)
    budget = max(10.0, REF_BUDGET_S - (time.perf_counter() - tc0))
    per_step = budget / max(1, args.steps + args.warmup)
    rows = int(max(1, min(cfg.C, (per_step - a) / b if b > 0 else cfg.C)))
    run(rows, args.warmup)
    dt = run(rows, args.steps)
    # a full step costs the measured sample step plus the remaining rows at the
    # measured per-row cost
    t_full = dt / args.steps + b * (cfg.C - rows)
    v = 1.0 / t_full
    sample = (f"{args.steps} oracle denoise steps (fp64 numpy) on the first {rows} of {cfg.C} canvas positions "
              f"of the {cfg.name} workload (full prefix, full vocabulary); full-step time = measured sample "
              f"step time + {cfg.C - rows} rows x the measured per-row cost ({b * 1e3:.3f} ms)")
    line = {"impl": "reference", "metric": "denoise steps/s", "value": v, "unit": "steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "canvas_tokens_per_s": v * cfg.B * cfg.C,
            "config": {"workload": f"{cfg.name}: B{cfg.B} C{cfg.C} S{cfg.S[0]} d{cfg.d} Hq{cfg.Hq}/Hk{cfg.Hk} "
                                   f"h{cfg.h} V{cfg.V} {cfg.dtype}, {cfg.max_steps}-step blocks, adaptive stop off"},
            "cpu_baseline": {"value": v, "unit": "steps/s", "cores": cpu_cores_used(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- b200 arm
def bench_b200(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from token_canvas_denoising_b200 import inputs as fx
    from token_canvas_denoising_b200.canvas import from_workload, schedule

    cfg = workload_cfg(args.workload)
    # each rank decodes its own requests: distinct canvas seeds per rank
    cfg_r = fx.derive(cfg, canvas_seeds=rank_canvas_seeds(cfg.canvas_seeds, rank))
    wl = fx.make_workload(cfg_r)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        cv, keep = from_workload(wl, stream=stream)
    sched = schedule(cfg.max_steps, cfg.stop_entropy, adaptive_stop=False)
    fb = flops_bytes(cfg)
    peaks = load_peaks()

    def run_steps(n, start):
        for i in range(start, start + n):
            if i % BLOCK_STEPS == 0 and i > 0:
                cv.reset()
            cv.step(sched)

    # warm-up (captures the step graph)
    run_steps(args.warmup, 0)
    cv.sync()
    launches_per_step = cv.launches_per_step

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        gpu_id = str(local_rank)
    clocks = ClockSampler(gpu_id)

    # ---- timed region 1: K denoise steps (one CUDA-graph launch each)
    cv.reset()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    run_steps(args.steps, 0)
    t_stop.record(stream)
    torch.cuda.synchronize()
    elapsed_ms = t_start.elapsed_time(t_stop)
    ck = clocks.stop()
    cv.sync()
    n_resets = (args.steps - 1) // BLOCK_STEPS
    if world > 1:
        elapsed_ms = max_over_ranks(elapsed_ms, world, "cuda")
        dist.barrier()

    # ---- timed region 2: the same steps with CUDA events recorded around the
    # LM-head kernel on its stream (a ring of NEV event pairs, one graph
    # variant each); gives the dominant kernel's average launch duration
    NEV = 4
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(NEV)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(NEV)]
    for e in ev_s + ev_e:  # torch creates the CUDA event on its first record
        e.record(stream)
    cv.set_timing_events(ev_s, ev_e)
    cv.reset()
    run_steps(NEV, 0)  # capture every variant before timing
    cv.sync()
    cv.reset()
    lm_steps = min(args.steps, 960)
    lm_ms = []
    for i in range(lm_steps):
        if i % BLOCK_STEPS == 0 and i > 0:
            cv.reset()
        cv.step(sched)
        j = i - (NEV - 1)
        if j >= 0:  # the pair used NEV-1 steps ago: wait for it (NEV-1 steps stay queued)
            ev_e[j % NEV].synchronize()
            lm_ms.append(ev_s[j % NEV].elapsed_time(ev_e[j % NEV]))
    torch.cuda.synchronize()
    for j in range(max(0, lm_steps - (NEV - 1)), lm_steps):
        lm_ms.append(ev_s[j % NEV].elapsed_time(ev_e[j % NEV]))
    cv.set_timing_events([], [])
    steps_per_s = job_rate(args.steps, world, elapsed_ms)
    lm_avg_ms = float(np.mean(lm_ms))
    lm_tflops = fb["flops_lm"] / (lm_avg_ms / 1e3) / 1e12

    # ---- end to end through the C ABI with host buffers: per block, the initial
    # state goes host->device (pinned) and the tokens come back device->host
    e2e = None
    if rank == 0 or world > 1:
        cv.reset()  # a fresh block: step 0, nothing frozen
        st0 = cv.get_state()
        pin = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in st0.items()}
        pin_np = {k: v.numpy() for k, v in pin.items()}
        tok_out = torch.empty(cfg.B * cfg.C, dtype=torch.int32).pin_memory()
        cv.set_state(pin_np)
        cv.decode(sched, tok_out)  # warm
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        total_steps = 0
        e0.record(stream)
        for _ in range(args.e2e_blocks):
            cv.set_state(pin_np)
            _, steps = cv.decode(sched, tok_out)
            total_steps += max(steps)
            assert max(steps) == cfg.max_steps, steps
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        h2d = sum(v.nbytes for v in pin_np.values())
        d2h = tok_out.numel() * 4 + cfg.B * 4
        e2e = {"value": job_rate(total_steps, world, e2e_ms), "unit": "steps/s",
               "h2d_bytes_per_step": int(round(h2d / BLOCK_STEPS)),
               "d2h_bytes_per_step": int(round(d2h / BLOCK_STEPS)),
               "note": f"{args.e2e_blocks} decode blocks of {BLOCK_STEPS} steps via dg_canvas_set_state "
                       "(pinned host -> device) + dg_decode_block (tokens to pinned host)"}
        if world > 1:
            e2e["value"] = job_rate(total_steps, world, max_over_ranks(e2e_ms, world, "cuda"))

    cpu = None
    if rank == 0 and world == 1:
        v, n, sample = run_oracle_sample(cfg, args.cpu_seconds, wl)
        cpu = {"value": v, "unit": "steps/s", "cores": cpu_cores_used(), "kind": "oracle", "sample": sample}

    if rank == 0:
        traffic = None
        tpath = os.path.join(ROOT, "profiles", f"lmhead_traffic_{cfg.name}.json")
        if os.path.exists(tpath):
            try:
                with open(tpath) as f:
                    traffic = json.load(f).get("bytes_per_launch")
            except Exception:
                traffic = None
        peak = peaks["bf16_tflops_sustained"]
        line = {
            "metric": "denoise steps/s", "value": steps_per_s, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic",
            "canvas_tokens_per_s": steps_per_s * cfg.B * cfg.C,
            "config": {"workload": f"{cfg.name}: B{cfg.B} C{cfg.C} S{cfg.S[0]} d{cfg.d} Hq{cfg.Hq}/Hk{cfg.Hk} "
                                   f"h{cfg.h} V{cfg.V} {cfg.dtype}, {cfg.max_steps}-step blocks, adaptive stop off",
                       "batch_canvases": cfg.B, "canvas_len": cfg.C, "prefix_len": cfg.S[0],
                       "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2: each step streams {fb['bytes_step'] / 1e6:.0f} MB of weights "
                             "and prefix K/V (> 126 MB L2)"},
            "clocks": ck,
            "e2e": e2e,
            "gpu_launches": int(args.steps * launches_per_step + n_resets),
            "roofline": {"bound": "tensor", "kernel": "lmhead_tc_kernel (LM head + entropy/argmax)",
                         "achieved": lm_tflops, "peak": peak, "unit": "TFLOP/s", "frac": lm_tflops / peak,
                         "traffic": traffic,
                         "peak_source": f"{peaks['source']} sustained bf16 (kernel timed inside a long step loop)",
                         "avg_ms": lm_avg_ms,
                         "algorithmic_flops_per_launch": fb["flops_lm"],
                         "hbm_bound_ms": fb["bytes_lm_weights"] / (peaks["hbm_gbs"] * 1e9) * 1e3},
            "step_roofline": {"flops": fb["flops_step"], "bytes": fb["bytes_step"],
                              "ms": max(fb["flops_step"] / (peaks["bf16_tflops"] * 1e12),
                                        fb["bytes_step"] / (peaks["hbm_gbs"] * 1e9)) * 1e3},
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    cv.close()
    return 0


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return bench_reference(args, rank, world)
    import torch
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=None)
    try:
        return bench_b200(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

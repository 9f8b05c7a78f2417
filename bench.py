"""Throughput of the canvas denoise step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload longctx]

A bench step is one denoise step: every row of the hot path (embed, Q/K/V
projection, bidirectional attention over prefix + canvas, Wo + residual, LM
head with fused entropy/argmax, freeze selection, re-noise, stop test) over the
whole batch of canvases, run as one CUDA-graph launch through the C ABI. Every
48 steps (the step cap) the canvases are redrawn on the device (a new block),
so each timed step does real freezing work. Inputs are synthetic and seeded;
the weights and prefix K/V are resident in HBM before the timed region.

The default workload is the largest that fits one GPU: longctx, four canvases
of 256 positions, each over its own 32,768-token prompt K/V, vocabulary
262,144 (1.82 TFLOP and 2.1 GB of weights and K/V per step).

Multi-GPU: the canvases are independent requests, so N ranks run N replicas
with no data-path collective (weak scaling); the reported time is the max over
ranks and the value counts the steps of every rank.
"""
import argparse
import hashlib
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
# per workload: (timed steps, warm-up steps, e2e decode blocks) when not given
DEFAULTS = {"tiny": (4800, 96, 20), "canvas256": (4800, 96, 20), "vocab262k": (480, 48, 4),
            "longctx": (240, 24, 2), "moe": (480, 48, 4), "vocab262k_fp8": (480, 48, 4),
            "longctx_fp8": (480, 48, 2), "moe_fp8": (480, 48, 4)}
SUSTAINED_AFTER_S = 1.0  # a kernel timed over a region at least this long takes the sustained peak


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
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="longctx")
    ap.add_argument("--e2e-blocks", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    a = ap.parse_args()
    st, wu, eb = DEFAULTS.get(a.workload, (480, 48, 4))
    a.steps = st if a.steps is None else a.steps
    a.warmup = wu if a.warmup is None else a.warmup
    a.e2e_blocks = eb if a.e2e_blocks is None else a.e2e_blocks
    return a


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


def workload_label(cfg):
    moe = (f", MoE {cfg.n_experts}+{cfg.n_shared} experts top-{cfg.top_k} I{cfg.moe_inter}"
           if cfg.n_experts else "") + (", e4m3 LM head" if cfg.lm_fp8 else "") + \
        (", e4m3 experts" if cfg.moe_fp8 else "")
    return (f"{cfg.name}: B{cfg.B} C{cfg.C} S{cfg.S[0]} d{cfg.d} Hq{cfg.Hq}/Hk{cfg.Hk} h{cfg.h} V{cfg.V} "
            f"{cfg.dtype}{moe}, {cfg.max_steps}-step blocks, adaptive stop off")


def flops_bytes(cfg):
    """Algorithmic flops and HBM bytes of one step and of the two gated kernels.

    LM head: 2 M d V flops; bytes = the weights once + Hs once + one 32-byte
    partial record per (row, vocab partition) written (about 148 per 256 rows,
    counted as 148 per row here as an upper bound on that small term).
    Attention: 4 C (S + C) h Hq flops per request; bytes = the prompt K/V once,
    Q, the canvas K/V and O."""
    M, d, V = cfg.B * cfg.C, cfg.d, cfg.V
    qd, kd = cfg.Hq * cfg.h, cfg.Hk * cfg.h
    es = 2 if cfg.dtype == "bf16" else 4
    S = sum(cfg.S)
    f_qkv = 2 * M * d * (qd + 2 * kd)
    f_attn = sum(4 * cfg.C * (s + cfg.C) * cfg.h * cfg.Hq for s in cfg.S)
    f_wo = 2 * M * qd * d
    f_lm = 2 * M * d * V
    f_moe = 0
    b_moe = 0
    if cfg.n_experts:
        I = cfg.moe_inter
        f_moe = 2 * M * d * cfg.n_experts + M * (cfg.top_k + cfg.n_shared) * 6 * d * I
        ex_es = 1 if getattr(cfg, "moe_fp8", False) else es  # e4m3 expert codes
        b_moe = (cfg.n_experts + cfg.n_shared) * 3 * d * I * ex_es + cfg.n_experts * d * es
    lm_es = 1 if getattr(cfg, "lm_fp8", False) else es  # e4m3 codes: one byte per weight
    b_lm = V * d * lm_es + M * d * lm_es + V * 4 * (lm_es == 1) + M * 148 * 32
    b_attn = 2 * S * kd * es + M * (2 * qd + 2 * kd) * es
    b_step = ((qd + 2 * kd) * d + d * qd) * es + V * d * lm_es + 2 * S * kd * es + M * d * es * 6 + b_moe
    return {"flops_step": f_qkv + f_attn + f_wo + f_lm + f_moe, "bytes_step": b_step,
            "flops_lm": f_lm, "bytes_lm": b_lm, "flops_attn": f_attn, "bytes_attn": b_attn}


def cpu_cores_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def oracle_model_of(cfg, wl):
    """The oracle's model dictionary for a workload (MoE and e4m3 LM-head
    weights included)."""
    m = {"dtype": cfg.dtype, "d": cfg.d, "Hq": cfg.Hq, "Hk": cfg.Hk, "h": cfg.h, "V": cfg.V}
    m.update({k: wl.weights[k] for k in ("embed", "wq", "wk", "wv", "wo", "lm_head")})
    if cfg.lm_fp8:
        m["lm_head_e4m3"], m["lm_head_scale"] = wl.weights["lm_head"], wl.weights["lm_head_scale"]
    if cfg.n_experts:
        m.update(n_experts=cfg.n_experts, top_k=cfg.top_k, moe_inter=cfg.moe_inter, n_shared=cfg.n_shared)
        m.update({k: wl.weights[k] for k in ("w_router", "w_gate", "w_up", "w_down")})
        if cfg.moe_fp8:
            m.update({k: wl.weights[k] for k in ("w_gate_scale", "w_up_scale", "w_down_scale")})
    return m


def oracle_step_timer(cfg, wl):
    """run(rows, n): wall time of n oracle denoise steps (adaptive stop off)
    on the first `rows` positions of every canvas of the workload, restarting
    the block when it is done. Weights and prefix K/V are widened to fp64
    first (outside the timed calls)."""
    from oracle import model as om
    m = oracle_model_of(cfg, wl)
    m = om.prewiden(m, ("wq", "wk", "wv", "wo") if cfg.lm_fp8 else ("wq", "wk", "wv", "wo", "lm_head"))
    prefix = [(om.widen(k, cfg.dtype), om.widen(v, cfg.dtype)) for k, v in zip(wl.prefix_k, wl.prefix_v)]
    sched = {"max_steps": cfg.max_steps, "stop_entropy": cfg.stop_entropy, "adaptive_stop": False}

    def run(rows, n):
        invT = None
        if cfg.inv_temp != "one":
            invT = wl.inv_temp.reshape(cfg.B, cfg.C)[:, :rows].reshape(-1)
        st = om.init_state(wl.seeds, rows, cfg.V)
        t0 = time.perf_counter()
        for _ in range(n):
            st, _ = om.denoise_step(m, prefix, st, sched, invT)
            if st["done"].all():
                st = om.init_state(wl.seeds, rows, cfg.V)
        return time.perf_counter() - t0
    return run


def oracle_rate(cfg, wl, budget_s, n_steps=None, n_warm=0):
    """The fp64 oracle's denoise steps/s on this host, within about budget_s.

    A per-step cost model t(r) = a + b r (a: work independent of the sampled
    rows, such as streaming the widened weights; b: per canvas row) is
    calibrated from steps on 1 row and on r2 = min(C, 16) rows. When a full
    step fits the budget, full steps are timed; otherwise steps on the first r
    rows of every canvas (r as large as the budget allows) are timed and the
    full-step time is the measured sample step plus (C - r) rows at the
    per-row cost b (the sampled rows attend to S + r keys instead of S + C;
    the prompt dominates the keys of the large workloads).
    Returns (steps/s, description of the sample)."""
    run = oracle_step_timer(cfg, wl)
    tc0 = time.perf_counter()
    t1 = run(1, 2) / 2
    r2 = min(cfg.C, 16)
    t2 = run(r2, 1) if r2 > 1 else t1
    b = max(0.0, (t2 - t1) / max(1, r2 - 1))
    a = max(1e-4, t1 - b)
    left = max(5.0, budget_s - (time.perf_counter() - tc0))
    n = n_steps or max(1, int(left / max(1e-3, a + b * cfg.C)))
    per_step = left / max(1, n + n_warm)
    rows = int(max(1, min(cfg.C, (per_step - a) / b if b > 0 else cfg.C)))
    if n_warm:
        run(rows, n_warm)
    dt = run(rows, n)
    t_full = dt / n + b * (cfg.C - rows)
    if rows == cfg.C:
        sample = (f"{n} full oracle denoise steps (fp64 numpy) of the {cfg.name} workload "
                  f"({cfg.B} x {cfg.C} positions)")
    else:
        sample = (f"{n} oracle denoise steps (fp64 numpy) on the first {rows} of {cfg.C} positions of each of the "
                  f"{cfg.B} canvas(es) of the {cfg.name} workload (full prompt, full vocabulary); full-step time = "
                  f"measured sample step + {cfg.C - rows} rows x the per-row cost ({b * 1e3:.2f} ms/row, "
                  f"calibrated on 1- and {r2}-row steps)")
    return 1.0 / t_full, sample


def source_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_of(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu
    summary, or None when there is none or the kernel's source changed since."""
    path = os.path.join(ROOT, "profiles", f"traffic_{kernel}_{workload}.json")
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("source_sha256_16") != source_sha(t["source"]):
            return None
        return t.get("bytes_per_launch")
    except Exception:
        return None


# ---------------------------------------------------------------- reference arm
def bench_reference(args, rank, world):
    """The fp64 oracle on this host's cores, on the same workload and unit.

    Each reference step is a bounded sample of one denoise step (see
    oracle_rate): the oracle's full step (embed, Q/K/V, attention over the
    whole prompt, Wo + residual (+ MoE), LM head over the whole vocabulary,
    entropy/argmax, freeze, re-noise) on the first r canvas positions, r
    chosen so that warm-up + timed steps fit in about REF_BUDGET_S seconds."""
    if rank != 0:
        return 0
    from token_canvas_denoising_b200 import inputs as fx
    cfg = workload_cfg(args.workload)
    wl = fx.make_workload(cfg)
    v, sample = oracle_rate(cfg, wl, REF_BUDGET_S, n_steps=args.steps, n_warm=args.warmup)
    line = {"impl": "reference", "metric": "denoise steps/s", "value": v, "unit": "steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "canvas_tokens_per_s": v * cfg.B * cfg.C,
            "config": {"workload": workload_label(cfg)},
            "cpu_baseline": {"value": v, "unit": "steps/s", "cores": cpu_cores_used(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- b200 arm
FP8_OVER_BF16 = 2.0  # nominal dense ratio 4.5 / 2.25 PFLOP/s


def peak_kind_of(region_s, clocks):
    """Which measured tensor peak a kernel timed in the step loop is held to:
    the sustained one (measured under the power cap) when the clock record of
    the timed region shows the cap active, or the region lasted a second or
    more; the burst one otherwise."""
    capped = "sw_power_cap" in (clocks or {}).get("reasons", [])
    return "sustained" if (region_s >= SUSTAINED_AFTER_S or capped) else "burst"


def kernel_roofline(name, kernel, flops, bytes_, avg_ms, peaks, peak_kind, traffic, fp8=False):
    """A contraction's roofline against the peak of its own operand type: the
    measured bf16 peak, times the nominal FP8/bf16 ratio for e4m3 operands."""
    mult = FP8_OVER_BF16 if fp8 else 1.0
    peak = mult * (peaks["bf16_tflops_sustained"] if peak_kind == "sustained" else peaks["bf16_tflops"])
    tflops = flops / (avg_ms / 1e3) / 1e12
    t_roof = max(flops / (mult * peaks["bf16_tflops"] * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9)) * 1e3
    return {"bound": "tensor", "kernel": kernel, "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
            "frac": tflops / peak, "traffic": traffic,
            "peak_source": f"{peaks['source']} {peak_kind} bf16"
                           + (" x 2 (nominal e4m3/bf16 dense ratio)" if fp8 else "") + " ("
                           + ("kernel timed inside a step loop under the power cap or of a second or more"
                              if peak_kind == "sustained"
                              else "kernel timed inside a step loop shorter than 1 s, power cap not reached")
                           + ")",
            "avg_ms": avg_ms, "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": bytes_,
            "hbm_bound_ms": bytes_ / (peaks["hbm_gbs"] * 1e9) * 1e3, "roofline_ms": t_roof,
            "frac_of_roofline_time": t_roof / avg_ms}


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
    cv.sync()
    n_resets = (args.steps - 1) // BLOCK_STEPS
    if world > 1:
        elapsed_ms = max_over_ranks(elapsed_ms, world, "cuda")
        dist.barrier()

    # ---- timed region 2: the same steps with CUDA events recorded on the
    # step's stream around the LM-head kernel and around the attention kernel
    # (rings of NEV event pairs, one graph variant each): the gated kernels'
    # average launch durations
    NEV = 4
    ev = {k: ([torch.cuda.Event(enable_timing=True) for _ in range(NEV)],
              [torch.cuda.Event(enable_timing=True) for _ in range(NEV)]) for k in ("lmhead", "attention")}
    for s_, e_ in ev.values():
        for e in s_ + e_:  # torch creates the CUDA event on its first record
            e.record(stream)
    for k, (s_, e_) in ev.items():
        cv.set_timing_events(s_, e_, kernel=k)
    cv.reset()
    run_steps(NEV, 0)  # capture every variant before timing
    cv.sync()
    cv.reset()
    k_steps = min(args.steps, 960)
    dur = {k: [] for k in ev}
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for i in range(k_steps):
        if i % BLOCK_STEPS == 0 and i > 0:
            cv.reset()
        cv.step(sched)
        j = i - (NEV - 1)
        if j >= 0:  # the pairs used NEV-1 steps ago: wait for them (NEV-1 steps stay queued)
            for k, (s_, e_) in ev.items():
                e_[j % NEV].synchronize()
                dur[k].append(s_[j % NEV].elapsed_time(e_[j % NEV]))
    r1.record(stream)
    torch.cuda.synchronize()
    for j in range(max(0, k_steps - (NEV - 1)), k_steps):
        for k, (s_, e_) in ev.items():
            dur[k].append(s_[j % NEV].elapsed_time(e_[j % NEV]))
    region2_s = r0.elapsed_time(r1) / 1e3
    ck = clocks.stop()
    for k in ev:
        cv.set_timing_events([], [], kernel=k)
    steps_per_s = job_rate(args.steps, world, elapsed_ms)
    peak_kind = peak_kind_of(region2_s, ck)
    # more than 128 rows run on CTA pairs (lmhead_tc_pair_kernel)
    lm_kernel = "lmhead_tc_pair_kernel" if cfg.B * cfg.C > 128 else "lmhead_tc_kernel"
    lm = kernel_roofline("lmhead", lm_kernel + "<" + ("e4m3" if cfg.lm_fp8 else "bf16")
                         + "> (LM head + entropy/argmax)", fb["flops_lm"], fb["bytes_lm"],
                         float(np.mean(dur["lmhead"])), peaks, peak_kind, traffic_of(lm_kernel, cfg.name),
                         fp8=cfg.lm_fp8)
    at = kernel_roofline("attention", "attn_tc_kernel (+ attn_merge_kernel for units shared by CTAs)", fb["flops_attn"],
                         fb["bytes_attn"], float(np.mean(dur["attention"])), peaks, peak_kind,
                         traffic_of("attn_tc_kernel", cfg.name))

    # ---- end to end through the C ABI with host buffers: per block, the initial
    # state goes host->device (pinned), dg_decode_block runs the block's steps
    # (its loop on the device) and the tokens come back device->host
    e2e = None
    if rank == 0 or world > 1:
        cv.reset()  # a fresh block: step 0, nothing frozen
        st0 = cv.get_state()
        pin = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in st0.items()}
        pin_np = {k: v.numpy() for k, v in pin.items()}
        tok_out = torch.empty(cfg.B * cfg.C, dtype=torch.int32).pin_memory()
        cv.set_state(pin_np)
        cv.decode(sched, tok_out)  # warm (builds the decode graph)
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
        v, sample = oracle_rate(cfg, wl, args.cpu_seconds)
        cpu = {"value": v, "unit": "steps/s", "cores": cpu_cores_used(), "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": "denoise steps/s", "value": steps_per_s, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic",
            "canvas_tokens_per_s": steps_per_s * cfg.B * cfg.C,
            "config": {"workload": workload_label(cfg),
                       "batch_canvases": cfg.B, "canvas_len": cfg.C, "prefix_len": cfg.S[0],
                       "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2: each step streams {fb['bytes_step'] / 1e6:.0f} MB of weights "
                             "and prefix K/V (> 126 MB L2)"},
            "clocks": ck,
            "e2e": e2e,
            "gpu_launches": int(args.steps * launches_per_step + n_resets),
            "roofline": lm,
            "rooflines": {"lmhead": lm, "attention": at},
            "step_roofline": {"flops": fb["flops_step"], "bytes": fb["bytes_step"],
                              "ms": max((fb["flops_step"] - fb["flops_lm"] * (1 - 1 / FP8_OVER_BF16) * cfg.lm_fp8)
                                        / (peaks["bf16_tflops"] * 1e12),
                                        fb["bytes_step"] / (peaks["hbm_gbs"] * 1e9)) * 1e3},
            "kernel_timing_region_s": region2_s,
            "cpu_baseline": cpu,
        }
        line["step_roofline"]["frac"] = line["step_roofline"]["ms"] / line["ms_per_step"]
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

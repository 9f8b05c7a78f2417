"""Turns a seeded Workload into the fp64 oracle's model dictionary.

Test-only glue: it moves arrays, it computes nothing."""
from oracle import model as om


def oracle_model(wl):
    c = wl.cfg
    m = {"dtype": c.dtype, "d": c.d, "Hq": c.Hq, "Hk": c.Hk, "h": c.h, "V": c.V}
    if c.n_layers:  # stacked layer weights and per-layer prompt caches
        m["n_layers"] = c.n_layers
    for k in ("embed", "wq", "wk", "wv", "wo", "lm_head"):
        m[k] = wl.weights[k]
    if c.lm_fp8:  # e4m3 codes with power-of-two row scales
        m["lm_head_e4m3"] = wl.weights["lm_head"]
        m["lm_head_scale"] = wl.weights["lm_head_scale"]
    if c.n_experts:
        m.update(n_experts=c.n_experts, top_k=c.top_k, moe_inter=c.moe_inter,
                 n_shared=c.n_shared)
        for k in ("w_router", "w_gate", "w_up", "w_down"):
            m[k] = wl.weights[k]
        if c.moe_fp8:  # e4m3 expert codes with row scales
            for k in ("w_gate_scale", "w_up_scale", "w_down_scale"):
                m[k] = wl.weights[k]
    return m


def oracle_prefix(wl):
    return list(zip(wl.prefix_k, wl.prefix_v))


def oracle_sched(cfg, adaptive=True, max_steps=None):
    return {"max_steps": cfg.max_steps if max_steps is None else max_steps,
            "stop_entropy": cfg.stop_entropy, "adaptive_stop": adaptive}


def oracle_init(wl):
    return om.init_state(wl.seeds, wl.cfg.C, wl.cfg.V)

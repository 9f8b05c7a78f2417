"""Comparison of the CUDA path with the fp64 oracle, step by step and stage by
stage.

Every stage of a GPU step is compared with the oracle fed the GPU's own
inputs to that stage, so each comparison measures that stage alone and uses
the stated tolerances without widening:

  stage                    oracle input               GPU output       tolerance
  Q, canvas K/V            the canvas tokens          q, k/v_canvas    |d| <= 1e-2 + 2e-2 |ref|
  attention O              GPU Q, K_c, V_c            attn_out         |d| <= 1e-2 + 2e-2 |ref|
  Wo + residual            GPU O (and the tokens)     hidden_attn      |d| <= 1e-2 + 2e-2 |ref|
  MoE block                GPU hidden_attn            hidden           |d| <= 1e-2 + 2e-2 |ref|
  LM head entropy          GPU hidden                 ent              |d| <= 1e-3 nats
  LM head argmax           GPU hidden                 argmax           equal
  freeze / stop / renoise  oracle entropies and       state after      equal
                           argmax of GPU hidden

Integer decisions are bit-exact except where the oracle's own decision is
within 1e-3 of a tie ("ambiguous"):
  - argmax: top-1 minus top-2 (unscaled) logit <= 1e-3; the GPU's token must
    then be within 1e-3 of the top logit;
  - freeze cut: positions whose entropy is within 1e-3 of the midpoint between
    the k-th and (k+1)-th smallest unfrozen entropies; the GPU must still
    freeze exactly k positions, each below the cut + 1e-3;
  - stop test: the smallest still-unfrozen entropy (over the positions the GPU
    left unfrozen) within 1e-3 of the threshold;
  - MoE routing: the k-th and (k+1)-th router logits within 1e-3; the GPU row
    must then match the oracle's output for one of the valid expert choices.
The GPU's stop decision must always agree with its own entropies and freeze
set. Where the GPU took another valid choice at an ambiguous decision, the
oracle continues from the GPU's state (free-running mode) and the step is
counted as diverged; every ambiguous decision is counted and reported.
"""
import itertools

import numpy as np

from oracle import model as om
from oracle import philox as op

ENT_TOL = 1e-3
AMBIG = 1e-3
ABS_TOL = 1e-2
REL_TOL = 2e-2
MAX_ROUTE_CHOICES = 16


def close(gpu, ref, atol=ABS_TOL, rtol=REL_TOL):
    """Count elements with |gpu - ref| > atol + rtol |ref|; also the largest |gpu - ref|."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    bad = np.abs(gpu - ref) > atol + rtol * np.abs(ref)
    return int(np.count_nonzero(bad)), float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0


def freeze_ambiguity(ent_row, frozen_row, k):
    """Oracle cut for one canvas: (tau, ambiguous mask over positions)."""
    unf = np.nonzero(~frozen_row)[0]
    if k <= 0 or k >= len(unf):
        return None, np.zeros(len(ent_row), bool)
    order = unf[np.argsort(ent_row[unf], kind="stable")]
    tau = 0.5 * (ent_row[order[k - 1]] + ent_row[order[k]])
    amb = np.zeros(len(ent_row), bool)
    amb[unf] = np.abs(ent_row[unf] - tau) <= AMBIG
    return tau, amb


class StepReport:
    """Errors and counts over a run of steps."""

    COUNTS = ("steps", "amb_argmax", "amb_cut", "amb_stop", "amb_route", "div_argmax", "div_freeze",
              "div_route", "diverged_steps")

    def __init__(self):
        self.errors = []
        for k in self.COUNTS:
            setattr(self, k, 0)
        self.max_dev = {}

    def fail(self, msg):
        self.errors.append(msg)

    def dev(self, name, value):
        self.max_dev[name] = max(self.max_dev.get(name, 0.0), float(value))

    @property
    def ambiguous(self):
        return self.amb_argmax + self.amb_cut + self.amb_stop + self.amb_route

    def summary(self):
        c = ", ".join(f"{k}={getattr(self, k)}" for k in self.COUNTS)
        d = ", ".join(f"{k}={v:.3g}" for k, v in sorted(self.max_dev.items()))
        return f"{c}; max deviations: {d}"


def _np(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def route_choices(r_row, k):
    """The valid top-k expert sets of one row within the routing tolerance:
    experts clearly above the cut are always chosen; the rest of the k come
    from the experts within 1e-3 of the cut. The oracle's own choice first."""
    order = np.argsort(-r_row, kind="stable")
    primary = tuple(sorted(order[:k].tolist()))
    if k >= len(r_row):
        return [primary], False
    cut = 0.5 * (r_row[order[k - 1]] + r_row[order[k]])
    near = [int(e) for e in np.nonzero(np.abs(r_row - cut) <= AMBIG)[0]]
    if r_row[order[k - 1]] - r_row[order[k]] > AMBIG:
        return [primary], False
    sure = [int(e) for e in np.nonzero(r_row > cut + AMBIG)[0]]
    need = k - len(sure)
    out = [primary]
    for comb in itertools.combinations(sorted(near), need):
        c = tuple(sorted(sure + list(comb)))
        if c != primary:
            out.append(c)
        if len(out) >= MAX_ROUTE_CHOICES:
            break
    return out, True


def check_tensor_stages(cfg, omodel, oprefix, tok, gpu, rep):
    """Q/K/V, attention, Wo + residual and MoE, each against the oracle fed
    the GPU's own input to that stage. With a stack of L layers, layer l < L-1
    is compared as a whole (its output against the oracle's layer l fed the
    GPU's input to it) and the last layer stage by stage."""
    B, C = cfg.B, cfg.C
    L = om.n_layers(omodel)
    X = om.embed(omodel, tok)
    lo = gpu.get("layer_out")
    for l in range(L - 1):
        ref = om.attention_layer(omodel, oprefix, X, B, C, l)[4]
        n, mx = close(lo[l], ref)
        rep.dev(f"layer{l}_out", mx)
        if n:
            rep.fail(f"layer {l} output: {n} elements out of tolerance (max abs diff {mx:.3g})")
        X = lo[l].astype(np.float64)
    if lo is not None and not np.array_equal(lo[L - 1], gpu["hidden_attn"]):
        rep.fail("the last layer's output differs from hidden_attn")
    last, oprefix = om.layer(omodel, L - 1), om.layer_prefix(omodel, oprefix, L - 1)
    omodel = last
    Qo, Kco, Vco = om.project_qkv(omodel, X)
    for name, g, o in (("q", gpu["q"], Qo), ("k_canvas", gpu["k_canvas"], Kco), ("v_canvas", gpu["v_canvas"], Vco)):
        n, mx = close(g, o.reshape(g.shape))
        rep.dev(name, mx)
        if n:
            rep.fail(f"{name}: {n} elements out of tolerance (max abs diff {mx:.3g})")
    Qg = gpu["q"].reshape(B * C, cfg.Hq, cfg.h).astype(np.float64)
    Kg = gpu["k_canvas"].reshape(B * C, cfg.Hk, cfg.h).astype(np.float64)
    Vg = gpu["v_canvas"].reshape(B * C, cfg.Hk, cfg.h).astype(np.float64)
    Oo = om.attention(omodel, Qg, Kg, Vg, oprefix, B, C)
    n, mx = close(gpu["attn_out"], Oo)
    rep.dev("attn_out", mx)
    if n:
        rep.fail(f"attention output: {n} elements out of tolerance (max abs diff {mx:.3g})")
    Hs_attn_o = om.out_proj_residual(omodel, X, gpu["attn_out"].astype(np.float64))
    n, mx = close(gpu["hidden_attn"], Hs_attn_o)
    rep.dev("hidden_attn", mx)
    if n:
        rep.fail(f"hidden after attention and Wo: {n} elements out of tolerance (max abs diff {mx:.3g})")
    if not cfg.n_experts:
        if not np.array_equal(gpu["hidden"], gpu["hidden_attn"]):
            rep.fail("hidden differs from hidden_attn without an MoE block")
        return
    Hsa = gpu["hidden_attn"].astype(np.float64)
    Hs_o, (r, idx, gates) = om.moe_block(omodel, Hsa)
    tol = ABS_TOL + REL_TOL * np.abs(Hs_o)
    ok = np.all(np.abs(gpu["hidden"] - Hs_o) <= tol, axis=1)
    for row in range(Hs_o.shape[0]):
        choices, amb = route_choices(r[row], cfg.top_k)
        if amb:
            rep.amb_route += 1
        if ok[row]:
            continue
        matched = False
        for ch in choices[1:]:
            alt, _ = om.moe_block(omodel, Hsa[row:row + 1], choice=[list(ch)])
            if np.all(np.abs(gpu["hidden"][row] - alt[0]) <= ABS_TOL + REL_TOL * np.abs(alt[0])):
                matched = True
                rep.div_route += 1
                break
        if not matched:
            d = np.abs(gpu["hidden"][row] - Hs_o[row])
            rep.fail(f"hidden after MoE, row {row}: max abs diff {d.max():.3g} "
                     f"({len(choices)} valid routing choice(s) tried)")
    if ok.any():
        rep.dev("hidden", float(np.max(np.abs(gpu["hidden"][ok] - Hs_o[ok]))))


def check_step(cfg, omodel, oprefix, osched, inv_temp, st_before, gpu, gst_after, rep, check_tensors=True):
    """Compare one GPU step, started from st_before (oracle layout, equal to
    the GPU's state before the step), stage by stage. gpu: numpy debug outputs;
    gst_after: the GPU's state after the step (ABI layout).
    Returns the oracle's state after the step: its own when the GPU took the
    same decisions, the GPU's when the GPU took another valid choice at an
    ambiguous decision (checked here)."""
    B, C, V = cfg.B, cfg.C, cfg.V
    tok = st_before["tok"]
    rep.steps += 1
    if check_tensors:
        check_tensor_stages(cfg, omodel, oprefix, tok, gpu, rep)

    # ---- LM head stage: the oracle on the GPU's own residual stream
    hidden = gpu["hidden"].astype(np.float64)
    invT = np.ones(B * C) if inv_temp is None else np.asarray(inv_temp, np.float64).reshape(-1)
    logits = om.lm_head_logits(omodel, hidden)
    ent_o, am_o, gap_o = om.entropy_argmax(logits, invT)
    ent_g = gpu["ent"].astype(np.float64)
    am_g = gpu["argmax"].astype(np.int64)
    d = np.abs(ent_g - ent_o)
    rep.dev("entropy", float(np.max(d)))
    if np.any(d > ENT_TOL):
        at = int(np.argmax(d))
        rep.fail(f"entropy off by {d[at]:.3g} nats at row {at} (tolerance {ENT_TOL})")
    live = np.repeat(~st_before["done"], C)
    am_amb = (gap_o <= AMBIG) & live
    rep.amb_argmax += int(np.count_nonzero(am_amb))
    wrong = am_g != am_o
    if np.any(wrong & ~am_amb & live):
        bad = np.nonzero(wrong & ~am_amb & live)[0]
        rep.fail(f"argmax differs at rows {bad[:6].tolist()} (oracle top-2 gap {gap_o[bad[0]]:.3g})")
    for row in np.nonzero(wrong & am_amb)[0]:
        if not (0 <= am_g[row] < V) or logits[row, am_g[row]] < logits[row, am_o[row]] - AMBIG:
            rep.fail(f"argmax at row {row}: GPU token {am_g[row]} is not within {AMBIG} of the top logit")
        else:
            rep.div_argmax += 1

    # ---- selection stage: the oracle's decisions from those entropies
    ent_o2 = ent_o.reshape(B, C)
    am_g2 = am_g.reshape(B, C)
    ost_next, recs = om.apply_selection(st_before, ent_o2, am_o.reshape(B, C), osched, V)
    fm_g = gpu["freeze_mask"].reshape(B, C).astype(bool)
    tok_g = gst_after["tokens"].reshape(B, C).astype(np.int64)
    fr_g = gst_after["frozen"].reshape(B, C).astype(bool)
    ent_g32 = gpu["ent"].reshape(B, C).astype(np.float32)
    thr = np.float32(osched["stop_entropy"])
    adaptive = bool(osched["adaptive_stop"])
    for b in range(B):
        rec = recs[b]
        if rec is None:  # canvas already done: nothing may change
            if not np.array_equal(tok_g[b], tok[b]) or bool(gst_after["done"][b]) is not True:
                rep.fail(f"canvas {b} changed after done")
            if int(gst_after["step"][b]) != int(st_before["step"][b]):
                rep.fail(f"canvas {b}: step counter moved after done")
            continue
        frozen0 = st_before["frozen"][b]
        k = rec["k"]
        tau, amb = freeze_ambiguity(ent_o2[b], frozen0, k)
        rep.amb_cut += int(np.count_nonzero(amb))
        if fm_g[b].sum() != k:
            rep.fail(f"canvas {b}: froze {fm_g[b].sum()} positions, the schedule says {k}")
        if np.any(fm_g[b] & frozen0):
            rep.fail(f"canvas {b}: re-froze a frozen position")
        diff = fm_g[b] != rec["freeze"]
        if np.any(diff & ~amb):
            rep.fail(f"canvas {b}: freeze set differs at unambiguous positions {np.nonzero(diff & ~amb)[0][:8].tolist()}")
        elif np.any(diff):
            rep.div_freeze += 1
        # stop test on the positions the GPU left unfrozen
        rest = ~(frozen0 | fm_g[b])
        gpu_stop = bool(gst_after["done"][b])
        self_stop = (not rest.any()) or (adaptive and bool(np.min(ent_g32[b][rest]) < thr))
        if gpu_stop != self_stop:
            rep.fail(f"canvas {b}: stop decision {gpu_stop} disagrees with the GPU's own entropies and freeze set")
        if rest.any():
            mr = float(np.min(ent_o2[b][rest]))
            o_stop = adaptive and mr < float(thr)
            stop_amb = adaptive and abs(mr - float(thr)) <= AMBIG
        else:
            o_stop, stop_amb = True, False
        if stop_amb:
            rep.amb_stop += 1
        elif gpu_stop != o_stop:
            rep.fail(f"canvas {b}: stop decision differs (gpu {gpu_stop}, oracle {o_stop})")
        if int(gst_after["step"][b]) != rec["t"] + 1:
            rep.fail(f"canvas {b}: step counter {gst_after['step'][b]} != {rec['t'] + 1}")
        # the GPU's own decisions are carried out as the method says
        if not np.array_equal(tok_g[b][frozen0], tok[b][frozen0]):
            rep.fail(f"canvas {b}: a frozen token changed")
        if not np.array_equal(tok_g[b][fm_g[b]], am_g2[b][fm_g[b]]):
            rep.fail(f"canvas {b}: a newly frozen token is not the argmax")
        if gpu_stop:
            if not np.all(fr_g[b]) or not np.array_equal(tok_g[b][rest], am_g2[b][rest]):
                rep.fail(f"canvas {b}: the stop did not commit the argmax of the open positions")
        else:
            if not np.array_equal(fr_g[b], frozen0 | fm_g[b]):
                rep.fail(f"canvas {b}: frozen mask is not the old one plus the freeze set")
            t = rec["t"]
            seed = int(st_before["seed"][b])
            want = np.array([op.canvas_draw(seed, t + 1, int(p), b, V) for p in np.nonzero(rest)[0]], np.int64)
            if not np.array_equal(tok_g[b][rest], want):
                rep.fail(f"canvas {b}: re-noise draws differ")
    gpu_next = abi_state_to_oracle(gst_after, B, C)
    same = all(np.array_equal(gpu_next[k], ost_next[k]) for k in ("tok", "frozen", "step", "done"))
    if same:
        return ost_next
    rep.diverged_steps += 1
    return gpu_next


def oracle_state_to_abi(st):
    return {"tokens": st["tok"].reshape(-1).astype(np.int32),
            "frozen": st["frozen"].reshape(-1).astype(np.uint8),
            "step": st["step"].astype(np.int32),
            "seed": st["seed"].astype(np.uint64),
            "done": st["done"].astype(np.uint8)}


def abi_state_to_oracle(s, B, C):
    return {"tok": s["tokens"].reshape(B, C).astype(np.int64),
            "frozen": s["frozen"].reshape(B, C).astype(bool),
            "step": s["step"].astype(np.int64),
            "done": s["done"].astype(bool),
            "seed": s["seed"].astype(np.uint64)}


def run_lockstep(cfg, canvas, omodel, oprefix, osched, abi_sched, inv_temp, n_steps=None,
                 free_running=True, check_tensors=True, init=None, tensor_steps=None):
    """Drive GPU and oracle side by side until every canvas is done (or
    n_steps). Free-running: the GPU keeps its own state for the whole decode
    (the oracle follows the GPU's valid choices at ambiguous decisions).
    Lock-step: the GPU restarts every step from the oracle's state.
    tensor_steps: if given, the tensor stages are compared only on these step
    indices (the LM-head and selection stages on every step).
    Returns (StepReport, steps run)."""
    rep = StepReport()
    ost = om.init_state(np.array(cfg.canvas_seeds, dtype=np.uint64), cfg.C, cfg.V) if init is None else init
    g0 = abi_state_to_oracle(canvas.get_state(), cfg.B, cfg.C)
    if not np.array_equal(g0["tok"], ost["tok"]):
        rep.fail("initial canvas differs from the oracle's Philox draws")
    steps = 0
    while not np.all(ost["done"]):
        if n_steps is not None and steps >= n_steps:
            break
        if not free_running:
            canvas.set_state(oracle_state_to_abi(ost))
        gpu = {k: _np(v) for k, v in canvas.step(abi_sched, debug=True).items()}
        gst = canvas.get_state()
        tens = check_tensors and (tensor_steps is None or steps in tensor_steps)
        ost = check_step(cfg, omodel, oprefix, osched, inv_temp, ost, gpu, gst, rep, check_tensors=tens)
        steps += 1
    rep.final_state = ost
    return rep, steps

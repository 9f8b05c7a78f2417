"""Comparison of the CUDA path with the fp64 oracle, step by step.

Tolerances (stated for the method's bf16 path; applied to f32 too):
  * attention output O and the residual stream: |gpu - ref| <= 1e-2 + 2e-2 |ref|
  * per-position entropy: |gpu - ref| <= 1e-3 nats
  * integers (argmax, freeze set, tokens, re-noise draws, steps): bit-exact,
    except where the oracle's decision is within 1e-3 of a tie:
      - argmax: top-1 minus top-2 logit <= 1e-3
      - freeze cut: positions whose oracle entropy is within 1e-3 of the
        midpoint between the k-th and (k+1)-th smallest unfrozen entropies
      - stop test: the smallest still-unfrozen oracle entropy within 1e-3 of
        the threshold
    There the GPU may decide either way but must stay valid (exactly k
    positions frozen, each to its argmax, every other one re-drawn).

Propagated tolerance for full-step comparisons. The GPU and the oracle both
round the residual stream Hs to bf16 at the same point, but from values that
differ in the last bits (f32 versus f64 accumulation, bf16 attention
probabilities), so an element of Hs can land one bf16 ulp apart. For a row
whose Hs equals the oracle's bit for bit the entropy must be within 1e-3 nats.
For a row with differing elements, the unscaled logit of any token can move by
at most dx = sum_i |dHs_i| max_v |W_vi|, and to first order the entropy of
softmax(l), l = invT x, moves by at most invT dx E_p|l - E_p l| (the derivative
of H with respect to l_j is -p_j (l_j - E_p l)); that bound plus 1e-3 is the
row's entropy tolerance, and argmax / freeze / stop decisions within those
bands count as ambiguous.

With the MoE block the residual stream is rounded twice: after attention and Wo
(Hs_attn) and after the MoE output is added (Hs). Hs_attn is checked with the
tolerance above. A one-ulp difference in an element of Hs_attn is carried into
Hs unchanged, so the Hs tolerance takes its relative part from
max(|Hs|, |Hs_attn|). The router sees the GPU's Hs_attn, so a row's routing is
ambiguous when the gap between its k-th and (k+1)-th oracle router logits is
within 1e-3 plus twice dr = max_e sum_i |dHs_attn_i| |W_router[e][i]|, the most
a router logit can move; such rows may follow another expert and their outputs
are not compared.
"""
import numpy as np

from oracle import model as om
from oracle import philox as op

ENT_TOL = 1e-3
AMBIG = 1e-3
ABS_TOL = 1e-2
REL_TOL = 2e-2


def close(gpu, ref, atol=ABS_TOL, rtol=REL_TOL, mag=None):
    """Count elements with |gpu - ref| > atol + rtol * mag (mag = |ref| by default)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    mag = np.abs(ref) if mag is None else np.asarray(mag, np.float64)
    bad = np.abs(gpu - ref) > atol + rtol * mag
    return int(np.count_nonzero(bad)), float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0


def freeze_ambiguity(ent_row, frozen_row, k, tol_row=None):
    """Oracle cut for one canvas: (tau, ambiguous mask over positions). A
    position is ambiguous when its entropy is within its own tolerance plus the
    largest tolerance of the two positions that define the cut."""
    unf = np.nonzero(~frozen_row)[0]
    if k <= 0 or k >= len(unf):
        return None, np.zeros(len(ent_row), bool)
    tol = np.full(len(ent_row), AMBIG) if tol_row is None else np.maximum(AMBIG, tol_row)
    order = unf[np.argsort(ent_row[unf], kind="stable")]
    tau = 0.5 * (ent_row[order[k - 1]] + ent_row[order[k]])
    cut_tol = max(tol[order[k - 1]], tol[order[k]])
    amb = np.zeros(len(ent_row), bool)
    amb[unf] = np.abs(ent_row[unf] - tau) <= np.maximum(AMBIG, tol[unf] + cut_tol - AMBIG)
    return tau, amb


class StepReport:
    def __init__(self):
        self.ambiguous = 0
        self.errors = []

    def fail(self, msg):
        self.errors.append(msg)


def propagated_tolerances(cfg, omodel, invT, gpu_hidden, oracle_hidden, wmax):
    """Per-row entropy tolerance and argmax band (see the module docstring)."""
    M = cfg.B * cfg.C
    dH = np.abs(np.asarray(gpu_hidden, np.float64) - np.asarray(oracle_hidden, np.float64))
    ent_tol = np.full(M, ENT_TOL)
    am_band = np.full(M, AMBIG)
    rows = np.nonzero(np.any(dH != 0.0, axis=1))[0]
    if rows.size:
        it = np.ones(M) if invT is None else np.asarray(invT, np.float64).reshape(-1)
        dx = dH[rows] @ wmax
        l = om.lm_head_logits(omodel, np.asarray(oracle_hidden, np.float64)[rows]) * it[rows][:, None]
        p = om.softmax_rows(l)
        lbar = np.sum(p * l, axis=1, keepdims=True)
        mad = np.sum(p * np.abs(l - lbar), axis=1)
        ent_tol[rows] = ENT_TOL + it[rows] * dx * mad
        am_band[rows] = np.maximum(AMBIG, 2.0 * dx)
    return ent_tol.reshape(cfg.B, cfg.C), am_band.reshape(cfg.B, cfg.C)


def route_ambiguous_rows(cfg, extras, omodel=None, gpu_hidden_attn=None):
    """Rows whose oracle MoE routing has its k-th and (k+1)-th router logits
    within 1e-3 plus twice the largest router-logit shift that the GPU's
    Hs_attn difference can cause: the GPU may pick the other expert there."""
    M = cfg.B * cfg.C
    amb = np.zeros(M, bool)
    route = extras.get("route")
    if route is None:
        return amb
    r = np.sort(route[0], axis=1)[:, ::-1]
    k = cfg.top_k
    band = np.full(M, AMBIG)
    if omodel is not None and gpu_hidden_attn is not None:
        dH = np.abs(np.asarray(gpu_hidden_attn, np.float64) - np.asarray(extras["Hs_attn"], np.float64))
        wr = np.abs(om.widen(omodel["w_router"], omodel["dtype"]))
        band = band + 2.0 * np.max(dH @ wr.T, axis=1)
    if k < r.shape[1]:
        amb = (r[:, k - 1] - r[:, k]) <= band
    return amb


def check_step(cfg, st_before, orec, ost_after, gpu, gst_after, rep, hidden_ref=None, attn_ref=None,
               ent_tol=None, am_band=None, skip_rows=None, hidden_attn_ref=None):
    """Compare one GPU step (started from st_before) with the oracle's.

    gpu: dict of numpy debug outputs (ent, argmax, freeze_mask, attn_out, hidden).
    gst_after: GPU state after the step (dict of numpy, flat as the ABI).
    ent_tol / am_band: per-position entropy tolerance and argmax ambiguity
    band ([B][C]); default 1e-3 everywhere.
    Returns True when the oracle step had an ambiguous decision."""
    B, C, V = cfg.B, cfg.C, cfg.V
    if ent_tol is None:
        ent_tol = np.full((B, C), ENT_TOL)
    if am_band is None:
        am_band = np.full((B, C), AMBIG)
    ent_g = gpu["ent"].reshape(B, C)
    am_g = gpu["argmax"].reshape(B, C)
    fm_g = gpu["freeze_mask"].reshape(B, C).astype(bool)
    tok_g = gst_after["tokens"].reshape(B, C)
    fr_g = gst_after["frozen"].reshape(B, C).astype(bool)
    ent_o, am_o, gap_o = orec["ent"], orec["am"], orec["gap"]
    ambiguous = False

    d = np.abs(ent_g - ent_o)
    if np.any(d > ent_tol):
        at = np.unravel_index(np.argmax(d - ent_tol), d.shape)
        rep.fail(f"entropy off by {d[at]:.3g} (tolerance {ent_tol[at]:.3g}) at {at}")
    am_amb = gap_o <= am_band
    if np.any((am_g != am_o) & ~am_amb):
        bad = np.argwhere((am_g != am_o) & ~am_amb)
        rep.fail(f"argmax mismatch at {bad[:4].tolist()} (gap {gap_o[tuple(bad[0])]:.3g})")
    if np.any(am_amb):
        ambiguous = True
    if attn_ref is not None and gpu.get("attn_out") is not None:
        n, mx = close(gpu["attn_out"], attn_ref)
        if n:
            rep.fail(f"attention output: {n} elements out of tolerance (max abs diff {mx:.3g})")
    mag = None
    if hidden_attn_ref is not None and gpu.get("hidden_attn") is not None:
        n, mx = close(gpu["hidden_attn"], hidden_attn_ref)
        if n:
            rep.fail(f"hidden before MoE: {n} elements out of tolerance (max abs diff {mx:.3g})")
        mag = np.maximum(np.abs(np.asarray(hidden_ref, np.float64)), np.abs(np.asarray(hidden_attn_ref, np.float64)))
    if hidden_ref is not None and gpu.get("hidden") is not None:
        keep = np.ones(B * C, bool) if skip_rows is None else ~skip_rows
        n, mx = close(gpu["hidden"][keep], np.asarray(hidden_ref)[keep], mag=None if mag is None else mag[keep])
        if n:
            bad = np.argwhere(np.abs(np.asarray(gpu["hidden"], np.float64) - hidden_ref) >
                              ABS_TOL + REL_TOL * (np.abs(hidden_ref) if mag is None else mag))
            bad = [b for b in bad.tolist() if keep[b[0]]][:4]
            rep.fail(f"hidden: {n} elements out of tolerance (max abs diff {mx:.3g}) at {bad}")

    for b in range(B):
        r = orec["canvas"][b]
        if r is None:  # canvas already done: nothing may change
            if not np.array_equal(tok_g[b], st_before["tok"][b]):
                rep.fail(f"canvas {b} changed after done")
            continue
        frozen0 = st_before["frozen"][b]
        k = r["k"]
        tau, amb = freeze_ambiguity(ent_o[b], frozen0, k, ent_tol[b])
        if fm_g[b].sum() != k:
            rep.fail(f"canvas {b}: froze {fm_g[b].sum()} positions, schedule says {k}")
        if np.any(fm_g[b] & frozen0):
            rep.fail(f"canvas {b}: re-froze a frozen position")
        if np.any(fm_g[b] != r["freeze"]):
            diff = fm_g[b] != r["freeze"]
            if np.any(diff & ~amb):
                rep.fail(f"canvas {b}: freeze set differs at unambiguous positions "
                         f"{np.nonzero(diff & ~amb)[0][:8].tolist()}")
            ambiguous = True
        if np.any(amb):
            ambiguous = True
        stop_amb = np.isfinite(r["min_rest"]) and abs(r["min_rest"] - cfg.stop_entropy) <= max(
            AMBIG, float(np.max(ent_tol[b])))
        if stop_amb:
            ambiguous = True
        gpu_stop = bool(gst_after["done"][b])
        if gpu_stop != r["stop"] and not stop_amb and not ambiguous:
            rep.fail(f"canvas {b}: stop decision differs (gpu {gpu_stop}, oracle {r['stop']})")
        if int(gst_after["step"][b]) != r["t"] + 1:
            rep.fail(f"canvas {b}: step counter {gst_after['step'][b]} != {r['t'] + 1}")
        # validity of the GPU's own decisions
        if not np.array_equal(tok_g[b][frozen0], st_before["tok"][b][frozen0]):
            rep.fail(f"canvas {b}: a frozen token changed")
        if not np.array_equal(tok_g[b][fm_g[b]], am_g[b][fm_g[b]]):
            rep.fail(f"canvas {b}: a newly frozen token is not the GPU argmax")
        rest = ~(frozen0 | fm_g[b])
        if gpu_stop:
            if not np.all(fr_g[b]) or not np.array_equal(tok_g[b][rest], am_g[b][rest]):
                rep.fail(f"canvas {b}: stop did not commit the argmax")
        else:
            t = r["t"]
            want = [op.canvas_draw(int(cfg.canvas_seeds[b]) if "seed" not in st_before else
                                   int(st_before["seed"][b]), t + 1, int(p), b, V)
                    for p in np.nonzero(rest)[0]]
            if not np.array_equal(tok_g[b][rest], np.array(want, dtype=tok_g.dtype)):
                rep.fail(f"canvas {b}: re-noise draws differ")
    if ambiguous:
        rep.ambiguous += 1
    else:
        # no ambiguous decision: the whole state must match the oracle's
        if not np.array_equal(tok_g, ost_after["tok"]):
            rep.fail("tokens differ from the oracle with no ambiguous decision")
        if not np.array_equal(fr_g, ost_after["frozen"]):
            rep.fail("frozen mask differs from the oracle with no ambiguous decision")
    return ambiguous


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


def lm_column_absmax(omodel):
    """max_v |W_lm[v][i]| per hidden dimension i (for the propagated tolerance)."""
    W = omodel["lm_head"]
    out = np.zeros(W.shape[1])
    for v0 in range(0, W.shape[0], 16384):
        out = np.maximum(out, np.max(np.abs(om.widen(W[v0:v0 + 16384], omodel["dtype"])), axis=0))
    return out


def run_lockstep(cfg, canvas, omodel, oprefix, osched, abi_sched, inv_temp, n_steps=None,
                 free_running=True, check_tensors=True, init=None):
    """Drive GPU and oracle side by side. In free-running mode the GPU keeps its
    own state while no ambiguous decision has happened; after one, and always in
    lock-step mode, the GPU restarts each step from the oracle's state.
    Returns the StepReport."""
    rep = StepReport()
    ost = om.init_state(np.array(cfg.canvas_seeds, dtype=np.uint64), cfg.C, cfg.V) if init is None else init
    g0 = canvas.get_state()
    init = abi_state_to_oracle(g0, cfg.B, cfg.C)
    if not np.array_equal(init["tok"], ost["tok"]):
        rep.fail("initial canvas differs from the oracle's Philox draws")
    synced = free_running
    steps = 0
    wmax = lm_column_absmax(omodel)
    while not np.all(ost["done"]):
        if n_steps is not None and steps >= n_steps:
            break
        if not synced:
            canvas.set_state(oracle_state_to_abi(ost))
        gpu = canvas.step(abi_sched, debug=True)
        gpu = {k: v.float().cpu().numpy() if v.dtype == __import__("torch").bfloat16 else v.cpu().numpy()
               for k, v in gpu.items()}
        gst = canvas.get_state()
        ost_next, orec = om.denoise_step(omodel, oprefix, ost, osched, inv_temp)
        ex = orec["extras"]
        skip = route_ambiguous_rows(cfg, ex, omodel, gpu.get("hidden_attn"))
        ent_tol, am_band = propagated_tolerances(cfg, omodel, inv_temp, gpu["hidden"], ex["Hs"], wmax)
        if skip.any():  # routing near a tie: the row's outputs may follow the other expert
            rep.ambiguous_routes = getattr(rep, "ambiguous_routes", 0) + int(skip.sum())
            ent_tol.reshape(-1)[skip] = np.inf
            am_band.reshape(-1)[skip] = np.inf
        amb = check_step(cfg, ost, orec, ost_next, gpu, gst, rep,
                         hidden_ref=ex["Hs"] if check_tensors else None,
                         attn_ref=ex["O"] if check_tensors else None,
                         ent_tol=ent_tol, am_band=am_band, skip_rows=skip,
                         hidden_attn_ref=ex["Hs_attn"] if (check_tensors and "route" in ex) else None)
        if amb:
            synced = False
        ost = ost_next
        steps += 1
    rep.final_state = ost
    return rep, steps

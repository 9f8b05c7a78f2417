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
"""
import numpy as np

from oracle import model as om
from oracle import philox as op

ENT_TOL = 1e-3
AMBIG = 1e-3
ABS_TOL = 1e-2
REL_TOL = 2e-2


def close(gpu, ref, atol=ABS_TOL, rtol=REL_TOL):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    bad = np.abs(gpu - ref) > atol + rtol * np.abs(ref)
    return int(np.count_nonzero(bad)), float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0


def freeze_ambiguity(ent_row, frozen_row, k):
    """Oracle cut for one canvas: (tau, ambiguous mask over positions)."""
    unf = np.nonzero(~frozen_row)[0]
    if k <= 0 or k >= len(unf):
        return None, np.zeros(len(ent_row), bool)
    srt = np.sort(ent_row[unf])
    tau = 0.5 * (srt[k - 1] + srt[k])
    amb = np.zeros(len(ent_row), bool)
    amb[unf] = np.abs(ent_row[unf] - tau) <= AMBIG
    return tau, amb


class StepReport:
    def __init__(self):
        self.ambiguous = 0
        self.errors = []

    def fail(self, msg):
        self.errors.append(msg)


def check_step(cfg, st_before, orec, ost_after, gpu, gst_after, rep, hidden_ref=None, attn_ref=None):
    """Compare one GPU step (started from st_before) with the oracle's.

    gpu: dict of numpy debug outputs (ent, argmax, freeze_mask, attn_out, hidden).
    gst_after: GPU state after the step (dict of numpy, flat as the ABI).
    Returns True when the oracle step had an ambiguous decision."""
    B, C, V = cfg.B, cfg.C, cfg.V
    ent_g = gpu["ent"].reshape(B, C)
    am_g = gpu["argmax"].reshape(B, C)
    fm_g = gpu["freeze_mask"].reshape(B, C).astype(bool)
    tok_g = gst_after["tokens"].reshape(B, C)
    fr_g = gst_after["frozen"].reshape(B, C).astype(bool)
    ent_o, am_o, gap_o = orec["ent"], orec["am"], orec["gap"]
    ambiguous = False

    d = np.abs(ent_g - ent_o)
    if np.any(d > ENT_TOL):
        rep.fail(f"entropy off by {d.max():.3g} at {np.unravel_index(np.argmax(d), d.shape)}")
    am_amb = gap_o <= AMBIG
    if np.any((am_g != am_o) & ~am_amb):
        bad = np.argwhere((am_g != am_o) & ~am_amb)
        rep.fail(f"argmax mismatch at {bad[:4].tolist()} (gap {gap_o[tuple(bad[0])]:.3g})")
    if np.any(am_amb):
        ambiguous = True
    if attn_ref is not None and gpu.get("attn_out") is not None:
        n, mx = close(gpu["attn_out"], attn_ref)
        if n:
            rep.fail(f"attention output: {n} elements out of tolerance (max abs diff {mx:.3g})")
    if hidden_ref is not None and gpu.get("hidden") is not None:
        n, mx = close(gpu["hidden"], hidden_ref)
        if n:
            rep.fail(f"hidden: {n} elements out of tolerance (max abs diff {mx:.3g})")

    for b in range(B):
        r = orec["canvas"][b]
        if r is None:  # canvas already done: nothing may change
            if not np.array_equal(tok_g[b], st_before["tok"][b]):
                rep.fail(f"canvas {b} changed after done")
            continue
        frozen0 = st_before["frozen"][b]
        k = r["k"]
        tau, amb = freeze_ambiguity(ent_o[b], frozen0, k)
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
        stop_amb = np.isfinite(r["min_rest"]) and abs(r["min_rest"] - cfg.stop_entropy) <= AMBIG
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


def run_lockstep(cfg, canvas, omodel, oprefix, osched, abi_sched, inv_temp, n_steps=None,
                 free_running=True, check_tensors=True):
    """Drive GPU and oracle side by side. In free-running mode the GPU keeps its
    own state while no ambiguous decision has happened; after one, and always in
    lock-step mode, the GPU restarts each step from the oracle's state.
    Returns the StepReport."""
    rep = StepReport()
    ost = om.init_state(np.array(cfg.canvas_seeds, dtype=np.uint64), cfg.C, cfg.V)
    g0 = canvas.get_state()
    init = abi_state_to_oracle(g0, cfg.B, cfg.C)
    if not np.array_equal(init["tok"], ost["tok"]):
        rep.fail("initial canvas differs from the oracle's Philox draws")
    synced = free_running
    steps = 0
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
        amb = check_step(cfg, ost, orec, ost_next, gpu, gst, rep,
                         hidden_ref=ex["Hs"] if check_tensors else None,
                         attn_ref=ex["O"] if check_tensors else None)
        if amb:
            synced = False
        ost = ost_next
        steps += 1
    return rep, steps

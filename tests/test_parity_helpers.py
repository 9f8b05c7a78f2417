"""CPU checks of the comparison rules the GPU parity tests use (tests/parity.py).

The element tolerance, the freeze-cut band and the routing choices are checked
on constructed cases. check_step is then run on "GPU outputs" made by the
oracle itself (its stages in storage precision, the selection carried out as
the method says): those must pass with no error, and each planted mistake in
them (a wrong entropy, argmax, freeze set, stop decision, re-noise draw,
frozen token, MoE routing) must be reported."""
import copy

import numpy as np
import pytest

from oracle import model as om
from oracle import philox as op
from token_canvas_denoising_b200 import inputs as fx
from tests import parity as pa
from tests.oracle_adapter import oracle_model, oracle_prefix, oracle_sched


def test_close_counts_against_ref():
    gpu, ref = np.array([1.0, 0.115]), np.array([1.011, 0.1])
    n, mx = pa.close(gpu, ref)  # 0.011 <= 0.01 + 0.02*1.011; 0.015 > 0.01 + 0.02*0.1
    assert n == 1 and abs(mx - 0.015) < 1e-12


def test_freeze_ambiguity_marks_only_positions_at_the_cut():
    ent = np.array([0.1, 0.2, 0.3, 0.3005, 0.9])
    tau, amb = pa.freeze_ambiguity(ent, np.zeros(5, bool), 3)
    assert abs(tau - 0.30025) < 1e-12 and amb.tolist() == [False, False, True, True, False]
    _, amb = pa.freeze_ambiguity(ent, np.zeros(5, bool), 1)
    assert not amb.any()
    tau, amb = pa.freeze_ambiguity(ent, np.array([False, False, True, False, False]), 2)
    assert abs(tau - 0.25025) < 1e-12 and not amb.any()  # the frozen position is not a candidate
    for k in (0, 5):
        tau, amb = pa.freeze_ambiguity(ent, np.zeros(5, bool), k)
        assert tau is None and not amb.any()


def test_route_choices_enumerate_the_near_ties_only():
    r = np.array([3.0, 1.0, 0.9995, 0.0, 2.0])
    choices, amb = pa.route_choices(r, 3)  # top-3 = {0, 4, 1}; expert 2 within 1e-3 of the cut
    assert amb and choices[0] == (0, 1, 4) and set(choices) == {(0, 1, 4), (0, 2, 4)}
    choices, amb = pa.route_choices(np.array([3.0, 1.0, 0.9, 0.0, 2.0]), 3)
    assert not amb and choices == [(0, 1, 4)]
    choices, amb = pa.route_choices(np.array([1.0, 1.0, 1.0, 0.0]), 2)  # three-way tie for two slots
    assert amb and set(choices) == {(0, 1), (0, 2), (1, 2)}


# ---------------------------------------------------------------- check_step on oracle-made outputs
def _small_case(moe=False, adaptive=False, layers=0):
    if layers:
        cfg = fx.Config("h_layers", B=2, C=12, S=(7, 0), d=32, Hq=2, Hk=1, h=16, V=64, dtype="f32", max_steps=5,
                        weight_seed=43, canvas_seeds=(3, 4), n_layers=layers)
    elif moe:
        cfg = fx.Config("h_moe", B=2, C=12, S=(7, 0), d=32, Hq=2, Hk=1, h=16, V=64, dtype="f32", max_steps=5,
                        weight_seed=41, canvas_seeds=(3, 4), n_experts=6, top_k=2, moe_inter=16, n_shared=1)
    else:
        cfg = fx.Config("h", B=2, C=12, S=(7, 0), d=32, Hq=2, Hk=1, h=16, V=64, dtype="f32", max_steps=5,
                        weight_seed=41, canvas_seeds=(3, 4))
    wl = fx.make_workload(cfg)
    return cfg, wl, oracle_model(wl), oracle_prefix(wl), oracle_sched(cfg, adaptive=adaptive)


def _fake_gpu_step(cfg, m, pre, sched, st):
    """A step made of the oracle's own stages, laid out as the GPU's debug
    outputs and ABI state."""
    new, rec = om.denoise_step(m, pre, st, sched, None)
    ex = rec["extras"]
    B, C = cfg.B, cfg.C
    fm = np.zeros((B, C), bool)
    for b, r in enumerate(rec["canvas"]):
        if r is not None:
            fm[b] = r["freeze"]
    gpu = {"ent": rec["ent"].reshape(-1).astype(np.float32), "argmax": rec["am"].reshape(-1).astype(np.int32),
           "freeze_mask": fm.reshape(-1).astype(np.uint8), "attn_out": ex["O"],
           "hidden": ex["Hs"], "hidden_attn": ex["Hs_attn"], "q": ex["Q"].reshape(B * C, -1),
           "k_canvas": ex["Kc"].reshape(B * C, -1), "v_canvas": ex["Vc"].reshape(B * C, -1),
           "layer_out": np.stack(ex["layers"])}
    return gpu, pa.oracle_state_to_abi(new), new


@pytest.mark.parametrize("moe,layers", [(False, 0), (True, 0), (False, 3)])
def test_check_step_accepts_the_oracles_own_steps(moe, layers):
    cfg, wl, m, pre, sched = _small_case(moe, layers=layers)
    st = om.init_state(wl.seeds, cfg.C, cfg.V)
    rep = pa.StepReport()
    while not st["done"].all():
        gpu, gst, new = _fake_gpu_step(cfg, m, pre, sched, st)
        nxt = pa.check_step(cfg, m, pre, sched, None, st, gpu, gst, rep)
        assert not rep.errors, rep.errors
        assert all(np.array_equal(nxt[k], new[k]) for k in ("tok", "frozen", "step", "done"))
        st = nxt
    assert rep.steps == cfg.max_steps and rep.diverged_steps == 0


def _planted(mutate, moe=False, adaptive=False, step=1):
    cfg, wl, m, pre, sched = _small_case(moe, adaptive)
    st = om.init_state(wl.seeds, cfg.C, cfg.V)
    for _ in range(step):
        st, _ = om.denoise_step(m, pre, st, sched, None)
    gpu, gst, _ = _fake_gpu_step(cfg, m, pre, sched, st)
    mutate(cfg, m, st, gpu, gst)
    rep = pa.StepReport()
    pa.check_step(cfg, m, pre, sched, None, st, gpu, gst, rep)
    return rep


def _first_rest(cfg, st, gpu):
    b = 0
    rest = np.nonzero(~st["frozen"][b] & ~gpu["freeze_mask"].reshape(cfg.B, cfg.C)[b].astype(bool))[0]
    return b * cfg.C + int(rest[0])


def test_planted_entropy_error_is_reported():
    def mut(cfg, m, st, gpu, gst):
        gpu["ent"][3] += np.float32(2e-3)
    assert any("entropy" in e for e in _planted(mut).errors)


def test_planted_argmax_error_is_reported():
    def mut(cfg, m, st, gpu, gst):
        gpu["argmax"][5] = (gpu["argmax"][5] + 1) % cfg.V
    assert any("argmax" in e for e in _planted(mut).errors)


def test_planted_freeze_swap_is_reported():
    def mut(cfg, m, st, gpu, gst):
        fm = gpu["freeze_mask"].reshape(cfg.B, cfg.C)
        on = np.nonzero(fm[0])[0][0]
        off = np.nonzero(~st["frozen"][0] & (fm[0] == 0))[0][-1]
        fm[0, on], fm[0, off] = 0, 1
    assert any("freeze set" in e for e in _planted(mut).errors)


def test_planted_wrong_renoise_draw_is_reported():
    def mut(cfg, m, st, gpu, gst):
        i = _first_rest(cfg, st, gpu)
        gst["tokens"][i] = (gst["tokens"][i] + 1) % cfg.V
    assert any("re-noise" in e for e in _planted(mut).errors)


def test_planted_changed_frozen_token_is_reported():
    def mut(cfg, m, st, gpu, gst):
        i = int(np.nonzero(st["frozen"][0])[0][0])
        gst["tokens"][i] = (gst["tokens"][i] + 1) % cfg.V
    assert any("frozen token changed" in e for e in _planted(mut, step=2).errors)


def test_planted_early_stop_is_reported():
    def mut(cfg, m, st, gpu, gst):
        gst["done"][0] = 1
    errs = _planted(mut).errors
    assert any("stop decision" in e for e in errs)


def test_planted_missed_adaptive_stop_is_reported():
    """A stop threshold above every entropy makes the oracle stop after the
    first freeze; a GPU that carries on is wrong by its own entropies too."""
    cfg, wl, m, pre, _ = _small_case()
    sched = {"max_steps": cfg.max_steps, "stop_entropy": 100.0, "adaptive_stop": True}
    st = om.init_state(wl.seeds, cfg.C, cfg.V)
    gpu, gst, new = _fake_gpu_step(cfg, m, pre, sched, st)
    assert new["done"].all()
    gst = pa.oracle_state_to_abi(om.init_state(wl.seeds, cfg.C, cfg.V))
    gst["done"][:] = 0
    rep = pa.StepReport()
    pa.check_step(cfg, m, pre, sched, None, st, gpu, gst, rep)
    assert any("disagrees with the GPU's own entropies" in e for e in rep.errors)


def test_planted_attention_error_is_reported():
    def mut(cfg, m, st, gpu, gst):
        gpu["attn_out"] = gpu["attn_out"].copy()
        gpu["attn_out"][2, 3] += 0.1
    assert any("attention output" in e for e in _planted(mut).errors)


def test_planted_moe_misroute_is_reported():
    """A row whose MoE output follows the wrong experts (not near a tie) fails."""
    def mut(cfg, m, st, gpu, gst):
        Hsa = gpu["hidden_attn"].astype(np.float64)
        r, idx, _ = om.moe_route(m, Hsa)
        wrong = np.argsort(r[4])[:cfg.top_k]  # the least likely experts
        alt, _ = om.moe_block(m, Hsa[4:5], choice=[list(wrong)])
        gpu["hidden"] = gpu["hidden"].copy()
        gpu["hidden"][4] = alt[0]
    errs = _planted(mut, moe=True).errors
    assert any("hidden after MoE, row 4" in e for e in errs)


def test_valid_choice_at_a_freeze_tie_is_followed_not_reported():
    """Two positions with (nearly) equal entropies at the cut: a GPU that
    freezes the other one is valid; the oracle then follows the GPU's state."""
    cfg, wl, m, pre, sched = _small_case()
    st = om.init_state(wl.seeds, cfg.C, cfg.V)
    gpu, gst, new = _fake_gpu_step(cfg, m, pre, sched, st)
    # move the entropy of the first position above the cut to just above the
    # k-th one by changing its hidden row to the k-th one's: same logits
    b = 0
    ent = gpu["ent"].reshape(cfg.B, cfg.C)[b].astype(np.float64)
    fm = gpu["freeze_mask"].reshape(cfg.B, cfg.C)[b].astype(bool)
    k = int(fm.sum())
    order = np.argsort(ent, kind="stable")
    p_in, p_out = int(order[k - 1]), int(order[k])
    hid = gpu["hidden"].copy()
    hid[b * cfg.C + p_out] = hid[b * cfg.C + p_in]
    gpu["hidden"] = hid
    gpu["hidden_attn"] = hid
    logits = om.lm_head_logits(m, hid.astype(np.float64))
    e2, a2, _ = om.entropy_argmax(logits, np.ones(cfg.B * cfg.C))
    gpu["ent"] = e2.astype(np.float32)
    gpu["argmax"] = a2.astype(np.int32)
    # the GPU freezes p_out instead of p_in (equal entropies: lower position wins in
    # the oracle; the other choice is within the band)
    lo, hi = min(p_in, p_out), max(p_in, p_out)
    fm2 = fm.copy()
    fm2[lo], fm2[hi] = False, True
    gpu["freeze_mask"].reshape(cfg.B, cfg.C)[b] = fm2
    tok = st["tok"].copy()
    frozen = st["frozen"] | gpu["freeze_mask"].reshape(cfg.B, cfg.C).astype(bool)
    am = gpu["argmax"].reshape(cfg.B, cfg.C)
    for bb in range(cfg.B):
        for p in range(cfg.C):
            if frozen[bb, p] and not st["frozen"][bb, p]:
                tok[bb, p] = am[bb, p]
            elif not frozen[bb, p]:
                tok[bb, p] = op.canvas_draw(int(st["seed"][bb]), 1, p, bb, cfg.V)
    gst = pa.oracle_state_to_abi({"tok": tok, "frozen": frozen, "step": st["step"] + 1,
                                  "seed": st["seed"], "done": np.zeros(cfg.B, bool)})
    rep = pa.StepReport()
    nxt = pa.check_step(cfg, m, pre, sched, None, st, gpu, gst, rep, check_tensors=False)
    assert not rep.errors, rep.errors
    assert rep.div_freeze == 1 and rep.diverged_steps == 1 and rep.amb_cut >= 2
    assert np.array_equal(nxt["tok"], tok) and np.array_equal(nxt["frozen"], frozen)


def test_planted_layer_error_is_reported():
    """A wrong output of an inner layer of a stack is reported for that layer."""
    cfg, wl, m, pre, sched = _small_case(layers=3)
    st = om.init_state(wl.seeds, cfg.C, cfg.V)
    gpu, gst, _ = _fake_gpu_step(cfg, m, pre, sched, st)
    gpu["layer_out"] = gpu["layer_out"].copy()
    gpu["layer_out"][1, 4, 2] += 0.5
    rep = pa.StepReport()
    pa.check_step(cfg, m, pre, sched, None, st, gpu, gst, rep)
    assert any("layer 1 output" in e for e in rep.errors)

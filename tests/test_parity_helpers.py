"""CPU checks of the comparison rules the GPU parity tests use (tests/parity.py):
the element tolerance, the freeze-cut ambiguity band, the MoE routing band and
the propagated entropy tolerance, on small constructed cases."""
import numpy as np

from oracle import model as om
from token_canvas_denoising_b200 import inputs as fx
from tests import parity as pa


def test_close_counts_against_ref_or_given_magnitude():
    gpu, ref = np.array([1.0, 0.115]), np.array([1.011, 0.1])
    n, mx = pa.close(gpu, ref)  # 0.011 <= 0.01 + 0.02*1.011; 0.015 > 0.01 + 0.02*0.1
    assert n == 1 and abs(mx - 0.015) < 1e-12
    n, _ = pa.close(gpu, ref, mag=np.array([1.0, 1.0]))  # relative part from a larger magnitude
    assert n == 0


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


def test_routing_band_grows_with_the_residual_difference():
    cfg = fx.Config(name="r", B=1, C=2, S=(0,), d=4, Hq=1, Hk=1, h=4, V=8, dtype="f32", max_steps=2,
                    weight_seed=1, canvas_seeds=(1,), n_experts=3, top_k=1, moe_inter=64, n_shared=0)
    logits = np.array([[1.0, 0.9995, 0.0], [1.0, 0.9, 0.0]])
    hs = np.zeros((2, 4))
    extras = {"route": (logits, None, None), "Hs_attn": hs}
    model = {"dtype": "f32", "w_router": np.full((3, 4), 0.5, np.float32)}
    amb = pa.route_ambiguous_rows(cfg, extras, model, hs)  # identical residuals: 1e-3 band
    assert amb.tolist() == [True, False]
    g = hs.copy()
    g[1, 0] = 0.1  # router logits of row 1 may move by 0.05: band 1e-3 + 0.1 covers its 0.1 gap
    amb = pa.route_ambiguous_rows(cfg, extras, model, g)
    assert amb.tolist() == [True, True]


def test_propagated_entropy_tolerance_bounds_the_actual_change():
    cfg = fx.Config(name="p", B=1, C=3, S=(0,), d=8, Hq=1, Hk=1, h=8, V=16, dtype="f32", max_steps=2,
                    weight_seed=1, canvas_seeds=(1,))
    rng = np.random.default_rng(0)
    model = {"dtype": "f32", "lm_head": rng.normal(0, 1, (16, 8)).astype(np.float32)}
    wmax = np.max(np.abs(model["lm_head"].astype(np.float64)), axis=0)
    hid = rng.normal(0, 1, (3, 8))
    invT = np.array([1.0, 3.0, 0.5])
    tol, band = pa.propagated_tolerances(cfg, model, invT, hid, hid, wmax)
    assert np.all(tol == pa.ENT_TOL) and np.all(band == pa.AMBIG)
    g = hid.copy()
    g[1, 2] += 2e-3
    tol, band = pa.propagated_tolerances(cfg, model, invT, g, hid, wmax)
    assert tol[0, 0] == pa.ENT_TOL and tol[0, 2] == pa.ENT_TOL and tol[0, 1] > pa.ENT_TOL
    ent = lambda h: om.entropy_of_logits(om.lm_head_logits(model, h[None, :]) * invT[1])[0]
    assert abs(ent(g[1]) - ent(hid[1])) <= tol[0, 1]
    assert band[0, 1] >= 2.0 * 2e-3 * wmax[2] - 1e-15

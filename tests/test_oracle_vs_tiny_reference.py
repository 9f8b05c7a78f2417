"""The oracle against an independent direct-formula implementation of the whole
loop (tests/tiny_reference.py) on tiny vocabularies: final tokens and step
counts must be identical and every step's per-position entropies equal to
1e-9 nats, for every initial canvas of V = 2, C = 4 and for random small cases
with and without the adaptive stop."""
import itertools

import numpy as np
import pytest

from oracle import model as om
from token_canvas_denoising_b200 import inputs as fx
from tests import tiny_reference as tr
from tests.oracle_adapter import oracle_init, oracle_model, oracle_prefix, oracle_sched


def _compare(cfg, adaptive, init=None):
    wl = fx.make_workload(cfg)
    st0 = oracle_init(wl)
    if init is not None:
        st0["tok"][:] = init
    fin, recs = om.decode(oracle_model(wl), oracle_prefix(wl), st0, oracle_sched(cfg, adaptive))
    tok, steps, ents = tr.decode(wl.weights, list(zip(wl.prefix_k, wl.prefix_v)), [int(s) for s in wl.seeds], cfg.C,
                           cfg.V, cfg.Hq, cfg.Hk, cfg.h, cfg.max_steps, cfg.stop_entropy, adaptive,
                           init_tok=None if init is None else init.tolist())
    assert fin["tok"].tolist() == tok
    assert fin["step"].tolist() == steps
    for b in range(cfg.B):
        for t in range(steps[b]):
            assert np.max(np.abs(recs[t]["ent"][b] - np.array(ents[b][t]))) < 1e-9, (b, t)


def test_draws_match_the_oracle_generator():
    from oracle import philox as op
    for (seed, step, pos, b, V) in [(0, 0, 0, 0, 2), (9, 3, 5, 1, 8), (2**40 + 7, 47, 255, 3, 262144)]:
        assert tr.draw(seed, step, pos, b, V) == op.canvas_draw(seed, step, pos, b, V)


@pytest.mark.parametrize("adaptive", [False, True])
def test_every_initial_canvas_v2_c4(adaptive):
    cfg = fx.Config(name="tiny2", B=1, C=4, S=(3,), d=8, Hq=2, Hk=1, h=4, V=2, dtype="f32", max_steps=3,
                    weight_seed=11, canvas_seeds=(9,))
    for init in itertools.product(range(2), repeat=4):
        _compare(cfg, adaptive, np.array([init]))


@pytest.mark.parametrize("V,C,B,adaptive", [(4, 5, 1, False), (8, 6, 2, True), (8, 6, 2, False), (4, 3, 3, True)])
def test_random_small_cases(V, C, B, adaptive):
    cfg = fx.Config(name="tinyr", B=B, C=C, S=tuple(2 + 3 * b for b in range(B)), d=8, Hq=2, Hk=1, h=4, V=V,
                    dtype="f32", max_steps=5, weight_seed=20 + V + C, canvas_seeds=tuple(30 + b for b in range(B)))
    _compare(cfg, adaptive)


@pytest.mark.parametrize("L,V,C,B,adaptive", [(2, 8, 6, 2, False), (3, 4, 5, 1, True), (2, 8, 4, 2, True)])
def test_multi_layer_small_cases(L, V, C, B, adaptive):
    """A stack of L layers (each attention + Wo + residual over its own prompt
    K/V, fed the previous layer's output) decodes identically in both
    implementations."""
    cfg = fx.Config(name="tinyl", B=B, C=C, S=tuple(2 + 3 * b for b in range(B)), d=8, Hq=2, Hk=1, h=4, V=V,
                    dtype="f32", max_steps=5, weight_seed=40 + L + V, canvas_seeds=tuple(50 + b for b in range(B)),
                    n_layers=L)
    _compare(cfg, adaptive)

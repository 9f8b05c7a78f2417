"""Full-size parity of the denoise path on the synthetic workloads, in the
launch configuration the benchmark uses (CUDA-graph steps through the C ABI),
against the fp64 oracle, stage by stage (tests/parity.py).

canvas256, vocab262k and moe are decoded to completion free-running (the GPU
keeps its own state for the whole block), with the adaptive stop off (the
full 48 steps) and on. Tokens, freeze sets, re-noise draws and step counts
must equal the oracle's except at decisions the oracle itself takes within
1e-3 of a tie; each report prints how many such decisions there were. The
tensor stages (Q/K/V, attention, Wo + residual, MoE) are compared on the first
three steps and the last; the LM head and the selection on every step.

longctx (four requests with 32K-token prompts) is compared on its first three
steps and on its last step (the GPU runs the 44 steps between on its own;
that step then starts from the GPU's state)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import model as om
from token_canvas_denoising_b200 import inputs as fx
from tests.oracle_adapter import oracle_model, oracle_prefix, oracle_sched
from tests.parity import abi_state_to_oracle, run_lockstep

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

_CACHE = {}


def _workload(name):
    """The seeded workload and the oracle model over it (dense weights widened
    to fp64 once), kept for the tests of the same workload."""
    if name not in _CACHE:
        _CACHE.clear()
        wl = fx.make_workload(fx.CONFIGS[name])
        _CACHE[name] = (wl, om.prewiden(oracle_model(wl)))
    return _CACHE[name]


def _decode(name, adaptive):
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.CONFIGS[name]
    wl, m = _workload(name)
    cv, keep = from_workload(wl)
    try:
        invT = None if cfg.inv_temp == "one" else wl.inv_temp.astype(np.float64)
        last = cfg.max_steps - 1
        rep, steps = run_lockstep(cfg, cv, m, oracle_prefix(wl), oracle_sched(cfg, adaptive=adaptive),
                                  schedule(cfg.max_steps, cfg.stop_entropy, adaptive), invT,
                                  free_running=True, check_tensors=True, tensor_steps={0, 1, 2, last})
        final = cv.get_state()
    finally:
        cv.close()
        del keep
        torch.cuda.empty_cache()
    print(f"{name} adaptive={adaptive}: {steps} steps; {rep.summary()}")
    assert not rep.errors, "\n".join(rep.errors[:20])
    assert np.all(final["done"]) and np.all(final["frozen"])
    assert np.array_equal(final["step"], rep.final_state["step"])
    if not adaptive:
        assert steps == cfg.max_steps and np.all(final["step"] == cfg.max_steps)
    else:
        assert 1 <= steps <= cfg.max_steps
    return rep, steps


@pytest.mark.parametrize("adaptive", [False, True])
def test_canvas256_full_decode(adaptive):
    _decode("canvas256", adaptive)


@pytest.mark.parametrize("adaptive", [False, True])
def test_vocab262k_full_decode(adaptive):
    _decode("vocab262k", adaptive)


@pytest.mark.parametrize("adaptive", [False, True])
def test_moe_full_decode(adaptive):
    _decode("moe", adaptive)


def test_longctx_first_steps_and_last_step():
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.CONFIGS["longctx"]
    wl, m = _workload("longctx")
    pre = oracle_prefix(wl)
    sched, osched = schedule(cfg.max_steps, cfg.stop_entropy, False), oracle_sched(cfg, adaptive=False)
    cv, keep = from_workload(wl)
    try:
        rep, steps = run_lockstep(cfg, cv, m, pre, osched, sched, None, n_steps=3, free_running=True)
        print(f"longctx first steps: {rep.summary()}")
        assert not rep.errors, "\n".join(rep.errors[:20])
        assert steps == 3
        for _ in range(3, cfg.max_steps - 1):
            cv.step(sched)
        st = abi_state_to_oracle(cv.get_state(), cfg.B, cfg.C)
        assert np.all(st["step"] == cfg.max_steps - 1) and not st["done"].any()
        rep2, steps2 = run_lockstep(cfg, cv, m, pre, osched, sched, None, n_steps=1, free_running=True, init=st)
        print(f"longctx last step: {rep2.summary()}")
        assert not rep2.errors, "\n".join(rep2.errors[:20])
        final = cv.get_state()
        assert steps2 == 1 and np.all(final["done"]) and np.all(final["frozen"])
        assert np.all(final["step"] == cfg.max_steps)
    finally:
        cv.close()
        del keep
        torch.cuda.empty_cache()

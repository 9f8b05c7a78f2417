"""Full-size parity of the denoise step on the large synthetic workloads, in the
launch configuration the benchmark uses (CUDA-graph steps through the C ABI),
against the fp64 oracle.

vocab262k: B1 C256 S4096 d2816 16/8 heads h128 V262144 with per-position
temperatures; longctx: four requests with 32K-token prompt prefixes each
(ragged-free, per-head scaled K/V). The first step is compared element-wise
(entropies, argmax, freeze sets, tokens, re-noise draws, attention output,
residual stream) under the ambiguity rules of tests/parity.py; the canvas256
workload is covered by the faster test in test_gpu_parity.py."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from token_canvas_denoising_b200 import inputs as fx
from tests.oracle_adapter import oracle_model, oracle_prefix, oracle_sched
from tests.parity import run_lockstep

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _run(name, n_steps):
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.CONFIGS[name]
    wl = fx.make_workload(cfg)
    cv, keep = from_workload(wl)
    try:
        invT = None if cfg.inv_temp == "one" else wl.inv_temp.astype(np.float64)
        rep, steps = run_lockstep(cfg, cv, oracle_model(wl), oracle_prefix(wl),
                                  oracle_sched(cfg, adaptive=True),
                                  schedule(cfg.max_steps, cfg.stop_entropy, True), invT,
                                  n_steps=n_steps, free_running=True, check_tensors=True)
    finally:
        cv.close()
        del keep
        torch.cuda.empty_cache()
    assert not rep.errors, "\n".join(rep.errors[:20])
    return rep


def test_vocab262k_first_steps():
    _run("vocab262k", 2)


def test_longctx_first_step():
    _run("longctx", 1)


def test_moe_first_step():
    _run("moe", 1)

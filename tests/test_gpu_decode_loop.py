"""The decode loop ends on the device: dg_decode_block is one graph launch
whose conditional while node repeats the step until the selection kernel finds
every canvas done, so a block that stops after k steps costs k steps (plus the
launch) and runs no step after the stop ("DiffusionGemma解析：扩散模型如何让LLM快5倍",
自适应停步机制: at most 48 steps, fewer when the canvas settles early).

On the canvas256 workload: a stop threshold above every entropy stops each
block after its first step (k = 1); without the adaptive stop the block runs
its whole schedule (k = 6 and k = 48). The loop must run exactly k steps (its
device-side counter), and its device time (events the decode graph records
just before and after the loop) must be at most (k + 0.2) times one step's
time, measured from back-to-back graph steps, plus 3 us per step for the
conditional node's turnaround between iterations (measured 1.3-2.2 us; a
step run after the stop would add a whole step to the count and to the time)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from token_canvas_denoising_b200 import inputs as fx

pytestmark = pytest.mark.gpu


def test_decode_block_runs_exactly_the_steps_it_needs():
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.CONFIGS["canvas256"]
    cv, keep = from_workload(fx.make_workload(cfg))
    stream = cv.stream
    try:
        step_sched = schedule(48, 0.05, False)
        for _ in range(5):
            cv.step(step_sched)
        cv.sync()
        n = 24
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cv.reset()
        e0.record(stream)
        for _ in range(n):
            cv.step(step_sched)
        e1.record(stream)
        torch.cuda.synchronize()
        t_step = e0.elapsed_time(e1) / n
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)  # torch creates the CUDA events on their first record
        d1.record(stream)
        cv.set_timing_events([d0], [d1], kernel="decode")
        cases = [(schedule(48, 100.0, True), 1), (schedule(6, 0.05, False), 6), (schedule(48, 0.05, False), 48)]
        for sched, k in cases:
            cv.reset()
            cv.decode(sched)  # builds the decode graph for this schedule
            cv.reset()
            toks, steps = cv.decode(sched)
            torch.cuda.synchronize()
            t = d0.elapsed_time(d1)
            st = cv.get_state()
            ran = cv.loop_steps()
            print(f"k={k}: loop ran {ran} steps, decode {t:.3f} ms, one step {t_step:.4f} ms, "
                  f"ratio {t / t_step:.2f}")
            assert ran == k
            assert steps == [k] and np.all(st["step"] == k) and np.all(st["done"]) and np.all(st["frozen"])
            assert np.array_equal(toks.numpy(), st["tokens"])
            assert t <= (k + 0.2) * t_step + k * 0.003, (k, t, t_step)
        cv.sync()
    finally:
        cv.close()

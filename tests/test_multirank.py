"""bench.py's multi-GPU host logic on CPU: two gloo ranks.

The canvases are independent requests, so N GPUs run N replicas with no
data-path collective: the only cross-rank steps are the timing all-reduce (the
job is as slow as its slowest rank), the whole-job rate (every rank's steps
over that time) and distinct canvas seeds per rank. The reference arm runs on
rank 0 alone."""
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_aggregate_like_bench():
    import torch.multiprocessing as mp
    from tests import multirank_worker as mw
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    elapsed = (3.0, 5.0)  # ms per rank
    procs = [ctx.Process(target=mw.worker, args=(r, 2, port, elapsed, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res = {r["rank"]: r for r in res}
    for r in (0, 1):
        assert res[r]["slowest"] == 5.0                       # max over ranks, on every rank
        assert res[r]["rate"] == pytest.approx(2 * 100 / 5e-3)  # both ranks' steps / slowest time
    assert not set(res[0]["seeds"]) & set(res[1]["seeds"])   # each replica decodes its own requests
    assert res[1]["ref_rc"] == 0 and res[1]["ref_out"] == ""  # only rank 0 prints the reference line


def test_single_rank_helpers_need_no_process_group():
    import bench
    assert bench.max_over_ranks(4.5, 1, "cpu") == 4.5
    assert bench.job_rate(48, 1, 2.0) == pytest.approx(24000.0)
    assert bench.rank_canvas_seeds((1, 2), 0) == (1, 2)

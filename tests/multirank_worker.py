"""One rank of the two-rank CPU test of bench.py's multi-GPU host logic (run
in a spawned process under the gloo backend)."""
import contextlib
import datetime
import io
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def worker(rank, world, port, elapsed_ms, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        slowest = bench.max_over_ranks(elapsed_ms[rank], world, "cpu")
        rate = bench.job_rate(100, world, slowest)
        seeds = bench.rank_canvas_seeds((7, 8, 9), rank)
        out = io.StringIO()
        ref_rc = None
        if rank != 0:  # the reference arm runs on rank 0 alone; the others exit 0 without work
            with contextlib.redirect_stdout(out):
                ref_rc = bench.bench_reference(None, rank, world)
        dist.barrier()
        q.put({"rank": rank, "slowest": slowest, "rate": rate, "seeds": seeds, "ref_rc": ref_rc,
               "ref_out": out.getvalue()})
    finally:
        dist.destroy_process_group()

"""The multi-rank host path of bench.py (world size 2, gloo, CPU): the timing
barrier, the max over ranks, the job aggregate, and the reference arm that
only rank 0 runs."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import bench
        bench.barrier(world)
        # each rank reports a different time; all of them get the slowest
        t = bench.max_over_ranks(0.25 + rank, world, torch.device("cpu"))
        v = bench.job_value(10.0, world)
        result = {"max": t, "value": v}
        if rank != 0:
            # the reference arm: ranks other than 0 exit at once, printing nothing
            import contextlib
            import io
            buf = io.StringIO()
            sys.argv = ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"]
            with contextlib.redirect_stdout(buf):
                bench.main()
            result["ref_out"] = buf.getvalue()
        bench.barrier(world)
        dist.destroy_process_group()
        q.put((rank, result))
    except Exception as e:  # reported to the parent, never swallowed
        q.put((rank, {"error": repr(e)}))


def test_two_ranks_share_max_time_and_aggregate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        assert "error" not in results[rank], results[rank]
        assert results[rank]["max"] == pytest.approx(1.25)
        assert results[rank]["value"] == pytest.approx(20.0)
    assert results[1]["ref_out"] == ""

"""bench.py's multi-rank plumbing on CPU: two gloo ranks (world size 2).

Covers what `bench.py --gpus N` does between ranks: process-group set-up from
the torchrun environment, the barrier, the max-over-ranks timing reduction,
the whole-job time per step, and the reference arm, where rank 0 alone
prints and the other ranks exit 0 without work.  The data path has no
collective, so nothing else crosses ranks.
"""

import io
import json
import multiprocessing as mp
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, ms_local: float, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    os.environ["OMP_NUM_THREADS"] = "1"
    sys.path.insert(0, ROOT)
    try:
        import torch.distributed as dist

        import bench
        r, wsz, local = bench.dist_setup(None)
        assert (r, wsz, local) == (rank, world, rank)
        assert dist.get_backend() == "gloo"
        bench.barrier(wsz)
        ms_max = bench.max_over_ranks(ms_local, wsz)
        value = bench.whole_job_us_per_step(ms_max, 10, wsz)
        args = bench.parse(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "0",
                                 "--gpus", str(world)])
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.run_reference(args)
        bench.barrier(wsz)
        dist.destroy_process_group()
        q.put((rank, ms_max, value, rc, buf.getvalue()))
    except BaseException as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e), None, ""))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [12.5, 20.0]  # device ms of each rank's timed steps
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times[r], q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in procs:
            rank, *rest = q.get(timeout=240)
            results[rank] = rest
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for rank in (0, 1):
        assert results[rank][0] != "error", results[rank]
        ms_max, value, rc, out = results[rank]
        assert ms_max == 20.0  # the slowest rank's time on every rank
        assert value == pytest.approx(20.0 * 1000.0 / (10 * 2))  # 20 steps in 20 ms: 1000 us per step
        assert rc == 0
    # the reference arm: rank 0 prints one JSON line, rank 1 nothing
    line = json.loads(results[0][3].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["unit"] == "us/step"
    assert line["config"]["workload"].startswith("tiny:")
    assert results[1][3] == ""

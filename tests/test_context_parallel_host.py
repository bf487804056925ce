"""Context-parallel verify plumbing on CPU: two gloo ranks all-gather their
(out, lse) partials, and merging them gives attention over the union of the
slices (checked with the fp64 oracle's combine and attention)."""

import multiprocessing as mp
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    try:
        import torch
        import torch.distributed as dist

        import oracle
        from speculative_decode_draft_b200.context_parallel import gather_partials
        dist.init_process_group("gloo")
        r = np.random.default_rng(5)
        n, D, rows = 40, 8, 3
        K, V, Q = r.standard_normal((n, D)), r.standard_normal((n, D)), r.standard_normal((rows, D))
        cuts = [0, 17, n]
        lo, hi = cuts[rank], cuts[rank + 1]
        o_l, l_l = oracle.attend_rows(Q, K[lo:hi], V[lo:hi], 0.5)      # this rank's slice
        po, pl = gather_partials(torch.from_numpy(o_l), torch.from_numpy(l_l))
        merged, lse = oracle.splitkv_combine(po.numpy(), pl.numpy())
        ref, ref_l = oracle.attend_rows(Q, K, V, 0.5)                    # the whole context
        dist.destroy_process_group()
        q.put((rank, tuple(po.shape), float(np.abs(merged - ref).max()), float(np.abs(lse - ref_l).max()),
               float(np.abs(po.numpy()[:, rank] - o_l).max())))
    except BaseException as e:
        q.put((rank, "error", repr(e), None, None))


def test_gather_partials_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = {}
    try:
        for _ in ps:
            rank, *rest = q.get(timeout=240)
            res[rank] = rest
    finally:
        for p in ps:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for rank in (0, 1):
        shape, err_o, err_l, own = res[rank]
        assert shape != "error", res[rank]
        assert shape == (3, 2, 8)        # [rows, world, D]
        assert own == 0.0                # this rank's partial sits in its own column
        assert err_o < 1e-12 and err_l < 1e-12

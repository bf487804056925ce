"""Context-parallel verify on one GPU: a sequence's context cut into slices,
each verified with wmtp_verify_attn_slice, merged with wmtp_splitkv_combine,
against the fp64 oracle's verify over the whole context.

The first test cuts contexts into page-aligned slices of one pool and runs
them one after the other on one device.  The last one runs the public entry
point, verify_attn_context_parallel, as two processes on cuda:0 whose
partials meet in one gloo all-gather, and compares both ranks' merged
results with the oracle's verify over the whole context.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import speculative_decode_draft_b200 as w
from speculative_decode_draft_b200.context_parallel import slice_query_positions

from _helpers import assert_close, assert_lse_close, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


def _slice_cache(kv, b_lens, starts, ends, P):
    """The pages of positions [start, end) of each sequence as their own cache."""
    B = len(b_lens)
    first = [s // P for s in starts]
    npg = max(-(-(e - s) // P) for s, e in zip(starts, ends))
    pt = torch.zeros(B, max(npg, 1), dtype=torch.int32, device=DEV)
    for b in range(B):
        n = -(-(ends[b] - starts[b]) // P)
        pt[b, :n] = kv.page_table[b, first[b]:first[b] + n]
    lens = torch.tensor([e - s for s, e in zip(starts, ends)], dtype=torch.int32, device=DEV)
    return w.PagedCache(kv.k_pool, kv.v_pool, pt, lens)


@pytest.mark.parametrize("D,G,P,num_q,lens,cuts", [
    (256, 8, 64, 4, [131076], [0, 32768, 65536, 131072]),          # last slice: the 4 queries only
    (256, 8, 64, 6, [49988, 20006], [0, 8192, 49984]),              # last slices: 4 tokens, and empty
    (64, 4, 16, 4, [3000], [0, 1024, 2048]),                        # the mma.sync verify path
    (256, 8, 64, 4, [1048580], [0, 262144, 524288, 786432]),       # 1M split four ways
])
def test_sliced_verify_merges_to_full_verify(D, G, P, num_q, lens, cuts):
    Hkv = 2
    B = len(lens)
    p = w.params(G * Hkv, Hkv, D, page_size=P, gamma_max=max(num_q - 1, 1))
    kv = synth.paged_kv(61, B, Hkv, D, P, lens, max(lens) + P, True, True, device=DEV)
    q = synth.queries(62, (B, num_q, G * Hkv, D), device=DEV)
    n_total = torch.tensor(lens, dtype=torch.int32, device=DEV)
    status = w.new_status(DEV)
    parts_o, parts_l = [], []
    for i, c in enumerate(cuts):
        starts = [min(c, n) for n in lens]
        ends = [min(cuts[i + 1], n) if i + 1 < len(cuts) else n for n in lens]
        cache = _slice_cache(kv, lens, starts, ends, P)
        q_pos0 = slice_query_positions(n_total, num_q, torch.tensor(starts, dtype=torch.int32, device=DEV))
        o, lse = w.verify_attn(p, q, cache, q_pos0=q_pos0, status=status)
        parts_o.append(o.reshape(-1, D))
        parts_l.append(lse.reshape(-1))
    part_o = torch.stack(parts_o, 1).contiguous()
    part_l = torch.stack(parts_l, 1).contiguous()
    out, lse = w.splitkv_combine(part_o, part_l)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kp, vp, pt, ln = f64(kv.k_pool), f64(kv.v_pool), kv.page_table.cpu().numpy(), np.asarray(lens)
    if max(lens) > 200000:  # one KV head at a time through the prefix oracle
        for b in range(B):
            for kvh in range(Hkv):
                pages = kv.page_table[b, :-(-lens[b] // P)].long()
                K = f64(kv.k_pool[pages, kvh].reshape(-1, D)[:lens[b]])
                V = f64(kv.v_pool[pages, kvh].reshape(-1, D)[:lens[b]])
                rows = slice(kvh * G, (kvh + 1) * G)
                qs = f64(q[b, :, rows]).reshape(num_q * G, D)
                L_ = np.repeat([lens[b] - num_q + i + 1 for i in range(num_q)], G)
                ref, ref_l = oracle.attend_prefixes(qs, K, V, L_, 1 / np.sqrt(D))
                got = f64(out.view(B, num_q, G * Hkv, D)[b, :, rows]).reshape(num_q * G, D)
                assert_close(got, ref, f"1M sliced verify b {b} kvh {kvh}")
        return
    ref, ref_lse = oracle.verify_attn(f64(q), kp, vp, pt, ln, P, 1 / np.sqrt(D))
    assert_close(f64(out).reshape(ref.shape), ref, f"sliced verify D={D} cuts={cuts}")
    assert_lse_close(f64(lse).reshape(ref_lse.shape), ref_lse, f"sliced verify lse cuts={cuts}")


def test_slice_after_a_query_gives_empty_rows():
    # a slice that starts after query 0's position: query 0 sees nothing there
    D, G, P, Hkv, num_q = 256, 8, 64, 2, 4
    n = 4096 + num_q
    p = w.params(G * Hkv, Hkv, D, page_size=P)
    kv = synth.paged_kv(63, 1, Hkv, D, P, [n], n + P, True, True, device=DEV)
    q = synth.queries(64, (1, num_q, G * Hkv, D), device=DEV)
    cache = _slice_cache(kv, [n], [4096], [n], P)
    q_pos0 = torch.tensor([n - num_q - 4096], dtype=torch.int32, device=DEV)  # query 0 at slice position 0
    o, lse = w.verify_attn(p, q, cache, q_pos0=q_pos0 - 1)  # as if the slice began one position later
    torch.cuda.synchronize()
    l = f64(lse)[0]
    assert np.all(np.isinf(l[0])) and np.all(l[0] < 0)      # query 0: position -1 of the slice, nothing
    assert np.all(np.isfinite(l[1:]))
    assert np.all(f64(o)[0, 0] == 0)


# ---------------------------------------------------------------- the public entry point, two ranks
def _cp_rank(rank, world, port, q):
    """One rank of a two-rank context-parallel verify on cuda:0: it holds
    positions [rank * n/2, (rank + 1) * n/2) of one 128K-token sequence in its
    own cache and calls verify_attn_context_parallel; the ranks' partials meet
    in one gloo all-gather.  The two processes share the GPU, but no kernel of
    one waits on the other: the exchange happens on the host."""
    import os
    import sys
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    try:
        import datetime

        import torch
        import torch.distributed as dist

        import synth
        import speculative_decode_draft_b200 as w
        from speculative_decode_draft_b200.context_parallel import verify_attn_context_parallel
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        D, G, Hkv, P, num_q, n = 256, 8, 2, 64, 4, 131076
        p = w.params(G * Hkv, Hkv, D, page_size=P, gamma_max=num_q - 1)
        kv = synth.paged_kv(71, 1, Hkv, D, P, [n], n + P, True, True, device="cuda:0")
        qv = synth.queries(72, (1, num_q, G * Hkv, D), device="cuda:0")
        cut = 65536  # page-aligned: rank 0 holds [0, 65536), rank 1 the rest (with the queries)
        lo, hi = (0, cut) if rank == 0 else (cut, n)
        npg = -(-(hi - lo) // P)
        local = w.PagedCache(kv.k_pool, kv.v_pool, kv.page_table[:, lo // P:lo // P + npg].contiguous(),
                             torch.tensor([hi - lo], dtype=torch.int32, device="cuda:0"))
        status = w.new_status("cuda:0")
        out, lse = verify_attn_context_parallel(
            p, qv, local, torch.tensor([lo], dtype=torch.int32, device="cuda:0"),
            torch.tensor([n], dtype=torch.int32, device="cuda:0"), status=status)
        torch.cuda.synchronize()
        dist.destroy_process_group()
        q.put((rank, int(status.item()), out.cpu().double().numpy(), lse.cpu().double().numpy()))
    except BaseException as e:  # report, never hang the parent
        q.put((rank, "error", repr(e), None))


@pytest.mark.timeout(600)
def test_verify_attn_context_parallel_two_ranks_match_the_oracle():
    import multiprocessing as mp
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_cp_rank, args=(r, 2, port, q)) for r in range(2)]
    for proc in ps:
        proc.start()
    res = {}
    try:
        for _ in ps:
            rank, *rest = q.get(timeout=480)
            res[rank] = rest
    finally:
        for proc in ps:
            proc.join(timeout=60)
            if proc.is_alive():
                proc.kill()
    for rank in (0, 1):
        assert res[rank][0] != "error", res[rank]
        assert res[rank][0] == 0, f"rank {rank}: device status {res[rank][0]:#x}"
    # the oracle over the whole context, from the same seeded inputs
    D, G, Hkv, P, num_q, n = 256, 8, 2, 64, 4, 131076
    kv = synth.paged_kv(71, 1, Hkv, D, P, [n], n + P, True, True, device=DEV)
    qv = synth.queries(72, (1, num_q, G * Hkv, D), device=DEV)
    lengths = np.repeat([len(oracle.causal_positions(n, num_q, i)) for i in range(num_q)], G)
    from _helpers import dense_kv_f64
    for kvh in range(Hkv):
        K, V = dense_kv_f64(kv, 0, n, kvh)
        rows = slice(kvh * G, (kvh + 1) * G)
        ref, ref_lse = oracle.attend_prefixes(f64(qv[0, :, rows]).reshape(num_q * G, D), K, V, lengths, 1 / 16)
        for rank in (0, 1):
            out, lse = res[rank][1], res[rank][2]
            assert_close(out[0, :, rows].reshape(num_q * G, D), ref, f"context parallel rank {rank} kvh {kvh}")
            assert_lse_close(lse[0, :, rows].reshape(-1), ref_lse, f"context parallel rank {rank} kvh {kvh}")

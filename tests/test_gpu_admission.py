"""Admission into one KV budget through the page allocator, then a decode step
of the admitted batch checked against the fp64 oracle.

Windowed-MTP's capacity claim (arxivlens view, Abstract): keeping the draft
layer's KV in a compact ring instead of a full paged cache frees that layer's
pool, which makes room for one more concurrent request.  Here one pool of
pages stands for the budget; requests are admitted through wmtp_pool_alloc
(all of a request's pages at once) until it refuses.  A native request takes
the pages of every paged layer (2 target + 1 draft); a windowed one the target
layers' pages plus pages worth its ring.  The budget is chosen so that the
native arm admits 2 requests and the windowed arm 3.  Each arm's batch is
then decoded through page tables taken from the allocator, over the one
shared pool: native draft attention and verify attention (native arm),
windowed draft attention over the rings and verify attention (windowed arm),
all compared with the oracle on the same pool and tables.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import speculative_decode_draft_b200 as w

from _helpers import assert_close, assert_lse_close, bits, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
Hq, Hkv, D, P, S, W, GAMMA, L, CTX = 16, 2, 256, 64, 4, 256, 3, 2, 8192


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


def test_ring_admits_one_more_request_and_the_batches_decode():
    p = w.params(Hq, Hkv, D, page_size=P, sinks=S, window=W, gamma_max=GAMMA)
    page_bytes = 2 * Hkv * P * D * 2
    num_pages = 800
    budget = num_pages * page_bytes
    plan = {arm: w.plan_admission(p, CTX, L, 1, arm == "windowed", budget) for arm in ("native", "windowed")}
    pages_layer = plan["native"]["pages_per_layer"]
    assert pages_layer == -(-(CTX + GAMMA + 1) // P)
    ring_pages = -(-plan["windowed"]["draft_bytes"] // page_bytes)
    need = {"native": (L + 1) * pages_layer, "windowed": L * pages_layer + ring_pages}

    gen = torch.Generator(device=DEV).manual_seed(90)
    k_pool = torch.randn(num_pages, Hkv, P, D, generator=gen, device=DEV).to(torch.bfloat16)
    v_pool = torch.randn(num_pages, Hkv, P, D, generator=gen, device=DEV).to(torch.bfloat16)
    kp, vp = f64(k_pool), f64(v_pool)
    pool = w.PagePool(num_pages)
    status = w.new_status(DEV)
    counts = {}
    for arm in ("native", "windowed"):
        admitted = []
        while True:
            try:
                admitted.append(pool.alloc(need[arm]))
            except w.WmtpError:
                break
        counts[arm] = len(admitted)
        B = len(admitted)
        used = np.concatenate([np.asarray(r) for r in admitted])
        assert len(np.unique(used)) == used.size and used.min() >= 0 and used.max() < num_pages
        assert pool.free_count == num_pages - B * need[arm]

        def table(l):
            return torch.tensor([r[l * pages_layer:(l + 1) * pages_layer] for r in admitted], dtype=torch.int32,
                                device=DEV)
        # verify layer 1 of every admitted request (queries at CTX .. CTX+3)
        n_ver = CTX + GAMMA + 1
        tv = table(1)
        cache = w.PagedCache(k_pool, v_pool, tv, torch.full((B,), n_ver, dtype=torch.int32, device=DEV))
        qv = synth.queries(91 + B, (B, GAMMA + 1, Hq, D), device=DEV)
        out, lse = w.verify_attn(p, qv, cache, status=status)
        ref, ref_lse = oracle.verify_attn(f64(qv), kp, vp, tv.cpu().numpy(), np.full(B, n_ver), P, 1 / 16)
        assert_close(f64(out), ref, f"{arm} verify")
        assert_lse_close(f64(lse), ref_lse, f"{arm} verify")
        qd = synth.queries(95 + B, (B, Hq, D), device=DEV)
        if arm == "native":
            # the draft layer's pages: its token at position CTX
            td = table(L)
            dc = w.PagedCache(k_pool, v_pool, td, torch.full((B,), CTX + 1, dtype=torch.int32, device=DEV))
            out, lse = w.draft_attn_full(p, qd, dc, status=status)
            ref, ref_lse = oracle.draft_attn_full(f64(qd), kp, vp, td.cpu().numpy(), np.full(B, CTX + 1), P,
                                                  1 / 16)
            assert_close(f64(out), ref, "native draft")
            assert_lse_close(f64(lse), ref_lse, "native draft")
        else:
            # the ring holds the draft layer's sink and window: history of
            # CTX + 1 seeded tokens per request
            kd, vd = synth.new_tokens(97, B, CTX + 1, Hkv, D, device=DEV)
            ring = w.Ring.allocate(p, B, DEV)
            w.ring_append(p, ring, kd, vd, torch.full((B,), CTX + 1, dtype=torch.int32, device=DEV),
                          status=status)
            out, lse = w.draft_attn_windowed(p, qd, ring, status=status)
            models = []
            for b in range(B):
                m = oracle.RingModel(S, W, GAMMA, Hkv, D)
                m.call(-1, bits(kd[b]), bits(vd[b]), False)
                models.append(m)
            ref, ref_lse = oracle.draft_attn_windowed(f64(qd), models, 1 / 16)
            assert_close(f64(out), ref, "windowed draft")
            assert_lse_close(f64(lse), ref_lse, "windowed draft")
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for r in admitted:
            pool.release(r)
        assert pool.free_count == num_pages
    assert counts == {"native": plan["native"]["max_requests"], "windowed": plan["windowed"]["max_requests"]}
    assert counts["windowed"] == counts["native"] + 1 == 3

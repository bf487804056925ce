"""GPU: the bounded in-kernel wait gives up, reports, and leaves the context usable.

Every mbarrier wait in the attention kernels is bounded: after a fixed number
of SM clocks it stops, sets WMTP_DEV_TIMEOUT in the status word and lets the
kernel return.  ``wmtp_selftest_wait`` runs that same wait on a barrier that
nothing completes.  The wait is bounded, so nothing here can hang the GPU.
"""

import time

import numpy as np
import pytest
import torch

import oracle
import synth
import speculative_decode_draft_b200 as w
from speculative_decode_draft_b200 import _lib as L

from _helpers import assert_close, cache_of, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


def test_completed_wait_sets_nothing():
    status = w.new_status(DEV)
    cycles = torch.full((1,), -1, dtype=torch.int64, device=DEV)
    w.selftest_wait(True, status=status, cycles=cycles)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert 0 <= int(cycles.item()) < 1_000_000


def test_wait_nothing_completes_gives_up_then_context_works():
    status = w.new_status(DEV)
    cycles = torch.zeros(1, dtype=torch.int64, device=DEV)
    t0 = time.perf_counter()
    w.selftest_wait(False, status=status, cycles=cycles)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    assert int(status.item()) == L.DEV_TIMEOUT
    c = int(cycles.item())
    # it waited the whole limit, and stopped soon after it
    assert L.WAIT_LIMIT_CYCLES < c < L.WAIT_LIMIT_CYCLES + 200_000_000, c
    assert wall < 15.0, wall

    # the same context still runs an attention call correctly
    Hq, Hkv, D, P, n = 16, 2, 256, 64, 3000
    p = w.params(Hq, Hkv, D, page_size=P, sinks=4, window=256, gamma_max=8)
    kv = synth.paged_kv(11, 1, Hkv, D, P, [n], n + 70, True, True, device=DEV)
    q = synth.queries(111, (1, Hq, D), device=DEV)
    st2 = w.new_status(DEV)
    out, _ = w.draft_attn_full(p, q, cache_of(kv), status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    ref, _ = oracle.draft_attn_full(f64(q), f64(kv.k_pool), f64(kv.v_pool), kv.page_table.cpu().numpy(),
                                    kv.kv_len.cpu().numpy(), P, 1 / np.sqrt(D))
    assert_close(f64(out), ref, "draft full after a timed-out wait")

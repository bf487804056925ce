"""The windowed draft's time does not depend on the context length.

Windowed-MTP bounds the draft's KV working set to the sink plus the window
whatever the context (readpriors post, What happened: a working set that
stays the same size at any context; arxivlens view, Abstract).  The ring
holds S + W entries at every length, so the windowed draft attention must
take the same time at 32K, 128K and 1M tokens of context: within +-10% of
the median of the three (device time of calls replayed from a CUDA graph).
The native draft over the paged cache, for contrast, grows with the context.
"""

import statistics

import pytest
import torch

import speculative_decode_draft_b200 as w
from speculative_decode_draft_b200.timing import fill_ring_to, graph_call_us

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("window", [2048, 4096])
def test_windowed_draft_time_is_flat_in_context(window):
    p = w.params(16, 2, 256, page_size=64, sinks=4, window=window, gamma_max=3)
    q = torch.randn(1, 16, 256, device=DEV).to(torch.bfloat16)
    out = torch.empty(1, 16, 256, dtype=torch.float32, device=DEV)
    lse = torch.empty(1, 16, dtype=torch.float32, device=DEV)
    ws = torch.empty(w.workspace_bytes("windowed", p, 1), dtype=torch.uint8, device=DEV)
    status = w.new_status(DEV)
    rings = {}
    for ctx in (32768, 131072, 1048576):
        rings[ctx] = w.Ring.allocate(p, 1, DEV)
        fill_ring_to(p, rings[ctx], ctx, seed=ctx, device=DEV)
        assert int(rings[ctx].len.item()) == ctx
    # two interleaved rounds, the better time per context (the first
    # measurement of a series can run slower whichever context it is)
    times = {}
    for _ in range(2):
        for ctx, ring in rings.items():
            t = graph_call_us(lambda: w.draft_attn_windowed(p, q, ring, out=out, lse=lse, workspace=ws,
                                                             status=status))
            times[ctx] = min(t, times.get(ctx, float("inf")))
    del rings
    assert int(status.item()) == 0
    mid = statistics.median(times.values())
    for ctx, t in times.items():
        assert abs(t - mid) <= 0.10 * mid, f"windowed draft {t:.2f} us at {ctx} tokens vs median {mid:.2f} us: {times}"

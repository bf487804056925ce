"""Device-side timing helpers shared by the tests and the benchmark.

CUDA-event timing of calls replayed from a captured CUDA graph, on the
stream that launches them.  Nothing here computes any part of the attention
path.
"""

from __future__ import annotations

import statistics

import torch


def graph_call_us(fn, calls: int = 10, repeats: int = 7) -> float:
    """Median device time of one ``fn()`` in microseconds: ``calls`` calls are
    captured in one CUDA graph, replayed once to warm up, then ``repeats``
    times between CUDA events; each replay's time is divided by ``calls``."""
    fn()  # first call outside the capture (kernel attributes, module loading)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(calls):
            fn()
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1000.0 / calls)
    del g
    return statistics.median(times)


def fill_ring_to(p, ring, length: int, seed: int, device, chunk: int = 65536) -> None:
    """Append ``length`` random tokens to every (empty) ring of ``ring``, in
    chunks; only the sink and window survivors are written.  Used to put a
    ring in the state it has at a given context length."""
    from .api import ring_append
    B = ring.batch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    done = 0
    while done < length:
        n = min(chunk, length - done)
        shape = (B, n, p.num_heads_kv, p.head_dim)
        k = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
        v = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
        ring_append(p, ring, k, v, torch.full((B,), n, dtype=torch.int32, device=device))
        done += n

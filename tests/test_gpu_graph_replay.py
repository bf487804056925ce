"""One decode step captured as a CUDA graph replays bit-identically to the
same step launched eagerly.

The bench times steps as graph replays, and the attention kernels are
launched as programmatic dependents of the previous stream work; this checks
that the captured dependencies (ring append -> windowed draft, paged write ->
verify, attention -> combine, and the verify that writes its own new tokens)
order the work exactly as stream order does.
"""

import pytest
import torch

import synth
import speculative_decode_draft_b200 as w

from _helpers import cache_of

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


def test_graph_replay_matches_eager_step():
    wl = synth.workload("32k")
    n0, Hq, Hkv, D, P = wl.context[0], wl.num_heads_q, wl.num_heads_kv, wl.head_dim, wl.page_size
    gamma, S, W = 3, wl.sinks, 256
    p = w.params(Hq, Hkv, D, page_size=P, sinks=S, window=W, gamma_max=gamma)
    cap = n0 + 2 * (gamma + 1) + P
    i32 = dict(dtype=torch.int32, device=DEV)
    draft = synth.paged_kv(21, 1, Hkv, D, P, [n0], cap, True, True, device=DEV)
    ver = synth.paged_kv(22, 1, Hkv, D, P, [n0], cap, True, True, device=DEV)
    ver2 = synth.paged_kv(27, 1, Hkv, D, P, [n0], cap, True, True, device=DEV)
    dcache, vcache, vcache2 = cache_of(draft), cache_of(ver), cache_of(ver2)
    ring = w.Ring.allocate(p, 1, DEV)
    k, v = synth.dense_from_paged(draft, 0, n0)
    w.ring_append(p, ring, k[None].contiguous(), v[None].contiguous(), torch.tensor([n0], **i32))
    kd, vd = synth.new_tokens(23, 1, gamma, Hkv, D, device=DEV, kv_scale=True)
    kv_, vv_ = synth.new_tokens(24, 1, gamma + 1, Hkv, D, device=DEV, kv_scale=True)
    qd = synth.queries(25, (gamma, 1, Hq, D), device=DEV)
    qv = synth.queries(26, (1, gamma + 1, Hq, D), device=DEV)
    one = torch.ones(1, **i32)
    pos_d = torch.arange(gamma, **i32).view(gamma, 1) + n0
    len_d = pos_d + 1
    pos_v = torch.tensor([n0], **i32)
    len_v = pos_v + gamma + 1
    trunc = torch.tensor([n0 + 1], **i32)  # accept one token: roll back two drafts
    none = torch.zeros(1, **i32)
    status = w.new_status(DEV)
    o_w = torch.empty(gamma, 1, Hq, D, dtype=torch.float32, device=DEV)
    o_n = torch.empty_like(o_w)
    l_w = torch.empty(gamma, 1, Hq, dtype=torch.float32, device=DEV)
    l_n = torch.empty_like(l_w)
    o_v = torch.empty(1, gamma + 1, Hq, D, dtype=torch.float32, device=DEV)
    l_v = torch.empty(1, gamma + 1, Hq, dtype=torch.float32, device=DEV)
    o_v2, l_v2 = torch.empty_like(o_v), torch.empty_like(l_v)
    ws = torch.empty(max(w.workspace_bytes("full", p, 1, max_pages=draft.max_pages),
                         w.workspace_bytes("verify", p, 1, num_q=gamma + 1, max_pages=ver.max_pages),
                         w.workspace_bytes("windowed", p, 1)), dtype=torch.uint8, device=DEV)

    def step():
        for j in range(gamma):
            w.ring_append(p, ring, kd[:, j:j + 1], vd[:, j:j + 1], one, speculative=True, status=status)
            w.draft_attn_windowed(p, qd[j], ring, out=o_w[j], lse=l_w[j], workspace=ws, status=status)
            w.paged_write(p, dcache, pos_d[j], kd[:, j:j + 1].contiguous(), vd[:, j:j + 1].contiguous(),
                          status=status)
            dcache.kv_len = len_d[j]
            w.draft_attn_full(p, qd[j], dcache, out=o_n[j], lse=l_n[j], workspace=ws, status=status)
        w.paged_write(p, vcache, pos_v, kv_, vv_, status=status)
        vcache.kv_len = len_v
        w.verify_attn(p, qv, vcache, out=o_v, lse=l_v, workspace=ws, status=status)
        # a second layer with the append fused into the verify call (rewriting
        # the same rows on replay leaves the pool unchanged)
        vcache2.kv_len = len_v
        w.verify_attn_append(p, qv, kv_, vv_, vcache2, out=o_v2, lse=l_v2, workspace=ws, status=status)
        w.ring_append(p, ring, kd[:, :1], vd[:, :1], none, truncate_to=trunc, status=status)

    snap = [t.clone() for t in (ring.k, ring.v, ring.tags, ring.len, ring.committed)]
    step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    eager = [t.clone() for t in (o_w, l_w, o_n, l_n, o_v, l_v, o_v2, l_v2, ring.k, ring.v, ring.tags, ring.len,
                                 ring.committed)]
    for dst, src in zip((ring.k, ring.v, ring.tags, ring.len, ring.committed), snap):
        dst.copy_(src)
    for t in (o_w, l_w, o_n, l_n, o_v, l_v, o_v2, l_v2):
        t.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    replay = (o_w, l_w, o_n, l_n, o_v, l_v, o_v2, l_v2, ring.k, ring.v, ring.tags, ring.len, ring.committed)
    for name, a, b in zip(("windowed out", "windowed lse", "native out", "native lse", "verify out",
                           "verify lse", "fused verify out", "fused verify lse", "ring k", "ring v", "ring tags",
                           "ring len", "ring committed"),
                          eager, replay):
        assert torch.equal(a, b), f"graph replay differs from eager launches: {name}"

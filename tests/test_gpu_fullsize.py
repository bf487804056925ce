"""GPU parity at the benchmark's full sizes, on sampled outputs.

The 128K and 1M configurations run in the launch configuration the bench
times (batch 1, 16 query / 2 KV heads, head_dim 256, page 64, shuffled pages,
per-KV-head scales; the same parameters, hence the same split plan): every
head of the native and windowed draft and verify layers 0 and 9 are checked
against the fp64 oracle.  The ragged four-sequence workload runs 512 decode
steps of drafts, ring appends, verify and accept/rollback: the ring is
compared bit for bit after every step, attention on sampled steps.

Oracle inputs never come from the kernels: the KV history is regathered from
a pool regenerated from its seed (never written by the library) plus a host
record of the tokens the test appended.  Nothing here needs the whole pool in
fp64; one sequence and KV head at a time is widened on the host.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import speculative_decode_draft_b200 as w

from _helpers import assert_close, assert_lse_close, bits, cache_of, dense_kv_f64, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


def _check_draft_rows(out, lse, q, K, V, lengths, G, kvh, what):
    """Heads kvh*G .. kvh*G+G-1 of a [Hq, D] output against prefixes of K/V."""
    rows = slice(kvh * G, (kvh + 1) * G)
    ref, ref_lse = oracle.attend_prefixes(f64(q[rows]), K, V, lengths, 1 / 16)
    assert_close(f64(out[rows]), ref, what)
    assert_lse_close(f64(lse[rows]), ref_lse, what)


def _check_verify(out, lse, qv, K, V, n_total, G, kvh, what):
    """All queries and heads of one KV head of a verify block [Qn, Hq, D]."""
    Qn = qv.shape[0]
    rows = slice(kvh * G, (kvh + 1) * G)
    qs = f64(qv[:, rows]).reshape(Qn * G, -1)
    lengths = np.repeat([len(oracle.causal_positions(n_total, Qn, i)) for i in range(Qn)], G)
    ref, ref_lse = oracle.attend_prefixes(qs, K, V, lengths, 1 / 16)
    assert_close(f64(out[:, rows]).reshape(Qn * G, -1), ref, what)
    assert_lse_close(f64(lse[:, rows]).reshape(-1), ref_lse, what)


def _windowed_ref(q, K, V, length, S, W, G, kvh):
    pos = oracle.window_positions(length, S, W)
    rows = f64(q[kvh * G:(kvh + 1) * G])
    return oracle.attend_rows(rows, K[pos], V[pos], 1 / 16)


# ---------------------------------------------------------------- 128K / 1M
@pytest.mark.timeout(1200)
@pytest.mark.parametrize("name,gamma,window", [("128k", 3, 2048), ("1m", 3, 4096), ("1m", 5, 1024),
                                               ("1m", 8, 4096)])
def test_fullsize_sampled(name, gamma, window):
    wl = synth.workload(name)
    n0, Hq, Hkv, D, P, S = wl.context[0], wl.num_heads_q, wl.num_heads_kv, wl.head_dim, wl.page_size, wl.sinks
    G = Hq // Hkv
    p = w.params(Hq, Hkv, D, page_size=P, sinks=S, window=window, gamma_max=gamma)
    cap = n0 + gamma + 2 + P
    status = w.new_status(DEV)

    # draft layer: the draft token sits at position n0 (kv_len = n0 + 1)
    draft = synth.paged_kv(wl.seed + 5, 1, Hkv, D, P, [n0 + 1], cap, wl.kv_scale, wl.shuffle_pages, device=DEV)
    q = synth.queries(wl.seed + 200, (1, Hq, D), device=DEV)
    out_n, lse_n = w.draft_attn_full(p, q, cache_of(draft), status=status)
    ring = w.Ring.allocate(p, 1, DEV)
    kd, vd = synth.dense_from_paged(draft, 0, n0 + 1)
    w.ring_append(p, ring, kd[None].contiguous(), vd[None].contiguous(),
                  torch.tensor([n0 + 1], dtype=torch.int32, device=DEV), status=status)
    del kd, vd
    out_w, lse_w = w.draft_attn_windowed(p, q, ring, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for kvh in range(Hkv):
        K, V = dense_kv_f64(draft, 0, n0 + 1, kvh)
        _check_draft_rows(out_n[0], lse_n[0], q[0], K, V, [n0 + 1] * G, G, kvh, f"{name} native draft kvh {kvh}")
        ref, ref_lse = _windowed_ref(q[0], K, V, n0 + 1, S, window, G, kvh)
        rows = slice(kvh * G, (kvh + 1) * G)
        assert_close(f64(out_w[0, rows]), ref, f"{name} windowed draft kvh {kvh}")
        assert_lse_close(f64(lse_w[0, rows]), ref_lse, f"{name} windowed draft kvh {kvh}")
        del K, V
    del draft, ring

    # verify layers 0 and 9 (independent KV; the gamma+1 new tokens are the
    # pool's contents at n0 .. n0+gamma)
    Qn = gamma + 1
    for layer in (0, 9):
        kv = synth.paged_kv(wl.seed + 10 + layer, 1, Hkv, D, P, [n0 + Qn], cap, wl.kv_scale, wl.shuffle_pages,
                            device=DEV)
        qv = synth.queries(wl.seed + 300 + layer, (1, Qn, Hq, D), device=DEV)
        out_v, lse_v = w.verify_attn(p, qv, cache_of(kv), status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for kvh in range(Hkv):
            K, V = dense_kv_f64(kv, 0, n0 + Qn, kvh)
            _check_verify(out_v[0], lse_v[0], qv[0], K, V, n0 + Qn, G, kvh, f"{name} verify layer {layer} kvh {kvh}")
            del K, V
        del kv


# ---------------------------------------------------------------- ragged4
class _History:
    """Host record of one layer's appended tokens, over a pool regenerated
    from its seed for the committed prefix."""

    def __init__(self, seed, wl, n0, cap):
        self.seed, self.wl, self.n0, self.cap = seed, wl, list(n0), cap
        self.tokens = [dict() for _ in n0]  # position -> (k [Hkv, D], v) bf16 on the host

    def write(self, b, pos, k, v):
        for j in range(k.shape[0]):
            self.tokens[b][pos + j] = (k[j].clone(), v[j].clone())

    def dense(self, pristine, b, length, kvh):
        n0 = self.n0[b]
        K, V = dense_kv_f64(pristine, b, min(length, n0), kvh)
        if length > n0:
            extra_k = np.stack([f64(self.tokens[b][t][0][kvh]) for t in range(n0, length)])
            extra_v = np.stack([f64(self.tokens[b][t][1][kvh]) for t in range(n0, length)])
            K, V = np.concatenate([K, extra_k]), np.concatenate([V, extra_v])
        return K, V

    def pristine(self):
        wl = self.wl
        return synth.paged_kv(self.seed, wl.batch, wl.num_heads_kv, wl.head_dim, wl.page_size, self.n0,
                              self.cap, wl.kv_scale, wl.shuffle_pages, device=DEV)


def _oracle_ring(S, W, gmax, Hkv, D, hist_k_bits, hist_v_bits, n0):
    """RingModel after appending positions 0 .. n0-1 in order.  Positions the
    ring no longer holds at n0 (S <= p < n0 - W) are later overwritten by
    p + W, so their values cannot reach the final state; they are appended
    as zeros to keep the setup fast.  ``hist_*_bits[p]`` is given for the
    surviving positions only (a dict)."""
    r = oracle.RingModel(S, W, gmax, Hkv, D)
    zero = np.zeros((Hkv, D), dtype=np.uint16)
    for pos in range(n0):
        if pos in hist_k_bits:
            r.append_one(hist_k_bits[pos], hist_v_bits[pos], False)
        else:
            r.append_one(zero, zero, False)
    r.commit()
    return r


def _ring_equal(ring, models, what):
    tags = ring.tags.cpu().numpy()
    ln = ring.len.cpu().numpy()
    cm = ring.committed.cpu().numpy()
    kb = bits(ring.k).transpose(0, 2, 1, 3)  # [B, S+W, Hkv, D]
    vb = bits(ring.v).transpose(0, 2, 1, 3)
    for b, m in enumerate(models):
        assert ln[b] == m.length and cm[b] == m.committed, f"{what}: len/committed of sequence {b}"
        assert np.array_equal(tags[b], m.tags()), f"{what}: tags of sequence {b}"
        assert np.array_equal(kb[b], m.k_array()) and np.array_equal(vb[b], m.v_array()), \
            f"{what}: ring K/V bytes of sequence {b}"


@pytest.mark.timeout(3000)
def test_ragged4_decode_steps():
    wl = synth.workload("ragged4")
    B, Hq, Hkv, D, P, S, W, gamma = (wl.batch, wl.num_heads_q, wl.num_heads_kv, wl.head_dim, wl.page_size,
                                     wl.sinks, wl.window, wl.gamma)
    G = Hq // Hkv
    n0 = np.array(wl.context, dtype=np.int64)
    steps = wl.steps
    p = w.params(Hq, Hkv, D, page_size=P, sinks=S, window=W, gamma_max=gamma)
    cap = int(n0.max()) + steps * (gamma + 1) + P
    status = w.new_status(DEV)
    i32 = dict(dtype=torch.int32, device=DEV)

    draft_hist = _History(wl.seed + 5, wl, n0, cap)
    ver_hist = _History(wl.seed + 10, wl, n0, cap)
    draft = draft_hist.pristine()
    ver = ver_hist.pristine()
    dcache, vcache = cache_of(draft), cache_of(ver)

    # rings filled with each sequence's committed history
    ring = w.Ring.allocate(p, B, DEV)
    w.ring_reset(p, ring)
    mx = int(n0.max())
    hk = torch.zeros(B, mx, Hkv, D, dtype=torch.bfloat16, device=DEV)
    hv = torch.zeros_like(hk)
    models = []
    for b in range(B):
        k, v = synth.dense_from_paged(draft, b, int(n0[b]))
        hk[b, :n0[b]].copy_(k)
        hv[b, :n0[b]].copy_(v)
        keep = list(range(min(S, n0[b]))) + list(range(max(S, n0[b] - W), n0[b]))
        kb, vb = bits(k[keep]), bits(v[keep])
        models.append(_oracle_ring(S, W, gamma, Hkv, D, dict(zip(keep, kb)), dict(zip(keep, vb)), int(n0[b])))
        del k, v
    w.ring_append(p, ring, hk, hv, torch.as_tensor(n0, **i32), status=status)
    del hk, hv
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _ring_equal(ring, models, "initial fill")

    accept = synth.accept_counts(wl.seed, steps, B, gamma)
    rng = np.random.default_rng(wl.seed + 31)
    sample = {0, 1, steps // 2 - 1, steps - 1} | set(int(x) for x in rng.choice(np.arange(2, steps - 1), 2, False))
    n = n0.copy()
    out_n = [torch.empty(B, Hq, D, dtype=torch.float32, device=DEV) for _ in range(gamma)]
    lse_n = [torch.empty(B, Hq, dtype=torch.float32, device=DEV) for _ in range(gamma)]
    out_w = [torch.empty_like(o) for o in out_n]
    lse_w = [torch.empty_like(l) for l in lse_n]
    one = torch.ones(B, **i32)
    for s in range(steps):
        check = s in sample
        kd, vd = synth.new_tokens(wl.seed * 1000 + 3 * s, B, gamma, Hkv, D, device=DEV, kv_scale=True)
        kv_, vv_ = synth.new_tokens(wl.seed * 1000 + 3 * s + 1, B, gamma + 1, Hkv, D, device=DEV, kv_scale=True)
        kbn, vbn = synth.new_tokens(wl.seed * 1000 + 3 * s + 2, B, 1, Hkv, D, device=DEV, kv_scale=True)
        qd = synth.queries(wl.seed * 1000 + 7 * s, (gamma, B, Hq, D), device=DEV)
        qv = synth.queries(wl.seed * 1000 + 7 * s + 1, (B, gamma + 1, Hq, D), device=DEV)
        n_t = torch.as_tensor(n, **i32)
        kd_h, vd_h = kd.cpu(), vd.cpu()
        for j in range(gamma):
            # windowed arm: speculative ring append, then attention over the ring
            w.ring_append(p, ring, kd[:, j:j + 1].contiguous(), vd[:, j:j + 1].contiguous(), one,
                          speculative=True, status=status)
            for b in range(B):
                models[b].call(-1, bits(kd_h[b, j:j + 1]), bits(vd_h[b, j:j + 1]), True)
            w.draft_attn_windowed(p, qd[j], ring, out=out_w[j], lse=lse_w[j], status=status)
            # native arm: the same token into the draft layer's pages
            w.paged_write(p, dcache, n_t + j, kd[:, j:j + 1].contiguous(), vd[:, j:j + 1].contiguous(), status=status)
            for b in range(B):
                draft_hist.write(b, int(n[b]) + j, kd_h[b, j:j + 1], vd_h[b, j:j + 1])
            if check:
                dcache.kv_len = n_t + j + 1
                w.draft_attn_full(p, qd[j], dcache, out=out_n[j], lse=lse_n[j], status=status)
        # verify layer: gamma+1 new tokens, causal attention over the full pages
        w.paged_write(p, vcache, n_t, kv_, vv_, status=status)
        kvh_, vvh_ = kv_.cpu(), vv_.cpu()
        for b in range(B):
            ver_hist.write(b, int(n[b]), kvh_[b], vvh_[b])
        vcache.kv_len = n_t + gamma + 1
        out_v, lse_v = w.verify_attn(p, qv, vcache, status=status)
        # accept a in 1..gamma+1: roll the ring back, append the bonus token
        a = accept[s].astype(np.int64)
        trunc = torch.as_tensor(n + np.minimum(a, gamma), **i32)
        nb = torch.as_tensor((a == gamma + 1).astype(np.int32), **i32)
        w.ring_append(p, ring, kbn, vbn, nb, truncate_to=trunc, status=status)
        kbn_h, vbn_h = kbn.cpu(), vbn.cpu()
        for b in range(B):
            take = 1 if a[b] == gamma + 1 else 0
            models[b].call(int(n[b] + min(a[b], gamma)), bits(kbn_h[b, :take]), bits(vbn_h[b, :take]), False)
        # the bonus token also goes into the draft layer's pages at n+gamma, for
        # every sequence: where it was not accepted (a <= gamma) that position
        # lies past the new length n+a and the next step's drafts overwrite it
        # (at draft gamma-a) before any draft attends it
        w.paged_write(p, dcache, torch.as_tensor(n + gamma, **i32), kbn, vbn, status=status)
        for b in range(B):
            draft_hist.write(b, int(n[b]) + gamma, kbn_h[b], vbn_h[b])
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"device status {int(status.item()):#x} at step {s}"
        _ring_equal(ring, models, f"step {s}")

        if check:
            pd, pv = draft_hist.pristine(), ver_hist.pristine()
            for b in range(B):
                for kvh in range(Hkv):
                    K, V = draft_hist.dense(pd, b, int(n[b]) + gamma, kvh)
                    for j in range(gamma):
                        L_ = int(n[b]) + j + 1
                        _check_draft_rows(out_n[j][b], lse_n[j][b], qd[j, b], K, V, [L_] * G, G, kvh,
                                          f"step {s} seq {b} native draft {j} kvh {kvh}")
                        ref, ref_lse = _windowed_ref(qd[j, b], K[:L_], V[:L_], L_, S, W, G, kvh)
                        rows = slice(kvh * G, (kvh + 1) * G)
                        assert_close(f64(out_w[j][b, rows]), ref, f"step {s} seq {b} windowed draft {j} kvh {kvh}")
                        assert_lse_close(f64(lse_w[j][b, rows]), ref_lse, f"step {s} seq {b} windowed {j}")
                    del K, V
                    K, V = ver_hist.dense(pv, b, int(n[b]) + gamma + 1, kvh)
                    _check_verify(out_v[b], lse_v[b], qv[b], K, V, int(n[b]) + gamma + 1, G, kvh,
                                  f"step {s} seq {b} verify kvh {kvh}")
                    del K, V
            del pd, pv
        n = n + a

"""GPU parity: every C-ABI call against the fp64 CPU oracle.

Floating-point outputs (fp32 output mode) must be within max-abs 2e-3 and
relative L2 1e-3 of the oracle; the bf16 output mode must equal the fp32
result rounded to bf16, bit for bit; ring state and paged writes bit-exact.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import speculative_decode_draft_b200 as w
from speculative_decode_draft_b200 import _lib as L

from _helpers import (assert_close, assert_lse_close, bits, bf16_ulp_diff, cache_of, f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


DEV = "cuda:0"


def _params(Hq, Hkv, D, P, S=4, W=256, gmax=8):
    return w.params(Hq, Hkv, D, page_size=P, sinks=S, window=W, gamma_max=gmax)


def _paged(seed, B, Hkv, D, P, lens, scale=True, shuffle=True, capacity=None):
    cap = capacity or max(max(lens), 1) + 70
    return synth.paged_kv(seed, B, Hkv, D, P, lens, cap, scale, shuffle, device=DEV)


def _oracle_pools(kv):
    return f64(kv.k_pool), f64(kv.v_pool), kv.page_table.cpu().numpy(), kv.kv_len.cpu().numpy()


# ---------------------------------------------------------------- native draft
@pytest.mark.parametrize("name", ["tiny", "32k"])
def test_draft_full_workloads(name):
    wl = synth.workload(name)
    p = _params(wl.num_heads_q, wl.num_heads_kv, wl.head_dim, wl.page_size, wl.sinks, wl.window)
    n = wl.context[0] + 1  # the draft step's token is already appended
    kv = _paged(wl.seed, 1, wl.num_heads_kv, wl.head_dim, wl.page_size, [n], wl.kv_scale, wl.shuffle_pages)
    q = synth.queries(wl.seed + 100, (1, wl.num_heads_q, wl.head_dim), device=DEV)
    status = w.new_status(DEV)
    out, lse = w.draft_attn_full(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kp, vp, pt, lens = _oracle_pools(kv)
    ref, ref_lse = oracle.draft_attn_full(f64(q), kp, vp, pt, lens, wl.page_size, 1 / np.sqrt(wl.head_dim))
    assert_close(f64(out), ref, f"draft full {name}")
    assert_lse_close(f64(lse), ref_lse, f"draft full {name}")


@pytest.mark.parametrize("D,G,P", [(64, 4, 16), (64, 8, 32), (256, 8, 64), (256, 4, 128), (256, 8, 256),
                                   (256, 1, 64), (64, 2, 16)])
def test_draft_full_ragged_batch(D, G, P):
    Hkv = 2
    lens = [1, 63, 64, 65, 700, 2049, 0]
    B = len(lens)
    p = _params(G * Hkv, Hkv, D, P)
    kv = _paged(11 + D + G + P, B, Hkv, D, P, lens)
    q = synth.queries(12, (B, G * Hkv, D), device=DEV)
    status = w.new_status(DEV)
    out, lse = w.draft_attn_full(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kp, vp, pt, ln = _oracle_pools(kv)
    ref, ref_lse = oracle.draft_attn_full(f64(q), kp, vp, pt, ln, P, 1 / np.sqrt(D))
    assert_close(f64(out), ref, "draft full ragged")
    assert_lse_close(f64(lse), ref_lse, "draft full ragged")
    assert np.all(f64(out)[-1] == 0) and np.all(np.isneginf(f64(lse)[-1]))  # empty sequence


def test_draft_full_bf16_output_is_rounded_fp32_output():
    """bf16 output mode = the fp32 result rounded to nearest even, bit for
    bit; the fp32 result meets the parity bar; and where |ref| >= 1e-2 the
    bf16 value is within one bf16 ulp of the oracle."""
    p = _params(16, 2, 256, 64)
    kv = _paged(21, 2, 2, 256, 64, [5000, 777])
    q = synth.queries(22, (2, 16, 256), device=DEV)
    ob, lb = w.draft_attn_full(p, q, cache_of(kv), out_fp32=False)
    of, lf = w.draft_attn_full(p, q, cache_of(kv), out_fp32=True)
    torch.cuda.synchronize()
    assert ob.dtype == torch.bfloat16
    np.testing.assert_array_equal(bits(ob), bits(of.to(torch.bfloat16)))
    np.testing.assert_array_equal(f64(lb), f64(lf))
    kp, vp, pt, ln = _oracle_pools(kv)
    ref, _ = oracle.draft_attn_full(f64(q), kp, vp, pt, ln, 64, 1 / 16)
    assert_close(f64(of), ref, "fp32 mode")
    big = np.abs(ref) >= 1e-2
    assert bf16_ulp_diff(ob[torch.from_numpy(big).to(ob.device)], ref[big]) <= 1


def test_custom_softmax_scale():
    p = w.params(8, 1, 64, page_size=16, sm_scale=0.37)
    kv = _paged(23, 1, 1, 64, 16, [300])
    q = synth.queries(24, (1, 8, 64), device=DEV)
    out, lse = w.draft_attn_full(p, q, cache_of(kv))
    kp, vp, pt, ln = _oracle_pools(kv)
    ref, ref_lse = oracle.draft_attn_full(f64(q), kp, vp, pt, ln, 16, 0.37)
    assert_close(f64(out), ref, "custom scale")
    assert_lse_close(f64(lse), ref_lse, "custom scale")


# ---------------------------------------------------------------- verify
@pytest.mark.parametrize("num_q,G,D,P", [(4, 4, 64, 16), (1, 8, 256, 64), (2, 8, 256, 64), (4, 8, 256, 64),
                                         (6, 8, 256, 64), (8, 8, 256, 64), (3, 5, 64, 32), (4, 8, 256, 16),
                                         # tcgen05 path: 15 rows (odd G), 16 rows, the 64-row maximum,
                                         # 33 rows (the first block without spare lanes for P_lo)
                                         (3, 5, 256, 32), (4, 4, 256, 128), (4, 16, 256, 256), (3, 11, 256, 64),
                                         # tcgen05 with M = 128: gamma = 8 (72 rows), 65 and 128 rows
                                         (9, 8, 256, 64), (5, 13, 256, 64), (8, 16, 256, 32)])
def test_verify_ragged(num_q, G, D, P):
    Hkv = 2
    lens = [num_q, num_q + 1, 64, 65 + num_q, 1500, 4100]
    B = len(lens)
    p = _params(G * Hkv, Hkv, D, P)
    kv = _paged(31 + num_q + G, B, Hkv, D, P, lens)
    q = synth.queries(32, (B, num_q, G * Hkv, D), device=DEV)
    status = w.new_status(DEV)
    out, lse = w.verify_attn(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kp, vp, pt, ln = _oracle_pools(kv)
    ref, ref_lse = oracle.verify_attn(f64(q), kp, vp, pt, ln, P, 1 / np.sqrt(D))
    assert_close(f64(out), ref, f"verify q={num_q}")
    assert_lse_close(f64(lse), ref_lse, f"verify q={num_q}")


@pytest.mark.parametrize("name", ["tiny", "32k"])
def test_verify_workloads(name):
    wl = synth.workload(name)
    Qn = wl.gamma + 1
    n = wl.context[0] + Qn
    p = _params(wl.num_heads_q, wl.num_heads_kv, wl.head_dim, wl.page_size)
    kv = _paged(wl.seed + 1, 1, wl.num_heads_kv, wl.head_dim, wl.page_size, [n], wl.kv_scale, wl.shuffle_pages)
    q = synth.queries(wl.seed + 200, (1, Qn, wl.num_heads_q, wl.head_dim), device=DEV)
    out, lse = w.verify_attn(p, q, cache_of(kv))
    kp, vp, pt, ln = _oracle_pools(kv)
    ref, ref_lse = oracle.verify_attn(f64(q), kp, vp, pt, ln, wl.page_size, 1 / np.sqrt(wl.head_dim))
    assert_close(f64(out), ref, f"verify {name}")
    assert_lse_close(f64(lse), ref_lse, f"verify {name}")


# ---------------------------------------------------------------- combine
def test_splitkv_combine_against_oracle():
    g = torch.Generator(device=DEV).manual_seed(41)
    rows, nsplit, D = 37, 19, 256
    po = torch.randn(rows, nsplit, D, generator=g, device=DEV)
    pl = torch.randn(rows, nsplit, generator=g, device=DEV) * 5
    pl[3, :5] = -float("inf")
    pl[7, :] = -float("inf")
    out, lse = w.splitkv_combine(po, pl)
    ref, ref_lse = oracle.splitkv_combine(f64(po), f64(pl))
    assert_close(f64(out), ref, "combine", max_abs=1e-5, rel=1e-6)
    assert_lse_close(f64(lse), ref_lse, "combine", tol=1e-5)
    assert np.all(f64(out)[7] == 0)


# ---------------------------------------------------------------- paged write
def test_paged_write_bit_exact():
    p = _params(8, 2, 256, 16)
    kv = _paged(51, 3, 2, 256, 16, [10, 40, 0], capacity=80)
    k_before, v_before = bits(kv.k_pool), bits(kv.v_pool)
    kn, vn = synth.new_tokens(52, 3, 5, 2, 256, device=DEV)
    pos0 = torch.tensor([10, 30, 75], dtype=torch.int32, device=DEV)
    status = w.new_status(DEV)
    w.paged_write(p, cache_of(kv), pos0, kn, vn, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    exp_k, exp_v = k_before.copy(), v_before.copy()
    pt = kv.page_table.cpu().numpy()
    kb, vb = bits(kn), bits(vn)
    for b in range(3):
        for j in range(5):
            pos = int(pos0[b]) + j
            exp_k[pt[b, pos // 16], :, pos % 16] = kb[b, j]
            exp_v[pt[b, pos // 16], :, pos % 16] = vb[b, j]
    np.testing.assert_array_equal(bits(kv.k_pool), exp_k)
    np.testing.assert_array_equal(bits(kv.v_pool), exp_v)


# ---------------------------------------------------------------- ring
def _ring_state(ring):
    return dict(k=bits(ring.k), v=bits(ring.v), tags=ring.tags.cpu().numpy(), len=ring.len.cpu().numpy(),
                com=ring.committed.cpu().numpy(), uk=bits(ring.undo_k), uv=bits(ring.undo_v),
                ut=ring.undo_tags.cpu().numpy())


def _compare_ring(ring, models):
    st = _ring_state(ring)
    for b, m in enumerate(models):
        assert st["len"][b] == m.length and st["com"][b] == m.committed
        np.testing.assert_array_equal(st["tags"][b], m.tags())
        np.testing.assert_array_equal(st["k"][b], m.k_array().transpose(1, 0, 2))
        np.testing.assert_array_equal(st["v"][b], m.v_array().transpose(1, 0, 2))
        for j, (slot, tag, uk, uv) in enumerate(m.undo):
            assert st["ut"][b, j] == tag
            np.testing.assert_array_equal(st["uk"][b, j], uk)
            np.testing.assert_array_equal(st["uv"][b, j], uv)


@pytest.mark.parametrize("S,W,gmax,D", [(4, 37, 4, 64), (0, 5, 3, 64), (2, 1, 3, 256), (4, 256, 8, 256)])
def test_ring_append_bit_exact_random_ops(S, W, gmax, D):
    B, Hkv = 3, 2
    p = _params(8, Hkv, D, 64, S, W, gmax)
    ring = w.Ring.allocate(p, B, DEV)
    models = [oracle.RingModel(S, W, gmax, Hkv, D) for _ in range(B)]
    rng = np.random.default_rng(S * 100 + W)
    status = w.new_status(DEV)
    seed = 1000
    for step in range(40):
        kind = rng.choice(["bulk", "spec", "accept"], p=[0.2, 0.45, 0.35])
        seed += 1
        if kind == "bulk" and all(m.length == m.committed for m in models):
            maxn = int(rng.integers(1, 3 * (S + W) + 3))
            n = rng.integers(0, maxn + 1, size=B).astype(np.int32)
            kn, vn = synth.new_tokens(seed, B, maxn, Hkv, D, device=DEV)
            w.ring_append(p, ring, kn, vn, torch.from_numpy(n).to(DEV), status=status)
            for b, m in enumerate(models):
                m.call(-1, bits(kn[b, :n[b]]), bits(vn[b, :n[b]]), False)
        elif kind == "spec":
            room = [gmax - (m.length - m.committed) for m in models]
            n = np.array([rng.integers(0, r + 1) for r in room], dtype=np.int32)
            maxn = max(int(n.max()), 1)
            kn, vn = synth.new_tokens(seed, B, maxn, Hkv, D, device=DEV)
            w.ring_append(p, ring, kn, vn, torch.from_numpy(n).to(DEV), speculative=True, status=status)
            for b, m in enumerate(models):
                m.call(-1, bits(kn[b, :n[b]]), bits(vn[b, :n[b]]), True)
        else:
            tt = np.array([m.committed + rng.integers(0, m.length - m.committed + 1) for m in models],
                          dtype=np.int32)
            n = rng.integers(0, 2, size=B).astype(np.int32)
            kn, vn = synth.new_tokens(seed, B, 1, Hkv, D, device=DEV)
            w.ring_append(p, ring, kn, vn, torch.from_numpy(n).to(DEV),
                          truncate_to=torch.from_numpy(tt).to(DEV), status=status)
            for b, m in enumerate(models):
                m.call(int(tt[b]), bits(kn[b, :n[b]]), bits(vn[b, :n[b]]), False)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        _compare_ring(ring, models)


def test_ring_status_bits():
    p = _params(8, 2, 64, 64, 4, 16, 2)
    ring = w.Ring.allocate(p, 2, DEV)
    kn, vn = synth.new_tokens(61, 2, 3, 2, 64, device=DEV)
    status = w.new_status(DEV)
    w.ring_append(p, ring, kn, vn, torch.tensor([3, 3], dtype=torch.int32, device=DEV), speculative=True,
                  status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & L.DEV_UNDO_FULL
    status.zero_()
    w.ring_append(p, ring, kn, vn, torch.tensor([2, 0], dtype=torch.int32, device=DEV), status=status)
    w.ring_append(p, ring, None, None, None, truncate_to=torch.tensor([1, 0], dtype=torch.int32, device=DEV),
                  status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & L.DEV_RING_STATE
    assert ring.len.cpu().tolist() == [2, 0]


# ---------------------------------------------------------------- windowed
def _ring_from_history(p, kv, lens, spec_tail, device):
    """Ring of each sequence built by a bulk append of positions
    0..len-spec_tail-1 then spec_tail speculative appends.  Returns the ring
    and matching oracle models."""
    B = len(lens)
    Hkv, D = p.num_heads_kv, p.head_dim
    maxn = max(lens)
    kd = torch.zeros(B, max(maxn, 1), Hkv, D, dtype=torch.bfloat16, device=device)
    vd = torch.zeros_like(kd)
    for b, n in enumerate(lens):
        if n:
            k, v = synth.dense_from_paged(kv, b, n)
            kd[b, :n] = k
            vd[b, :n] = v
    ring = w.Ring.allocate(p, B, device)
    models = [oracle.RingModel(p.sinks, p.window, p.gamma_max, Hkv, D) for _ in range(B)]
    n0 = np.array([max(n - spec_tail, 0) for n in lens], dtype=np.int32)
    w.ring_append(p, ring, kd, vd, torch.from_numpy(n0).to(device))
    for b, m in enumerate(models):
        m.call(-1, bits(kd[b, :n0[b]]), bits(vd[b, :n0[b]]), False)
    for j in range(spec_tail):
        nj = np.array([1 if n0[b] + j < lens[b] else 0 for b in range(B)], dtype=np.int32)
        ks = torch.stack([kd[b, min(n0[b] + j, max(maxn, 1) - 1)] for b in range(B)])[:, None].contiguous()
        vs = torch.stack([vd[b, min(n0[b] + j, max(maxn, 1) - 1)] for b in range(B)])[:, None].contiguous()
        w.ring_append(p, ring, ks, vs, torch.from_numpy(nj).to(device), speculative=True)
        for b, m in enumerate(models):
            m.call(-1, bits(ks[b, :nj[b]]), bits(vs[b, :nj[b]]), True)
    torch.cuda.synchronize()
    return ring, models


@pytest.mark.parametrize("S,W,D,G", [(4, 256, 64, 4), (4, 2048, 256, 8), (0, 100, 256, 8), (7, 64, 64, 8),
                                     (4, 1024, 256, 8), (4, 4096, 256, 8)])
def test_windowed_draft_vs_oracle(S, W, D, G):
    Hkv = 2
    lens = [1, S + W - 1, S + W, S + W + 1, 3 * (S + W) + 17, 5000]
    B = len(lens)
    p = _params(G * Hkv, Hkv, D, 64, S, W, 4)
    kv = _paged(71 + W, B, Hkv, D, 64, lens)
    ring, models = _ring_from_history(p, kv, lens, 3, DEV)
    _compare_ring(ring, models)
    q = synth.queries(72, (B, G * Hkv, D), device=DEV)
    status = w.new_status(DEV)
    out, lse = w.draft_attn_windowed(p, q, ring, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    scale = 1 / np.sqrt(D)
    ref, ref_lse = oracle.draft_attn_windowed(f64(q), models, scale)
    assert_close(f64(out), ref, "windowed vs ring oracle")
    assert_lse_close(f64(lse), ref_lse, "windowed vs ring oracle")
    # the same set read from the full history
    kp, vp, pt, ln = _oracle_pools(kv)
    ref2, _ = oracle.draft_attn_windowed_paged(f64(q), kp, vp, pt, np.asarray(lens), 64, S, W, scale)
    assert_close(f64(out), ref2, "windowed vs history oracle")


def test_windowed_equals_full_when_window_covers_context():
    S, W, D, G, Hkv = 4, 2048, 256, 8, 2
    lens = [100, 2052]
    p = _params(G * Hkv, Hkv, D, 64, S, W, 4)
    kv = _paged(81, 2, Hkv, D, 64, lens)
    ring, _ = _ring_from_history(p, kv, lens, 3, DEV)
    q = synth.queries(82, (2, G * Hkv, D), device=DEV)
    ow, lw = w.draft_attn_windowed(p, q, ring)
    of, lf = w.draft_attn_full(p, q, cache_of(kv))
    kp, vp, pt, ln = _oracle_pools(kv)
    ref, _ = oracle.draft_attn_full(f64(q), kp, vp, pt, ln, 64, 1 / 16)
    assert_close(f64(ow), ref, "windowed == full")
    assert_close(f64(of), ref, "full")
    np.testing.assert_allclose(f64(ow), f64(of), atol=1e-5, rtol=0)


# ---------------------------------------------------------------- windowed draft over pages
@pytest.mark.parametrize("S,W,lens,P,D,G", [
    (4, 256, [2049], 16, 64, 4),                 # tiny shapes
    (4, 2048, [32769], 64, 256, 8),              # window inside a long history
    (0, 100, [5000, 64], 64, 256, 8),            # no sinks; W not a multiple of 64
    (200, 50, [100], 64, 256, 8),                # shorter than the sinks
    (4, 2048, [1500, 2052], 64, 256, 8),         # window reaches the sinks: the full set
    (64, 1000, [70000, 123, 64 * 37 + 5], 32, 256, 8),  # ragged batch, window start mid-page
    (5, 130, [9000], 128, 256, 4),               # sinks and window share no tile boundary
])
def test_windowed_paged_vs_oracle(S, W, lens, P, D, G):
    Hkv = 2
    p = _params(G * Hkv, Hkv, D, P, S, W)
    kv = _paged(91 + S, len(lens), Hkv, D, P, lens)
    q = synth.queries(92 + W, (len(lens), G * Hkv, D), device=DEV)
    status = w.new_status(DEV)
    out, lse = w.draft_attn_windowed_paged(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kp, vp, pt, ln = _oracle_pools(kv)
    scale = 1 / np.sqrt(D)
    ref, ref_lse = oracle.draft_attn_windowed_paged(f64(q), kp, vp, pt, ln, P, S, W, scale)
    assert_close(f64(out), ref, f"windowed paged S={S} W={W} lens={lens}")
    assert_lse_close(f64(lse), ref_lse, f"windowed paged S={S} W={W}")
    # the full set when the window reaches the sinks
    if all(n <= S + W for n in lens):
        of, _ = w.draft_attn_full(p, q, cache_of(kv))
        np.testing.assert_allclose(f64(out), f64(of), atol=1e-5, rtol=0)


def test_windowed_paged_window_changes_per_call():
    # an adaptive window: the same cache read with a different W on each call
    S, D, G, Hkv, P = 4, 256, 8, 2, 64
    lens = [40000]
    kv = _paged(95, 1, Hkv, D, P, lens)
    q = synth.queries(96, (1, G * Hkv, D), device=DEV)
    kp, vp, pt, ln = _oracle_pools(kv)
    for W in (64, 1000, 4096, 40000):
        p = _params(G * Hkv, Hkv, D, P, S, W)
        out, _ = w.draft_attn_windowed_paged(p, q, cache_of(kv))
        ref, _ = oracle.draft_attn_windowed_paged(f64(q), kp, vp, pt, ln, P, S, W, 1 / 16)
        assert_close(f64(out), ref, f"windowed paged W={W}")


def test_windowed_paged_rejects_bad_window():
    p = _params(16, 2, 256, 64, 4, 0)
    kv = _paged(97, 1, 2, 256, 64, [100])
    q = synth.queries(98, (1, 16, 256), device=DEV)
    with pytest.raises(L.WmtpError):
        w.draft_attn_windowed_paged(p, q, cache_of(kv))


# ---------------------------------------------------------------- device status
def test_bad_page_table_and_length_set_status():
    p = _params(8, 1, 64, 16)
    kv = _paged(91, 2, 1, 64, 16, [100, 50])
    kv.page_table[0, 2] = 10 ** 6
    q = synth.queries(92, (2, 8, 64), device=DEV)
    status = w.new_status(DEV)
    w.draft_attn_full(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & L.DEV_PAGE_OOB
    kv.page_table[0, 2] = 0
    kv.kv_len[1] = kv.page_table.shape[1] * 16 + 1
    status.zero_()
    out, lse = w.draft_attn_full(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & L.DEV_LEN_OOB
    assert np.all(f64(out)[1] == 0)


def test_workspace_query_matches_binding():
    p = _params(16, 2, 256, 64)
    n = w.workspace_bytes("full", p, 1, max_pages=16384)
    assert n > 0 and n % 256 == 0
    assert w.workspace_bytes("verify", p, 1, num_q=4, max_pages=16384) >= n


def test_verify_takes_values_of_any_bf16_magnitude():
    """The tcgen05 verify reads V in its own bf16 format: values far beyond
    the fp16 range (1e5, -3e30) and tiny ones (1e-30) go through exactly, and
    no status bit is raised."""
    p = _params(16, 2, 256, 64)
    kv = _paged(95, 1, 2, 256, 64, [300])
    kv.v_pool[kv.page_table[0, 1], 1, 5, 7] = 1.0e5
    kv.v_pool[kv.page_table[0, 2], 0, 9, 100] = -3.0e30
    kv.v_pool[kv.page_table[0, 0], 1, 0, :] = 1.0e-30
    q = synth.queries(96, (1, 4, 16, 256), device=DEV)
    status = w.new_status(DEV)
    out, lse = w.verify_attn(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kp, vp, pt, ln = _oracle_pools(kv)
    ref, ref_lse = oracle.verify_attn(f64(q), kp, vp, pt, ln, 64, 1 / 16)
    # relative to each element's own scale: the planted values dominate a few
    # output columns by 30 orders of magnitude
    got = f64(out)
    scale = np.maximum(np.abs(ref), 1.0)
    assert np.all(np.abs(got - ref) <= 2e-3 * scale), float(np.max(np.abs(got - ref) / scale))
    assert_lse_close(f64(lse), ref_lse, "verify large values")


@pytest.mark.parametrize("kind", ["verify", "draft"])
def test_page_outside_the_pool_is_skipped(kind):
    """A page-table entry outside the pool raises WMTP_DEV_PAGE_OOB and the
    tile holding it is left out of the attention: the result equals the
    oracle's attention over the other positions (head_dim 256, page 64, so
    one page is one 64-token tile; verify runs on the tcgen05 kernel)."""
    Hkv, G, D, P = 2, 8, 256, 64
    num_q = 4 if kind == "verify" else 1
    n = 9000 + num_q
    p = _params(G * Hkv, Hkv, D, P)
    kv = _paged(97, 1, Hkv, D, P, [n])
    bad_page = 37  # positions 2368 .. 2431
    kv.page_table[0, bad_page] = kv.k_pool.shape[0] + 5
    shape = (1, num_q, G * Hkv, D) if kind == "verify" else (1, G * Hkv, D)
    q = synth.queries(98, shape, device=DEV)
    status = w.new_status(DEV)
    fn = w.verify_attn if kind == "verify" else w.draft_attn_full
    out, lse = fn(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & L.DEV_PAGE_OOB
    # the oracle over every position but the bad page's, gathered through the
    # valid entries of the table
    kp, vp = f64(kv.k_pool), f64(kv.v_pool)
    pt = kv.page_table.cpu().numpy()[0].astype(np.int64)
    keep = np.array([t for t in range(n) if t // P != bad_page])
    qs = f64(q).reshape(num_q, G * Hkv, D)
    got, got_lse = f64(out).reshape(num_q, G * Hkv, D), f64(lse).reshape(num_q, G * Hkv)
    for kvh in range(Hkv):
        K = kp[pt[keep // P], kvh, keep % P]
        V = vp[pt[keep // P], kvh, keep % P]
        for i in range(num_q):
            last = n - num_q + i  # causal limit of query i
            sel = keep <= last
            rows = slice(kvh * G, (kvh + 1) * G)
            ref, ref_lse = oracle.attend_rows(qs[i, rows], K[sel], V[sel], 1 / 16)
            assert_close(got[i, rows], ref, f"{kind} skip kvh {kvh} q {i}")
            assert_lse_close(got_lse[i, rows], ref_lse, f"{kind} skip kvh {kvh} q {i}")

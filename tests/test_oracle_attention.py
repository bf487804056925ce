"""Pins for the fp64 attention oracle (CPU only).

Each test checks the oracle against something other than its own formula: a
library routine (torch's float64 scaled_dot_product_attention and logsumexp),
40-digit decimal arithmetic, closed forms, invariances, or the figures the
pages print (tests/golden/pages_figures.txt).
"""

import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            out[k] = float(v)
    return out


def _rng(seed=0):
    return np.random.default_rng(seed)


def _sdpa(q, K, V, scale, mask=None):
    """torch float64 SDPA of rows q [R, D] over K/V [n, D] (a library pin)."""
    qt = torch.from_numpy(np.ascontiguousarray(q))[None, None]
    kt = torch.from_numpy(np.ascontiguousarray(K))[None, None]
    vt = torch.from_numpy(np.ascontiguousarray(V))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    return o[0, 0].numpy()


# ---------------------------------------------------------------------------
# attend: library, high precision, closed forms
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n,d,scale", [(1, 4, 0.5), (7, 8, 0.125), (200, 64, 0.125), (513, 256, 1 / 16)])
def test_attend_matches_torch_sdpa_float64(n, d, scale):
    r = _rng(n + d)
    q = r.standard_normal((3, d))
    K = r.standard_normal((n, d)) * 2.0
    V = r.standard_normal((n, d))
    o, lse = A.attend_rows(q, K, V, scale)
    ref = _sdpa(q, K, V, scale)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(torch.from_numpy(scale * (q @ K.T)), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_attend_matches_decimal_bruteforce():
    """40-digit decimal arithmetic, term by term, on a tiny case."""
    getcontext().prec = 40
    r = _rng(3)
    n, d, scale = 6, 3, 0.7
    q = r.standard_normal(d)
    K = r.standard_normal((n, d)) * 3
    V = r.standard_normal((n, d))
    s = [sum(Decimal(float(q[j])) * Decimal(float(K[t, j])) for j in range(d)) * Decimal(scale)
         for t in range(n)]
    e = [x.exp() for x in s]
    tot = sum(e)
    o_ref = [float(sum(e[t] * Decimal(float(V[t, j])) for t in range(n)) / tot) for j in range(d)]
    lse_ref = float(tot.ln())
    o, lse = A.attend(q, K, V, scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-14)
    assert abs(lse - lse_ref) < 1e-13


def test_attend_zero_query_is_mean_of_values():
    r = _rng(4)
    K = r.standard_normal((37, 16))
    V = r.standard_normal((37, 16))
    o, lse = A.attend(np.zeros(16), K, V, 0.25)
    np.testing.assert_allclose(o, V.mean(axis=0), rtol=0, atol=1e-14)
    assert abs(lse - math.log(37)) < 1e-14


def test_attend_single_key_returns_its_value():
    r = _rng(5)
    q, k, v = r.standard_normal(8), r.standard_normal((1, 8)), r.standard_normal((1, 8))
    o, lse = A.attend(q, k, v, 0.3)
    np.testing.assert_array_equal(o, v[0])
    assert abs(lse - 0.3 * float(k[0] @ q)) < 1e-14


def test_attend_two_keys_logistic_closed_form():
    r = _rng(6)
    q = r.standard_normal(5)
    K = r.standard_normal((2, 5))
    V = r.standard_normal((2, 5))
    scale = 0.9
    s0, s1 = scale * K[0] @ q, scale * K[1] @ q
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    o, lse = A.attend(q, K, V, scale)
    np.testing.assert_allclose(o, w0 * V[0] + (1 - w0) * V[1], rtol=0, atol=1e-14)
    assert abs(lse - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) < 1e-13


def test_attend_constant_values_give_that_constant():
    """Weights sum to one: V rows all equal c gives exactly c (to rounding)."""
    r = _rng(7)
    K = r.standard_normal((300, 32)) * 4
    V = np.full((300, 32), 2.5)
    o, _ = A.attend(r.standard_normal(32), K, V, 0.5)
    np.testing.assert_allclose(o, 2.5, rtol=0, atol=1e-13)


def test_attend_shift_invariance():
    """Adding c to every score leaves o alone and adds c to lse."""
    r = _rng(8)
    q = r.standard_normal(12)
    K = r.standard_normal((50, 12))
    V = r.standard_normal((50, 12))
    c = 3.75
    q2 = np.concatenate([q, [1.0]])
    K2 = np.concatenate([K, np.full((50, 1), c / 0.5)], axis=1)
    V2 = V
    o1, l1 = A.attend(q, K, V, 0.5)
    o2, l2 = A.attend(q2, K2, V2, 0.5)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    assert abs(l2 - (l1 + c)) < 1e-12


def test_attend_permutation_invariance_and_empty():
    r = _rng(9)
    q = r.standard_normal(8)
    K = r.standard_normal((20, 8))
    V = r.standard_normal((20, 8))
    perm = r.permutation(20)
    o1, l1 = A.attend(q, K, V, 1.0)
    o2, l2 = A.attend(q, K[perm], V[perm], 1.0)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    assert abs(l1 - l2) < 1e-13
    o, lse = A.attend(q, K[:0], V[:0], 1.0)
    assert np.all(o == 0) and lse == -np.inf


def test_attend_prefixes_matches_torch_sdpa_with_prefix_mask():
    # library pin: float64 SDPA with a boolean mask that keeps key t for row r
    # iff t < lengths[r] (the causal-verify and growing-draft shapes)
    r = _rng(11)
    n, d, R = 37, 16, 6
    K, V, Q = r.standard_normal((n, d)), r.standard_normal((n, d)), r.standard_normal((R, d))
    lengths = np.array([1, 5, 36, 37, 20, 2])
    o, lse = A.attend_prefixes(Q, K, V, lengths, 0.3)
    mask = np.arange(n)[None, :] < lengths[:, None]
    np.testing.assert_allclose(o, _sdpa(Q, K, V, 0.3, mask), atol=1e-12, rtol=0)
    s = 0.3 * (Q @ K.T)
    ref_lse = torch.logsumexp(torch.from_numpy(np.where(mask, s, -np.inf)), -1).numpy()
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12, rtol=0)


def test_attend_prefixes_bruteforce_and_edges():
    # pure-Python loops on a tiny case, an empty prefix, and the full prefix
    r = _rng(12)
    n, d = 6, 3
    K, V, Q = r.standard_normal((n, d)), r.standard_normal((n, d)), r.standard_normal((3, d))
    lengths = [0, 4, 6]
    o, lse = A.attend_prefixes(Q, K, V, lengths, 0.5)
    assert np.all(o[0] == 0) and lse[0] == -np.inf
    for row in (1, 2):
        L_ = lengths[row]
        sc = [0.5 * sum(Q[row, c] * K[t, c] for c in range(d)) for t in range(L_)]
        mx = max(sc)
        ex = [math.exp(x - mx) for x in sc]
        tot = sum(ex)
        for c in range(d):
            assert abs(o[row, c] - sum(ex[t] * V[t, c] for t in range(L_)) / tot) < 1e-12
        assert abs(lse[row] - (mx + math.log(tot))) < 1e-12
    with pytest.raises(ValueError):
        A.attend_prefixes(Q, K, V, [1, 2, 7], 0.5)


def test_bf16_widening_is_exact():
    x = torch.randn(1000, dtype=torch.float32).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(A.bf16_bits_to_f64(bits), x.double().numpy())


# ---------------------------------------------------------------------------
# attended sets
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("length,S,W,expect", [
    (10, 2, 3, [0, 1, 7, 8, 9]),
    (5, 0, 3, [2, 3, 4]),
    (3, 4, 2, [0, 1, 2]),
    (6, 4, 2, [0, 1, 2, 3, 4, 5]),
    (7, 4, 2, [0, 1, 2, 3, 5, 6]),
    (1, 4, 256, [0]),
    (0, 4, 256, []),
])
def test_window_positions_small_cases(length, S, W, expect):
    assert A.window_positions(length, S, W).tolist() == expect


def test_window_size_and_identity_with_full():
    for S in (0, 1, 4):
        for W in (1, 3, 16):
            for n in range(0, 40):
                pos = A.window_positions(n, S, W)
                assert len(pos) == min(n, S + W)
                assert len(set(pos.tolist())) == len(pos)
                if n <= S + W:
                    assert pos.tolist() == list(range(n))
                if n > 0:
                    assert pos[-1] == n - 1  # the current token is attended


def test_window_drops_about_99_percent_at_1m():
    g = _golden()
    ctx = int(g["context_1m"])
    for W in (1024, 2048, 4096):
        kept = len(A.window_positions(ctx, 4, W))
        assert kept == 4 + W
        assert 1 - kept / ctx >= g["dropped_fraction_at_1m"]


def test_causal_positions():
    assert A.causal_positions(10, 4, 0).tolist() == list(range(7))
    assert A.causal_positions(10, 4, 3).tolist() == list(range(10))
    assert A.causal_positions(10, 1, 0).tolist() == A.full_positions(10).tolist()


# ---------------------------------------------------------------------------
# paged calls
# ---------------------------------------------------------------------------

def _paged(seed, B, Hkv, D, P, lens, shuffle):
    r = _rng(seed)
    maxp = max(-(-n // P) for n in lens) + 1
    npages = B * maxp
    kp = r.standard_normal((npages, Hkv, P, D))
    vp = r.standard_normal((npages, Hkv, P, D))
    perm = r.permutation(npages) if shuffle else np.arange(npages)
    table = perm.reshape(B, maxp)
    return kp, vp, table


def _dense(pool, table, b, n, P, kvh):
    return np.stack([pool[table[b, p // P], kvh, p % P] for p in range(n)]) if n else np.zeros((0, pool.shape[-1]))


def test_draft_full_matches_sdpa_on_dense_history_and_gqa():
    B, Hq, Hkv, D, P = 2, 8, 2, 16, 4
    lens = [13, 30]
    kp, vp, table = _paged(10, B, Hkv, D, P, lens, True)
    q = _rng(11).standard_normal((B, Hq, D))
    o, lse = A.draft_attn_full(q, kp, vp, table, lens, P, 0.25)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            K = _dense(kp, table, b, lens[b], P, h // G)
            V = _dense(vp, table, b, lens[b], P, h // G)
            np.testing.assert_allclose(o[b, h], _sdpa(q[b, h][None], K, V, 0.25)[0], atol=1e-12, rtol=0)


def test_gqa_head_mapping():
    """Head h must read KV head h // G: make KV head 1's values constant."""
    B, Hq, Hkv, D, P = 1, 6, 3, 8, 4
    kp, vp, table = _paged(12, B, Hkv, D, P, [9], False)
    vp[:, 1] = 5.0
    q = _rng(13).standard_normal((B, Hq, D))
    o, _ = A.draft_attn_full(q, kp, vp, table, [9], P, 0.5)
    np.testing.assert_allclose(o[0, 2:4], 5.0, atol=1e-13, rtol=0)
    assert np.abs(o[0, 0:2] - 5.0).min() > 1e-3 and np.abs(o[0, 4:6] - 5.0).min() > 1e-3


def test_page_table_layout_independence():
    B, Hq, Hkv, D, P = 1, 4, 1, 8, 4
    lens = [21]
    kp, vp, table = _paged(14, B, Hkv, D, P, lens, False)
    q = _rng(15).standard_normal((B, Hq, D))
    o1, l1 = A.draft_attn_full(q, kp, vp, table, lens, P, 0.5)
    perm = _rng(16).permutation(kp.shape[0])
    inv = np.argsort(perm)
    kp2, vp2 = kp[perm], vp[perm]          # page x now lives at inv[x]
    o2, l2 = A.draft_attn_full(q, kp2, vp2, inv[table], lens, P, 0.5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_verify_matches_sdpa_causal_and_reduces_to_draft():
    B, Qn, Hq, Hkv, D, P = 2, 4, 4, 2, 16, 8
    lens = [40, 19]
    kp, vp, table = _paged(17, B, Hkv, D, P, lens, True)
    q = _rng(18).standard_normal((B, Qn, Hq, D))
    o, lse = A.verify_attn(q, kp, vp, table, lens, P, 0.25)
    G = Hq // Hkv
    for b in range(B):
        n = lens[b]
        mask = np.arange(n)[None, :] <= (n - Qn + np.arange(Qn))[:, None]
        for h in range(Hq):
            K = _dense(kp, table, b, n, P, h // G)
            V = _dense(vp, table, b, n, P, h // G)
            ref = _sdpa(q[b, :, h], K, V, 0.25, mask)
            np.testing.assert_allclose(o[b, :, h], ref, atol=1e-12, rtol=0)
    # query 0 == native draft at length n - Qn + 1; Qn = 1 verify == draft
    lens0 = [n - Qn + 1 for n in lens]
    od, ld = A.draft_attn_full(q[:, 0], kp, vp, table, lens0, P, 0.25)
    np.testing.assert_allclose(o[:, 0], od, atol=1e-13, rtol=0)
    o1, l1 = A.verify_attn(q[:, :1], kp, vp, table, lens, P, 0.25)
    od1, ld1 = A.draft_attn_full(q[:, 0], kp, vp, table, lens, P, 0.25)
    np.testing.assert_allclose(o1[:, 0], od1, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l1[:, 0], ld1, atol=1e-13, rtol=0)


def test_windowed_paged_equals_full_when_window_covers_context():
    B, Hq, Hkv, D, P = 1, 4, 1, 8, 4
    lens = [23]
    kp, vp, table = _paged(19, B, Hkv, D, P, lens, True)
    q = _rng(20).standard_normal((B, Hq, D))
    of, lf = A.draft_attn_full(q, kp, vp, table, lens, P, 0.5)
    ow, lw = A.draft_attn_windowed_paged(q, kp, vp, table, lens, P, 3, 20, 0.5)
    np.testing.assert_array_equal(of, ow)
    ow2, _ = A.draft_attn_windowed_paged(q, kp, vp, table, lens, P, 3, 19, 0.5)
    assert np.abs(ow2 - of).max() > 1e-6


def test_windowed_paged_matches_sdpa_with_window_mask():
    B, Hq, Hkv, D, P = 1, 2, 1, 8, 4
    n, S, W = 37, 3, 5
    kp, vp, table = _paged(21, B, Hkv, D, P, [n], True)
    q = _rng(22).standard_normal((B, Hq, D))
    ow, lw = A.draft_attn_windowed_paged(q, kp, vp, table, [n], P, S, W, 0.5)
    K = _dense(kp, table, 0, n, P, 0)
    V = _dense(vp, table, 0, n, P, 0)
    mask = np.zeros((1, n), dtype=bool)
    mask[0, :S] = True
    mask[0, n - W:] = True
    for h in range(Hq):
        np.testing.assert_allclose(ow[0, h], _sdpa(q[0, h][None], K, V, 0.5, mask)[0], atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# split-KV combine
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bounds", [
    [(0, 50)],
    [(0, 1), (1, 2), (2, 50)],
    [(0, 17), (17, 17), (17, 33), (33, 50)],
    [(i, i + 1) for i in range(50)],
])
def test_combine_of_any_partition_equals_unsplit(bounds):
    r = _rng(23)
    q = r.standard_normal(16)
    K = r.standard_normal((50, 16)) * 2
    V = r.standard_normal((50, 16))
    po, pl = A.split_partials(q, K, V, bounds, 0.5)
    o, lse = A.splitkv_combine(po[None], pl[None])
    o_ref, lse_ref = A.attend(q, K, V, 0.5)
    np.testing.assert_allclose(o[0], o_ref, atol=1e-13, rtol=0)
    assert abs(lse[0] - lse_ref) < 1e-12


def test_combine_all_empty_and_matches_torch_logsumexp():
    o, lse = A.splitkv_combine(np.zeros((2, 3, 4)), np.full((2, 3), -np.inf))
    assert np.all(o == 0) and np.all(lse == -np.inf)
    r = _rng(24)
    pl = r.standard_normal((5, 7)) * 10
    po = r.standard_normal((5, 7, 3))
    _, lse = A.splitkv_combine(po, pl)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(pl), -1).numpy(), atol=1e-12, rtol=0)


def test_oracle_package_exports():
    for name in ["attend", "attend_prefixes", "draft_attn_full", "draft_attn_windowed", "verify_attn",
                 "splitkv_combine", "RingModel", "window_positions"]:
        assert hasattr(oracle, name)

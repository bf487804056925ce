"""Host-side KV page allocation and admission planning (include/wmtp_pool.h).

CPU only: the pool and the planner touch no device.  The allocator is checked
against a plain set model under random alloc/release sequences; the planner's
footprints against the layouts the attention calls use, and its 1M-context
reclaimed share and extra request against the figures the pages print.
"""

import os

import pytest
from hypothesis import given, settings, strategies as st

import speculative_decode_draft_b200 as w
from speculative_decode_draft_b200 import _lib as L

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            out[k] = float(v)
    return out


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from speculative_decode_draft_b200 import build
    build.build()
    L.load()


def test_pool_alloc_release_and_errors():
    pool = w.PagePool(10)
    assert pool.free_count == 10
    a = pool.alloc(4)
    assert a == [0, 1, 2, 3] and pool.free_count == 6
    with pytest.raises(L.WmtpError) as e:
        pool.alloc(7)  # all or nothing
    assert e.value.code == L.WMTP_ERR_WORKSPACE and pool.free_count == 6
    for bad in ([3, 3], [4], [-1], [10], [1, 99]):
        with pytest.raises(L.WmtpError) as e:
            pool.release(bad)  # duplicate, not held, out of range: nothing released
        assert e.value.code == L.WMTP_ERR_INVALID_ARG and pool.free_count == 6
    pool.release([1, 3])
    assert pool.free_count == 8
    b = pool.alloc(8)
    assert sorted(b) == [1, 3, 4, 5, 6, 7, 8, 9]
    assert pool.alloc(0) == [] and pool.free_count == 0
    pool.release(a[::2] + b)  # 1 and 3 came back inside b
    assert pool.free_count == 10
    with pytest.raises(L.WmtpError):
        w.PagePool(0)


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 64), st.lists(st.tuples(st.booleans(), st.integers(0, 70), st.integers(0, 2**31 - 1)),
                                    max_size=40))
def test_pool_matches_set_model(n, ops):
    pool = w.PagePool(n)
    free = set(range(n))
    held = []
    for is_alloc, k, seed in ops:
        if is_alloc:
            if k <= len(free):
                got = pool.alloc(k)
                assert len(set(got)) == k and set(got) <= free
                free -= set(got)
                held += got
            else:
                with pytest.raises(L.WmtpError):
                    pool.alloc(k)
        else:
            m = min(k, len(held))
            take = [held[(seed + 7 * i) % len(held)] for i in range(m)] if held else []
            take = list(dict.fromkeys(take))  # distinct
            pool.release(take)
            free |= set(take)
            held = [x for x in held if x not in set(take)]
        assert pool.free_count == len(free)


def _params(window=4096, gamma=3):
    return w.params(16, 2, 256, page_size=64, sinks=4, window=window, gamma_max=gamma)


def test_admission_footprints_follow_the_layouts():
    p = _params()
    n = 1048576
    nat = w.plan_admission(p, n, 10, 1, False, 0)
    win = w.plan_admission(p, n, 10, 1, True, 0)
    # a paged layer: ceil((n + gamma + 1) / P) pages of K and V, Hkv x P x D bf16 each
    assert nat["pages_per_layer"] == -(-(n + 4) // 64) == 16385
    assert nat["page_bytes"] == 2 * 2 * 64 * 256 * 2
    assert nat["target_bytes"] == win["target_bytes"] == 10 * 16385 * 131072
    assert nat["draft_bytes"] == 16385 * 131072
    # the ring: S+W slots of K and V (as wmtp_ring's [B][Hkv][S+W][D]) + tags,
    # gamma_max undo entries + tags, two lengths
    assert win["draft_bytes"] == 2 * 4100 * 2 * 256 * 2 + 4100 * 4 + 2 * 3 * 2 * 256 * 2 + 3 * 4 + 8
    with pytest.raises(L.WmtpError):
        w.plan_admission(_params(window=0), n, 10, 1, True, 0)


def test_reclaimed_share_and_extra_request_at_1m_match_the_pages():
    g = _golden()
    p = _params()
    n = int(g["context_1m"])
    L_t, L_d = int(g["target_full_attention_layers"]), int(g["draft_layers"])
    nat = w.plan_admission(p, n, L_t, L_d, False, 0)
    win = w.plan_admission(p, n, L_t, L_d, True, 0)
    share = 1 - win["bytes_per_request"] / nat["bytes_per_request"]
    assert g["kv_reclaimed_fraction_lo"] <= share <= g["kv_reclaimed_fraction_hi"]
    # a B200 holds 180 GB; with 20 GB for weights the KV budget admits one
    # more concurrent 1M-token request once the draft pool is reclaimed
    budget = 160 * 10**9
    a_nat = w.plan_admission(p, n, L_t, L_d, False, budget)["max_requests"]
    a_win = w.plan_admission(p, n, L_t, L_d, True, budget)["max_requests"]
    assert a_win - a_nat == int(g["extra_requests_at_1m"])
    # never fewer requests with the ring, at any budget
    for b in range(0, 400 * 10**9, 7 * 10**9):
        assert (w.plan_admission(p, n, L_t, L_d, True, b)["max_requests"]
                >= w.plan_admission(p, n, L_t, L_d, False, b)["max_requests"])


def test_admission_agrees_with_allocating_the_pages():
    # admit requests into a pool of the budget's pages until allocation fails
    p = _params(window=1024)
    n = 20000
    budget = 3 * 10**9
    for windowed in (False, True):
        plan = w.plan_admission(p, n, 10, 1, windowed, budget)
        # the ring is not paged: give the pool the budget minus the rings of
        # the planned requests, and count requests whose paged layers fit
        rings = plan["draft_bytes"] * plan["max_requests"] if windowed else 0
        pool = w.PagePool((budget - rings) // plan["page_bytes"])
        layers = 10 if windowed else 11
        admitted = 0
        while True:
            try:
                pool.alloc(layers * plan["pages_per_layer"])
            except L.WmtpError:
                break
            admitted += 1
        assert admitted == plan["max_requests"]

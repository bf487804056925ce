"""Pins for the ring-buffer oracle (CPU only).

The ring model is checked against (a) small cases worked out by hand from the
slot rule, and (b) a second, independent description of what the ring must
hold: the plain history list of every position's latest K/V, from which the
sink + window entries are read off directly.  Random operation sequences
(hypothesis) drive both.
"""

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import RingModel


def _tok(p, hkv=1, d=2):
    """A distinct, recognisable [Hkv, D] value for position p (uint16 bits)."""
    return np.full((hkv, d), p + 1, dtype=np.uint16)


def test_hand_worked_small_ring():
    # S=2, W=3: slots 0,1 are sinks; positions >= 2 cycle through slots 2,3,4.
    r = RingModel(2, 3, 3, 1, 2)
    r.call(-1, np.stack([_tok(p) for p in range(7)]), np.stack([_tok(p) for p in range(7)]), False)
    # p: 0->0 1->1 2->2 3->3 4->4 5->2 6->3
    assert r.tags().tolist() == [0, 1, 5, 6, 4]
    assert r.length == 7 and r.committed == 7
    # speculative 7 (slot 4, evicts 4) and 8 (slot 2, evicts 5)
    r.call(-1, np.stack([_tok(7), _tok(8)]), np.stack([_tok(7), _tok(8)]), True)
    assert r.tags().tolist() == [0, 1, 8, 6, 7]
    assert r.committed == 7 and r.length == 9
    # reject 8: restore 5 into slot 2
    r.call(8, np.zeros((0, 1, 2), np.uint16), np.zeros((0, 1, 2), np.uint16), False)
    assert r.tags().tolist() == [0, 1, 5, 6, 7]
    assert r.length == r.committed == 8
    assert (r.k_array()[2] == _tok(5)).all()


def test_hand_worked_rollback_all_and_wrap_with_small_window():
    # W=1 smaller than the speculative depth: undo must restore in reverse.
    r = RingModel(1, 1, 3, 1, 2)
    r.call(-1, np.stack([_tok(0), _tok(1)]), np.stack([_tok(0), _tok(1)]), False)
    assert r.tags().tolist() == [0, 1]
    r.call(-1, np.stack([_tok(2), _tok(3), _tok(4)]), np.stack([_tok(2), _tok(3), _tok(4)]), True)
    assert r.tags().tolist() == [0, 4]
    r.call(2, np.zeros((0, 1, 2), np.uint16), np.zeros((0, 1, 2), np.uint16), False)
    assert r.tags().tolist() == [0, 1]
    assert (r.k_array()[1] == _tok(1)).all()


def test_first_fill_is_identity_layout():
    r = RingModel(4, 8, 3, 2, 4)
    n = 9
    r.call(-1, np.stack([_tok(p, 2, 4) for p in range(n)]), np.stack([_tok(p, 2, 4) for p in range(n)]), False)
    assert r.tags().tolist() == list(range(9)) + [-1, -1, -1]


def test_errors():
    r = RingModel(2, 3, 2, 1, 2)
    r.call(-1, np.stack([_tok(0)]), np.stack([_tok(0)]), False)
    with pytest.raises(ValueError):
        r.call(-1, np.stack([_tok(1), _tok(2), _tok(3)]), np.stack([_tok(1), _tok(2), _tok(3)]), True)
    r2 = RingModel(2, 3, 2, 1, 2)
    r2.call(-1, np.stack([_tok(0), _tok(1)]), np.stack([_tok(0), _tok(1)]), False)
    with pytest.raises(ValueError):
        r2.truncate(1)  # below committed
    with pytest.raises(ValueError):
        r2.truncate(5)  # beyond length


# ---------------------------------------------------------------------------
# random operation sequences vs the history list
# ---------------------------------------------------------------------------

class History:
    """The independent description: a list of every position's value."""

    def __init__(self):
        self.vals = []
        self.committed = 0

    def append(self, v):
        self.vals.append(v)

    def truncate(self, to):
        del self.vals[to:]

    def expected(self, S, W):
        n = len(self.vals)
        keep = list(range(min(S, n))) + list(range(max(S, n - W), n))
        return {p: self.vals[p] for p in keep}


ops = st.lists(
    st.tuples(st.sampled_from(["spec", "accept", "bulk"]), st.integers(0, 40), st.integers(0, 6)),
    min_size=1, max_size=30)


@settings(max_examples=200, deadline=None)
@given(S=st.integers(0, 4), W=st.integers(1, 9), gmax=st.integers(1, 5), seq=ops)
def test_ring_matches_history_under_random_ops(S, W, gmax, seq):
    r = RingModel(S, W, gmax, 1, 2)
    h = History()
    counter = [0]

    def fresh(n):
        vals = []
        for _ in range(n):
            counter[0] += 1
            vals.append(_tok(counter[0] % 60000))
        return vals

    for kind, a, b in seq:
        if kind == "spec":
            room = gmax - (r.length - r.committed)
            n = min(b, room)
            vals = fresh(n)
            if n:
                r.call(-1, np.stack(vals), np.stack(vals), True)
                for v in vals:
                    h.append(v)
        elif kind == "accept":
            # keep some of the speculative tokens, maybe add one committed token
            pending = r.length - r.committed
            keep = a % (pending + 1)
            to = r.committed + keep
            extra = fresh(b % 2)
            r.call(to, np.stack(extra) if extra else np.zeros((0, 1, 2), np.uint16),
                   np.stack(extra) if extra else np.zeros((0, 1, 2), np.uint16), False)
            h.truncate(to)
            for v in extra:
                h.append(v)
        else:
            if r.length != r.committed:
                continue
            vals = fresh(a)
            if vals:
                r.call(-1, np.stack(vals), np.stack(vals), False)
                for v in vals:
                    h.append(v)
        # the invariant
        exp = h.expected(S, W)
        tags = r.tags()
        assert r.length == len(h.vals)
        assert set(int(t) for t in tags if t >= 0) == set(exp)
        for slot, t in enumerate(tags):
            if t >= 0:
                assert slot == r.slot_of(int(t))
                assert (r.k_array()[slot] == exp[int(t)]).all()
                assert (r.v_array()[slot] == exp[int(t)]).all()


def test_windowed_over_ring_equals_window_over_history():
    """Attention over the ring's entries == attention over the sink+window
    positions of the plain history, after a wrap and a rollback."""
    import torch
    from oracle import attention as A
    S, W, Hkv, Hq, D = 3, 7, 2, 4, 8
    rng = np.random.default_rng(30)
    hist = torch.randn(40, Hkv, D, generator=torch.Generator().manual_seed(31)).to(torch.bfloat16)
    bits = hist.view(torch.int16).numpy().view(np.uint16)
    r = RingModel(S, W, 3, Hkv, D)
    r.call(-1, bits[:30], bits[:30], False)
    r.call(-1, bits[30:33], bits[30:33], True)
    r.call(31, bits[:0], bits[:0], False)
    q = rng.standard_normal((1, Hq, D))
    o_ring, l_ring = A.draft_attn_windowed(q, [r], 0.5)
    # the same history laid out as a paged pool with page size 1
    kp = hist.double().numpy()[:31, :, None, :]
    table = np.arange(31)[None]
    o_hist, l_hist = A.draft_attn_windowed_paged(q, kp, kp, table, [31], 1, S, W, 0.5)
    np.testing.assert_array_equal(o_ring, o_hist)
    np.testing.assert_array_equal(l_ring, l_hist)

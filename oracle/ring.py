"""The compact draft ring buffer, modelled as a plain Python list.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix: under Windowed-MTP the draft reads only the attention sink
and a sliding window, and a compact ring buffer that stores just those entries
turns the smaller working set into freed KV memory, in place of the whole
draft KV pool ("Windowed-MTP ..." arxivlens view, *Abstract*; *Results* and
*Technical contributions* of its analysis; readpriors post, *What happened*).

What the pages leave open, and the readings taken here:

* Capacity: ``S + W`` data slots (S sinks, W window entries).
* Slot of position ``p``: ``p`` for ``p < S``; ``S + (p - S) mod W`` after.
  During the first fill this is the identity, so a ring that has never wrapped
  holds position ``p`` in slot ``p``.  Unused slots carry tag ``-1``.
* Speculative draft tokens: a draft step appends its token before the target
  has accepted it.  If the target later rejects it, the window entry it
  evicted is still needed.  So each speculative append first saves the entry
  it overwrites into an undo log (at most ``gamma_max`` entries since the last
  commit); a truncation to length ``n'`` restores those entries newest first.
  A non-speculative call commits: the committed length becomes the current
  length and the undo log empties.
* Invariant after any sequence of calls: the ring holds exactly positions
  ``{0 .. min(S, len)-1} U {max(S, len-W) .. len-1}``, each at its slot, with
  the K/V last appended for that position.

Every operation is the sequential, one-token-at-a-time definition; nothing is
batched or reordered.
"""

from __future__ import annotations

import numpy as np


class RingModel:
    """One sequence's ring: a list of ``S + W`` entries ``(tag, k, v)``.

    ``k`` and ``v`` are ``[Hkv, D]`` arrays of whatever dtype the caller uses
    (the tests keep the raw bf16 bit patterns as ``uint16`` so comparisons are
    bit-exact).
    """

    def __init__(self, sinks: int, window: int, gamma_max: int, num_kv_heads: int,
                 head_dim: int, dtype=np.uint16):
        if sinks < 0 or window < 1 or gamma_max < 0:
            raise ValueError("need sinks >= 0, window >= 1, gamma_max >= 0")
        self.S = int(sinks)
        self.W = int(window)
        self.gamma_max = int(gamma_max)
        self.num_kv_heads = int(num_kv_heads)
        self.head_dim = int(head_dim)
        self.dtype = dtype
        zero = np.zeros((num_kv_heads, head_dim), dtype=dtype)
        self.entries = [(-1, zero.copy(), zero.copy()) for _ in range(self.S + self.W)]
        self.length = 0
        self.committed = 0
        # undo[j] = (slot, old_tag, old_k, old_v) saved by the j-th speculative
        # append since the last commit (position committed + j).
        self.undo = []

    # -- layout ------------------------------------------------------------
    @property
    def slots(self) -> int:
        return self.S + self.W

    def slot_of(self, p: int) -> int:
        return p if p < self.S else self.S + (p - self.S) % self.W

    def expected_tags(self, length: int | None = None) -> set:
        """Positions the ring must hold at ``length`` (the invariant)."""
        n = self.length if length is None else int(length)
        head = range(min(self.S, n))
        tail = range(max(self.S, n - self.W), n)
        return set(head) | set(tail)

    # -- the operations ------------------------------------------------------
    def append_one(self, k: np.ndarray, v: np.ndarray, speculative: bool) -> None:
        p = self.length
        s = self.slot_of(p)
        if speculative:
            if len(self.undo) >= self.gamma_max:
                raise ValueError("undo log full: more speculative appends than gamma_max")
            old_tag, old_k, old_v = self.entries[s]
            self.undo.append((s, old_tag, old_k, old_v))
        self.entries[s] = (p, np.array(k, dtype=self.dtype, copy=True),
                           np.array(v, dtype=self.dtype, copy=True))
        self.length = p + 1

    def truncate(self, to: int) -> None:
        """Roll speculative entries back until ``length == to``."""
        to = int(to)
        if to < self.committed or to > self.length:
            raise ValueError(f"truncate_to {to} outside [committed {self.committed}, length {self.length}]")
        while self.length > to:
            s, tag, k, v = self.undo.pop()
            self.entries[s] = (tag, k, v)
            self.length -= 1

    def commit(self) -> None:
        self.committed = self.length
        self.undo = []

    def call(self, truncate_to: int, k_new: np.ndarray, v_new: np.ndarray,
             speculative: bool) -> None:
        """One library call: optional truncation, then appends, then (if not
        speculative) a commit.  ``k_new``/``v_new`` are ``[n_new, Hkv, D]``."""
        if truncate_to is not None and truncate_to >= 0:
            self.truncate(truncate_to)
        for j in range(k_new.shape[0]):
            self.append_one(k_new[j], v_new[j], speculative)
        if not speculative:
            self.commit()

    # -- views ----------------------------------------------------------------
    def tags(self) -> np.ndarray:
        return np.asarray([e[0] for e in self.entries], dtype=np.int64)

    def k_array(self) -> np.ndarray:
        return np.stack([e[1] for e in self.entries])  # [S+W, Hkv, D]

    def v_array(self) -> np.ndarray:
        return np.stack([e[2] for e in self.entries])

    def attended_entries(self):
        """(tags, K ``[n, Hkv, D]``, V) of the entries in the sink + window set,
        ordered by position."""
        want = self.expected_tags()
        chosen = sorted((e for e in self.entries if e[0] in want), key=lambda e: e[0])
        if not chosen:
            z = np.zeros((0, self.num_kv_heads, self.head_dim), dtype=self.dtype)
            return np.zeros(0, np.int64), z, z
        tags = np.asarray([e[0] for e in chosen], dtype=np.int64)
        return tags, np.stack([e[1] for e in chosen]), np.stack([e[2] for e in chosen])

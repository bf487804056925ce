"""fp64 softmax attention over explicit attended-position sets.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

What the path computes, read from the pages:

* Native MTP draft attention -- one decode query per draft step attends over
  the *entire* KV cache of the draft layer, once for each of the gamma draft
  forwards of a decode step ("Windowed-MTP ..." arxivlens view, *Abstract*;
  howtospark case study, *Background*).
* Windowed-MTP draft attention -- the same query attends only to the attention
  sink (the first S positions) plus a sliding window (the last W positions):
  a StreamingLLM-style window applied to the draft only (arxivlens view,
  *Abstract*; readpriors post, *What happened*).
* Verify -- the target scores gamma+1 tokens in one batched forward with
  attention over the whole context, which is what keeps the target's output
  distribution unchanged (arxivlens view, *Abstract*; howtospark case study,
  *Method*, where one cycle is three draft forwards plus one batched verify).  Query i of the
  verify block sits at position ``kv_len - num_q + i`` and attends causally to
  positions ``0 .. kv_len - num_q + i``.

The attention itself is the textbook definition, written out once in
``attend``: scores ``s_t = sm_scale * <q, k_t>``, weights
``p_t = exp(s_t - max s) / sum exp(s - max s)``, output ``o = sum_t p_t v_t``
and log-sum-exp ``lse = max s + log sum exp(s - max s)``.  An empty attended
set gives ``o = 0`` and ``lse = -inf`` (a reading: the pages never reach it).

GQA: query head ``h`` reads KV head ``h // G`` with ``G = Hq / Hkv`` (a
reading; the pages give no head mapping).

Paged KV: position ``p`` of sequence ``b`` lives in page
``page_table[b, p // P]`` at row ``p % P``; pools are ``[pages, Hkv, P, D]``.
"""

from __future__ import annotations

import numpy as np

EMPTY_LSE = -np.inf


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns (uint16) to float64, exactly.

    A bf16 value is the upper half of the IEEE binary32 value with the same
    bits, so shifting into the high half and reading binary32 is exact.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _as_f64(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x)
    return bf16_bits_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)


# --------------------------------------------------------------------------
# attended sets
# --------------------------------------------------------------------------

def full_positions(kv_len: int) -> np.ndarray:
    """Native draft: every cached position ``0 .. kv_len-1``.

    arxivlens view, *Abstract* (full KV cache per draft forward); howtospark
    case study, *Background* (the draft reads the whole cache every step).
    """
    return np.arange(int(kv_len), dtype=np.int64)


def window_positions(length: int, sinks: int, window: int) -> np.ndarray:
    """Windowed draft: the first ``sinks`` positions plus the last ``window``.

    arxivlens view, *Abstract* (StreamingLLM-style sink plus window, applied
    to the draft alone); readpriors post, *What happened* (the window keeps
    the draft's KV working set the same size at any context).  Reading: the window is the last W positions of the cache
    *after* the current token was appended, so the current token is always
    attended.  Sink and window never overlap: the window starts at
    ``max(sinks, length - window)``.
    """
    length = int(length)
    sink_end = min(int(sinks), length)
    win_start = max(int(sinks), length - int(window))
    head = np.arange(sink_end, dtype=np.int64)
    tail = np.arange(win_start, length, dtype=np.int64) if win_start < length else np.zeros(0, np.int64)
    return np.concatenate([head, tail])


def causal_positions(kv_len: int, num_q: int, i: int) -> np.ndarray:
    """Verify query ``i`` of ``num_q``: positions ``0 .. kv_len - num_q + i``.

    arxivlens view, *Abstract* (full-context verification); the causal limit is
    the standard one for a batch of new tokens appended at the end.
    """
    last = int(kv_len) - int(num_q) + int(i)
    return np.arange(max(last + 1, 0), dtype=np.int64)


# --------------------------------------------------------------------------
# the attention definition
# --------------------------------------------------------------------------

def attend(q: np.ndarray, keys: np.ndarray, values: np.ndarray, sm_scale: float):
    """Softmax attention of one query over ``keys``/``values`` (fp64).

    q ``[D]``, keys ``[n, D]``, values ``[n, D]`` -> (o ``[D]``, lse scalar).
    """
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    n = keys.shape[0]
    if n == 0:
        return np.zeros(q.shape[-1], dtype=np.float64), EMPTY_LSE
    s = float(sm_scale) * (keys @ q)
    m = s.max()
    p = np.exp(s - m)
    l = p.sum()
    o = (p @ values) / l
    lse = m + np.log(l)
    return o, float(lse)


def attend_rows(qs: np.ndarray, keys: np.ndarray, values: np.ndarray, sm_scale: float):
    """``attend`` for several queries over the same keys: qs ``[R, D]``."""
    outs, lses = [], []
    for r in range(qs.shape[0]):
        o, lse = attend(qs[r], keys, values, sm_scale)
        outs.append(o)
        lses.append(lse)
    return np.stack(outs), np.asarray(lses, dtype=np.float64)


def attend_prefixes(qs: np.ndarray, keys: np.ndarray, values: np.ndarray, lengths, sm_scale: float):
    """Row ``r`` of ``qs`` attends the first ``lengths[r]`` keys (fp64).

    The ``attend`` definition for several queries whose key sets are prefixes
    of one key list: a causal verify block (query ``i`` sees positions
    ``0 .. n+i``) or draft steps at growing lengths.  One score matrix serves
    every row; scores past a row's length are excluded before its maximum,
    exponentials and sums are taken.  qs ``[R, D]``, keys/values ``[n, D]``,
    lengths ``[R]`` with ``0 <= lengths[r] <= n`` -> (o ``[R, D]``, lse
    ``[R]``); an empty prefix gives (0, -inf).
    """
    qs = np.asarray(qs, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    lengths = np.asarray(lengths, dtype=np.int64).reshape(-1)
    R, D = qs.shape
    n = keys.shape[0]
    if lengths.shape[0] != R or (lengths < 0).any() or (lengths > n).any():
        raise ValueError("need one length per row, each in [0, n]")
    o = np.zeros((R, D), dtype=np.float64)
    lse = np.full(R, EMPTY_LSE, dtype=np.float64)
    live = lengths > 0
    if n == 0 or not live.any():
        return o, lse
    s = float(sm_scale) * (keys @ qs.T)                          # [n, R]
    s[np.arange(n)[:, None] >= lengths[None, :]] = -np.inf        # outside the prefix
    m = np.where(live, s.max(axis=0), 0.0)
    p = np.exp(s - m[None, :])                                    # exp(-inf) = 0
    l = p.sum(axis=0)
    o[live] = (p.T @ values)[live] / l[live, None]
    lse[live] = m[live] + np.log(l[live])
    return o, lse


def gather_paged(pool: np.ndarray, table_row: np.ndarray, positions: np.ndarray,
                 page_size: int, kv_head: int) -> np.ndarray:
    """Rows of one KV head at ``positions`` from a ``[pages, Hkv, P, D]`` pool."""
    positions = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(table_row, dtype=np.int64)[positions // page_size]
    return pool[pages, kv_head, positions % page_size, :]


def _group(hq: int, hkv: int) -> int:
    if hkv <= 0 or hq % hkv != 0:
        raise ValueError(f"query heads {hq} not a multiple of kv heads {hkv}")
    return hq // hkv


# --------------------------------------------------------------------------
# the three attention calls of a decode step
# --------------------------------------------------------------------------

def draft_attn_full(q, k_pool, v_pool, page_table, kv_len, page_size, sm_scale):
    """Native MTP draft attention (one query per sequence and head).

    q ``[B, Hq, D]``; pools ``[pages, Hkv, P, D]``; page_table ``[B, max_pages]``;
    kv_len ``[B]`` (includes the token just appended).  Returns o ``[B, Hq, D]``
    and lse ``[B, Hq]``.  arxivlens view, *Abstract*.
    """
    B, Hq, D = q.shape
    Hkv = k_pool.shape[1]
    G = _group(Hq, Hkv)
    o = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), EMPTY_LSE)
    for b in range(B):
        pos = full_positions(kv_len[b])
        for kvh in range(Hkv):
            K = gather_paged(k_pool, page_table[b], pos, page_size, kvh)
            V = gather_paged(v_pool, page_table[b], pos, page_size, kvh)
            for g in range(G):
                h = kvh * G + g
                o[b, h], lse[b, h] = attend(q[b, h], K, V, sm_scale)
    return o, lse


def draft_attn_windowed_paged(q, k_pool, v_pool, page_table, kv_len, page_size,
                              sinks, window, sm_scale):
    """Windowed draft attention over a full paged history (sink + window set).

    The same attended set as ``draft_attn_windowed`` but read from the complete
    paged cache instead of the compact ring; used to check the ring against the
    history.  arxivlens view, *Abstract*; readpriors post, *What happened*.
    """
    B, Hq, D = q.shape
    Hkv = k_pool.shape[1]
    G = _group(Hq, Hkv)
    o = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), EMPTY_LSE)
    for b in range(B):
        pos = window_positions(kv_len[b], sinks, window)
        for kvh in range(Hkv):
            K = gather_paged(k_pool, page_table[b], pos, page_size, kvh)
            V = gather_paged(v_pool, page_table[b], pos, page_size, kvh)
            for g in range(G):
                h = kvh * G + g
                o[b, h], lse[b, h] = attend(q[b, h], K, V, sm_scale)
    return o, lse


def draft_attn_windowed(q, rings, sm_scale):
    """Windowed draft attention over each sequence's compact ring buffer.

    ``rings`` is a list of ``RingModel`` (one per sequence).  The attended keys
    are the ring entries whose position tag lies in the sink + window set of
    the ring's current length -- after any append / rollback sequence that is
    every occupied entry.  arxivlens view, *Abstract* (the compact ring buffer
    that keeps only the sink and window entries); readpriors post, *What
    happened*.
    """
    B, Hq, D = q.shape
    o = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), EMPTY_LSE)
    for b in range(B):
        tags, K, V = rings[b].attended_entries()
        Hkv = rings[b].num_kv_heads
        G = _group(Hq, Hkv)
        for kvh in range(Hkv):
            for g in range(G):
                h = kvh * G + g
                o[b, h], lse[b, h] = attend(q[b, h], _as_f64(K[:, kvh, :]),
                                            _as_f64(V[:, kvh, :]), sm_scale)
    return o, lse


def verify_attn(q, k_pool, v_pool, page_table, kv_len, page_size, sm_scale):
    """Target verify attention: ``num_q = gamma+1`` causal queries per sequence.

    q ``[B, Qn, Hq, D]``; kv_len ``[B]`` includes the ``Qn`` new tokens.  Query
    ``i`` attends ``causal_positions(kv_len, Qn, i)``.  Returns o
    ``[B, Qn, Hq, D]`` and lse ``[B, Qn, Hq]``.  arxivlens view, *Abstract*.
    """
    B, Qn, Hq, D = q.shape
    Hkv = k_pool.shape[1]
    G = _group(Hq, Hkv)
    o = np.zeros((B, Qn, Hq, D))
    lse = np.full((B, Qn, Hq), EMPTY_LSE)
    for b in range(B):
        for i in range(Qn):
            pos = causal_positions(kv_len[b], Qn, i)
            for kvh in range(Hkv):
                K = gather_paged(k_pool, page_table[b], pos, page_size, kvh)
                V = gather_paged(v_pool, page_table[b], pos, page_size, kvh)
                for g in range(G):
                    h = kvh * G + g
                    o[b, i, h], lse[b, i, h] = attend(q[b, i, h], K, V, sm_scale)
    return o, lse


# --------------------------------------------------------------------------
# split-KV partials and their log-sum-exp combine
# --------------------------------------------------------------------------

def split_partials(q, keys, values, bounds, sm_scale):
    """Attention of one query over each contiguous chunk ``keys[b0:b1]``.

    ``bounds`` is a list of ``(b0, b1)``.  Returns part_o ``[nsplit, D]`` and
    part_lse ``[nsplit]``; an empty chunk gives ``(0, -inf)``.  The split-KV
    decomposition is not on the pages; it is the standard flash-decoding
    identity that the combine below undoes.
    """
    outs, lses = [], []
    for b0, b1 in bounds:
        o, lse = attend(q, keys[b0:b1], values[b0:b1], sm_scale)
        outs.append(o)
        lses.append(lse)
    return np.stack(outs), np.asarray(lses, dtype=np.float64)


def splitkv_combine(part_o, part_lse):
    """Merge split partials: ``o = sum_s e^{lse_s - m} o_s / sum_s e^{lse_s - m}``.

    part_o ``[..., nsplit, D]``, part_lse ``[..., nsplit]`` -> o ``[..., D]``,
    lse ``[...]`` with ``lse = m + log sum_s e^{lse_s - m}``, ``m = max_s lse_s``.
    Splits with ``lse = -inf`` (empty) carry no weight; if every split is empty
    the result is ``(0, -inf)``.
    """
    part_o = np.asarray(part_o, dtype=np.float64)
    part_lse = np.asarray(part_lse, dtype=np.float64)
    lead = part_lse.shape[:-1]
    D = part_o.shape[-1]
    o = np.zeros(lead + (D,))
    lse = np.full(lead, EMPTY_LSE)
    for idx in np.ndindex(*lead) if lead else [()]:
        ls = part_lse[idx]
        finite = np.isfinite(ls)
        if not finite.any():
            continue
        m = ls[finite].max()
        w = np.where(finite, np.exp(np.where(finite, ls, m) - m), 0.0)
        tot = w.sum()
        o[idx] = (w[:, None] * part_o[idx]).sum(axis=0) / tot
        lse[idx] = m + np.log(tot)
    return o, lse

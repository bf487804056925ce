"""GPU parity of the attention kernels on the inputs that reach their
hardest numerics, against the fp64 oracle (mostly the tcgen05 verify).

The verify kernel keeps a per-row reference maximum that it raises only when
a tile beats it by more than 2^8, and then rescales that row of the
accumulator in tensor memory; its value product runs with the weights in
fp16.  Seeded Gaussian inputs rarely reach either: these tests plant keys
that do.

* Late high scores: keys aligned with chosen query rows are planted so that a
  row's score jumps by 12..40 log2 units several times inside one split,
  across tiles, at the first and last token of splits and in the split that
  ends the context.  Every jump moves that row's reference and rescales it.
* Falling scores: the largest score of a row sits at the first token of its
  split and later planted scores are smaller, so the reference never moves
  and the later weights are tiny.
* A large softmax scale: sm_scale 8x the default makes every row peaked.
* An attention sink over a flat sea: one key carries most of the weight of
  its split and a hundred thousand nearly equal keys share the rest.  Their
  weights are ~2^-20 of the sink's, where fp16 numbers are subnormal unless
  the kernel keeps them in the normal range.
* A planted key among the new tokens is seen only by the queries at or after
  its position (causal limit on the last tile).
* A flat sea of a million keys in one split (native draft, 64 sequences): an
  accumulation of a million nearly equal products of one sign.

The attention definition is the pages' (arxivlens view, Abstract: verification
stays full-context); the oracle is plain fp64 softmax attention.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import speculative_decode_draft_b200 as w

from _helpers import assert_close, assert_lse_close, cache_of, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LOG2E = 1.4426950408889634
TILE = 64


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


def _nsplit(p, B, num_q, max_pages):
    """The split count of a verify call, recovered from its workspace size
    (fp32 partial outputs then partial LSEs, each padded to 256 bytes)."""
    need = w.workspace_bytes("verify", p, B, num_q=num_q, max_pages=max_pages)
    rows = B * num_q * p.num_heads_q
    pad = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for ns in range(1, 4097):
        if pad(rows * ns * p.head_dim * 4) + pad(rows * ns * 4) == need:
            return ns
    raise AssertionError("split count not found")


def _split_tiles(n_tok, nsplit):
    ntiles = -(-n_tok // TILE)
    tps = -(-ntiles // nsplit)
    return [(s * tps, min((s + 1) * tps, ntiles)) for s in range(nsplit) if s * tps < ntiles]


def _plant(kv, pos, kvh, vec):
    """Overwrite K at sequence 0, position `pos`, KV head `kvh` (bf16)."""
    P = kv.page_size
    pg = int(kv.page_table[0, pos // P])
    kv.k_pool[pg, kvh, pos % P] = vec.to(torch.bfloat16)


def _aligned_key(q_row, target_log2, sm_scale):
    """A key whose score against `q_row` is about `target_log2` (log2 units)."""
    qf = q_row.float()
    alpha = target_log2 / (float((qf * qf).sum()) * sm_scale * LOG2E)
    return qf * alpha


def _run_and_check(p, qv, kv, sm_scale, what):
    status = w.new_status(DEV)
    out, lse = w.verify_attn(p, qv, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"{what}: status {int(status.item()):#x}"
    ref, ref_lse = oracle.verify_attn(f64(qv), f64(kv.k_pool), f64(kv.v_pool), kv.page_table.cpu().numpy(),
                                      kv.kv_len.cpu().numpy(), kv.page_size, sm_scale)
    assert_close(f64(out), ref, what)
    assert_lse_close(f64(lse), ref_lse, what)
    return out


def _setup(num_q, G, n_commit, seed, Hkv=2, D=256, P=64, sm_scale=0.0):
    Hq = G * Hkv
    n = n_commit + num_q
    p = w.params(Hq, Hkv, D, page_size=P, gamma_max=num_q - 1, sm_scale=sm_scale)
    kv = synth.paged_kv(seed, 1, Hkv, D, P, [n], n + 2 * P, True, True, device=DEV)
    qv = synth.queries(seed + 1, (1, num_q, Hq, D), device=DEV)
    return p, kv, qv, n


@pytest.mark.parametrize("num_q,G", [(4, 8), (6, 8), (9, 8)])
def test_verify_late_high_scores_move_the_reference(num_q, G):
    """Scores that rise by > 2^8 several times inside splits, across tiles and
    at split boundaries (tcgen05 path: 32 / 48 / 72 rows)."""
    p, kv, qv, n = _setup(num_q, G, 32768, 400 + num_q)
    scale = 1 / 16
    splits = _split_tiles(n, _nsplit(p, 1, num_q, kv.page_table.shape[1]))
    assert len(splits) >= 8
    Hkv = p.num_heads_kv
    rng = np.random.default_rng(401)
    chosen = [0, 1, len(splits) // 2, len(splits) - 2, len(splits) - 1]
    for si in chosen:
        t0, t1 = splits[si]
        first, last = t0 * TILE, min(t1 * TILE, n - num_q) - 1  # committed positions only
        inner = [first, first + TILE // 2, (t0 + (t1 - t0) // 2) * TILE + 5, last - TILE - 3, last]
        inner = sorted({x for x in inner if first <= x <= last})
        for kvh in range(Hkv):
            i, g = int(rng.integers(num_q)), int(rng.integers(G))
            row = qv[0, i, kvh * G + g]
            for j, pos in enumerate(inner):  # rising: each beats the last by 12 log2 units
                _plant(kv, pos, kvh, _aligned_key(row, 12.0 * (j + 1), scale))
    _run_and_check(p, qv, kv, scale, f"late high scores q={num_q} G={G}")


def test_verify_falling_scores_keep_the_reference():
    """The largest score of a row at the first token of its split, smaller
    planted scores later: the reference never moves, later weights are
    2^-12 .. 2^-36 of the first."""
    num_q, G = 4, 8
    p, kv, qv, n = _setup(num_q, G, 32768, 420)
    scale = 1 / 16
    splits = _split_tiles(n, _nsplit(p, 1, num_q, kv.page_table.shape[1]))
    for si in (0, 3, len(splits) // 2, len(splits) - 1):
        t0, t1 = splits[si]
        first, last = t0 * TILE, min(t1 * TILE, n - num_q) - 1
        for kvh in range(p.num_heads_kv):
            row = qv[0, si % num_q, kvh * G + (si % G)]
            _plant(kv, first, kvh, _aligned_key(row, 48.0, scale))
            for j, pos in enumerate((first + TILE + 1, (first + last) // 2, last)):
                if first < pos <= last:
                    _plant(kv, pos, kvh, _aligned_key(row, 36.0 - 12.0 * j, scale))
    _run_and_check(p, qv, kv, scale, "falling scores")


@pytest.mark.parametrize("sm_scale,num_q", [(0.5, 4), (0.5, 9), (1.0, 4)])
def test_verify_large_softmax_scale(sm_scale, num_q):
    """sm_scale 8x and 16x the default 1/16: every row is peaked and the
    reference moves often across the context."""
    p, kv, qv, n = _setup(num_q, 8, 32768, 430 + num_q, sm_scale=sm_scale)
    _run_and_check(p, qv, kv, sm_scale, f"sm_scale {sm_scale} q={num_q}")


def test_verify_plant_among_new_tokens_is_causal():
    """A dominant key, aligned with query 3 of the first head of each KV head,
    at the position of verify query 2: queries 0 and 1 must not see it,
    query 3 of that head is dominated by it."""
    num_q, G = 4, 8
    p, kv, qv, n = _setup(num_q, G, 8192, 440)
    for kvh in range(p.num_heads_kv):
        _plant(kv, n - num_q + 2, kvh, _aligned_key(qv[0, 3, kvh * G], 40.0, 1 / 16))
    _run_and_check(p, qv, kv, 1 / 16, "plant among the new tokens")


@pytest.mark.timeout(900)
def test_verify_sink_over_a_flat_sea():
    """An attention sink at position 0 over 1,048,576 nearly equal keys, in
    64 identical sequences: with 64 sequences a split spans ~116K tokens, so
    the split holding the sink also holds a large part of the sea.  Every
    query row scores the sink 20.39 log2 units above the sea; relative to
    the sink a sea weight is 12.25 steps of fp16's smallest subnormal
    (2^-24), where a plain fp16 rounding would bias every one of them the
    same way.  The sea's values have mean 2 and the sink's -2, so such a
    bias shows in the output."""
    num_q, G, Hkv, D, P, B = 4, 8, 2, 256, 64, 64
    Hq = G * Hkv
    n = (1 << 20) + num_q
    sea_pages = 64
    npg = -(-n // P)
    # physical pages: 0 holds the sink (position 0) and sea keys after it,
    # 1..64 hold the sea and back every further logical page in turn, the last
    # page holds the new tokens (sea-like as well)
    num_pages = 2 + sea_pages
    gen = torch.Generator(device=DEV).manual_seed(450)
    k_pool = (torch.randn(num_pages, Hkv, P, D, generator=gen, device=DEV) * 1e-3).to(torch.bfloat16)
    v_pool = (2.0 + 0.1 * torch.randn(num_pages, Hkv, P, D, generator=gen, device=DEV)).to(torch.bfloat16)
    row = torch.empty(npg, dtype=torch.int32)
    row[0] = 0
    row[1:] = 1 + torch.arange(npg - 1, dtype=torch.int32) % sea_pages
    row[(n - num_q) // P:] = num_pages - 1
    table = row[None].expand(B, npg).contiguous()
    kv = synth.PagedKV(k_pool, v_pool, table.to(DEV), torch.full((B,), n, dtype=torch.int32, device=DEV), P)
    q0 = synth.queries(451, (Hkv, D), device=DEV)
    qv = q0[None, None, :, None, :].expand(B, num_q, Hkv, G, D).reshape(B, num_q, Hq, D).contiguous()
    for kvh in range(Hkv):
        _plant(kv, 0, kvh, _aligned_key(q0[kvh], 20.39, 1 / 16))
        v_pool[0, kvh, 0] = (-2.0 + 0.1 * torch.randn(D, generator=gen, device=DEV)).to(torch.bfloat16)
    p = w.params(Hq, Hkv, D, page_size=P, gamma_max=num_q - 1)
    assert _nsplit(p, B, num_q, npg) <= 16
    status = w.new_status(DEV)
    out, lse = w.verify_attn(p, qv, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # every sequence has the same inputs, so one oracle result serves all of
    # them; one score matrix per KV head, prefix lengths = causal limits
    tbl = row.numpy().astype(np.int64)
    pos = np.arange(n)
    lengths = np.repeat([len(oracle.causal_positions(n, num_q, i)) for i in range(num_q)], G)
    kp, vp = f64(k_pool), f64(v_pool)
    for kvh in range(Hkv):
        K = kp[tbl[pos // P], kvh, pos % P]
        V = vp[tbl[pos // P], kvh, pos % P]
        rows = slice(kvh * G, (kvh + 1) * G)
        qs = f64(qv[0, :, rows]).reshape(num_q * G, D)
        ref, ref_lse = oracle.attend_prefixes(qs, K, V, lengths, 1 / 16)
        del K, V
        got = f64(out[:, :, rows]).reshape(B, num_q * G, D)
        got_lse = f64(lse[:, :, rows]).reshape(B, num_q * G)
        assert_close(got, np.broadcast_to(ref, got.shape), f"sink over a flat sea kvh {kvh}")
        for b in range(B):
            assert_lse_close(got_lse[b], ref_lse, f"sink over a flat sea kvh {kvh} seq {b}")


@pytest.mark.timeout(900)
def test_native_draft_flat_sea_in_one_long_split():
    """The native draft of 64 sequences of 1,048,576 tokens runs one split per
    sequence and KV head, so one CTA accumulates a whole million-token
    context.  With nearly equal weights and values of one sign (mean 2) an
    accumulation that drops the low-order bits of each product against the
    running sum would bias the result by ~0.5%; the kernel's runs of 16,384
    tokens keep it inside the parity bar."""
    G, Hkv, D, P, B = 8, 2, 256, 64, 64
    Hq = G * Hkv
    n = 1 << 20
    npg = n // P
    num_pages = 65
    gen = torch.Generator(device=DEV).manual_seed(460)
    k_pool = (torch.randn(num_pages, Hkv, P, D, generator=gen, device=DEV) * 1e-3).to(torch.bfloat16)
    v_pool = (2.0 + 0.1 * torch.randn(num_pages, Hkv, P, D, generator=gen, device=DEV)).to(torch.bfloat16)
    row = torch.arange(npg, dtype=torch.int32) % num_pages
    kv = synth.PagedKV(k_pool, v_pool, row[None].expand(B, npg).contiguous().to(DEV),
                       torch.full((B,), n, dtype=torch.int32, device=DEV), P)
    q0 = synth.queries(461, (Hq, D), device=DEV)
    q = q0[None].expand(B, Hq, D).contiguous()
    p = w.params(Hq, Hkv, D, page_size=P)
    status = w.new_status(DEV)
    out, lse = w.draft_attn_full(p, q, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    tbl = row.numpy().astype(np.int64)
    pos = np.arange(n)
    kp, vp = f64(k_pool), f64(v_pool)
    for kvh in range(Hkv):
        K = kp[tbl[pos // P], kvh, pos % P]
        V = vp[tbl[pos // P], kvh, pos % P]
        rows = slice(kvh * G, (kvh + 1) * G)
        ref, ref_lse = oracle.attend_prefixes(f64(q0[rows]), K, V, np.full(G, n), 1 / 16)
        del K, V
        got = f64(out[:, rows])
        assert_close(got, np.broadcast_to(ref, got.shape), f"native draft flat sea kvh {kvh}")
        for b in range(0, B, 21):
            assert_lse_close(f64(lse[b, rows]), ref_lse, f"native draft flat sea kvh {kvh} seq {b}")

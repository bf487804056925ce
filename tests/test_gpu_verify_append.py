"""GPU parity of wmtp_verify_attn_append: the paged write of a verify
layer's new tokens fused into the verify call.

The call must leave the pools exactly as wmtp_paged_write at positions
kv_len - num_q .. kv_len - 1 would (bit for bit), and return what
wmtp_verify_attn over those pools returns: checked against the fp64 oracle
and, bit for bit, against the two-call sequence on a copy of the same
pools.  The cases put the new rows inside one tile, across a tile and a page
boundary (two splits' tiles), in tile 0 of a short sequence, on 16-token
pages (four TMA boxes a tile), in ragged batches, on 72-row blocks (M = 128),
and on the mma.sync verify's shapes (head_dim 64, 8 rows), where the write
is its own launch.  The attention definition is the pages' (arxivlens view,
Abstract: verification stays full-context; howtospark case study, Method: a
verify layer appends its gamma+1 tokens); the oracle is plain fp64 softmax
attention.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
import speculative_decode_draft_b200 as w

from _helpers import assert_close, assert_lse_close, bits, cache_of, f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    w.load()


def _clone(kv):
    return synth.PagedKV(kv.k_pool.clone(), kv.v_pool.clone(), kv.page_table, kv.kv_len, kv.page_size)


CASES = [
    # num_q, G, D, page, lengths (kv_len, new tokens included)
    (4, 8, 256, 64, [32768 + 4]),            # new rows inside one tile
    (4, 8, 256, 64, [64 * 100 + 2]),         # rows 6398..6401: across a tile and a page boundary
    (4, 8, 256, 64, [60]),                   # all in tile 0 (issued before the block barrier)
    (4, 8, 256, 16, [5000 + 4]),             # 16-token pages: four boxes a tile
    (6, 8, 256, 256, [40000, 123, 70001]),   # ragged batch, 256-token pages
    (9, 8, 256, 64, [30000 + 9, 777]),       # 72 rows per KV head: M = 128
    (4, 4, 64, 16, [2048 + 4]),              # head_dim 64: the mma.sync verify, write launched in front
    (2, 4, 256, 64, [9000]),                 # 8 rows: the mma.sync verify
]


@pytest.mark.parametrize("num_q,G,D,P,lengths", CASES)
def test_verify_append_matches_write_then_verify(num_q, G, D, P, lengths):
    Hkv = 2
    Hq = G * Hkv
    B = len(lengths)
    seed = 900 + num_q * 7 + D + P + B
    p = w.params(Hq, Hkv, D, page_size=P, gamma_max=num_q - 1)
    kv = synth.paged_kv(seed, B, Hkv, D, P, lengths, max(lengths) + 2 * P, True, True, device=DEV)
    q = synth.queries(seed + 1, (B, num_q, Hq, D), device=DEV)
    kn, vn = synth.new_tokens(seed + 2, B, num_q, Hkv, D, device=DEV, kv_scale=True)
    two = _clone(kv)

    # expected pools: the new rows at the last num_q positions of each sequence
    exp_k, exp_v = bits(kv.k_pool).copy(), bits(kv.v_pool).copy()
    pt = kv.page_table.cpu().numpy()
    kb, vb = bits(kn), bits(vn)
    for b, n in enumerate(lengths):
        for j in range(num_q):
            pos = n - num_q + j
            exp_k[pt[b, pos // P], :, pos % P] = kb[b, j]
            exp_v[pt[b, pos // P], :, pos % P] = vb[b, j]

    status = w.new_status(DEV)
    out, lse = w.verify_attn_append(p, q, kn, vn, cache_of(kv), status=status)
    # the two-call sequence on a copy of the pools
    pos0 = (kv.kv_len - num_q).to(torch.int32).contiguous()
    w.paged_write(p, cache_of(two), pos0, kn, vn, status=status)
    out2, lse2 = w.verify_attn(p, q, cache_of(two), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    np.testing.assert_array_equal(bits(kv.k_pool), exp_k)
    np.testing.assert_array_equal(bits(kv.v_pool), exp_v)
    assert torch.equal(out, out2) and torch.equal(lse, lse2), "fused and two-call results differ"
    ref, ref_lse = oracle.verify_attn(f64(q), f64(kv.k_pool), f64(kv.v_pool), pt, kv.kv_len.cpu().numpy(), P,
                                      1 / np.sqrt(D))
    assert_close(f64(out), ref, f"append q={num_q} G={G} D={D} P={P} {lengths}")
    assert_lse_close(f64(lse), ref_lse, f"append q={num_q} G={G} D={D} P={P} {lengths}")


def test_verify_append_skips_rows_on_bad_pages():
    """A new row on a page outside the pool is not written and raises
    WMTP_DEV_PAGE_OOB; the rows on good pages are written."""
    num_q, G, Hkv, D, P = 4, 8, 2, 256, 64
    n = 64 * 10 + 2  # rows 638, 639 on logical page 9, rows 640, 641 on page 10
    p = w.params(G * Hkv, Hkv, D, page_size=P, gamma_max=num_q - 1)
    kv = synth.paged_kv(960, 1, Hkv, D, P, [n], n + 2 * P, True, True, device=DEV)
    q = synth.queries(961, (1, num_q, G * Hkv, D), device=DEV)
    kn, vn = synth.new_tokens(962, 1, num_q, Hkv, D, device=DEV)
    kv.page_table[0, 10] = kv.k_pool.shape[0] + 5
    before = bits(kv.k_pool).copy()
    status = w.new_status(DEV)
    w.verify_attn_append(p, q, kn, vn, cache_of(kv), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & w._lib.DEV_PAGE_OOB
    after = bits(kv.k_pool)
    pg9 = int(kv.page_table[0, 9])
    np.testing.assert_array_equal(after[pg9, :, 62], bits(kn)[0, 0])
    np.testing.assert_array_equal(after[pg9, :, 63], bits(kn)[0, 1])
    changed = np.argwhere((after != before).any(axis=(1, 2, 3)))[:, 0].tolist()
    assert changed == [pg9], f"pages written: {changed}"

"""Host-only checks of the C ABI: the library loads, exports every function
that include/wmtp.h declares, and rejects bad arguments before touching the
GPU (none of these calls reach a CUDA API)."""

import ctypes
import os
import re
from ctypes import byref, c_size_t

import pytest

import speculative_decode_draft_b200 as w
from speculative_decode_draft_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(wmtp_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from speculative_decode_draft_b200 import build
    build.build()
    return L.load()


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared, "no declarations found"
    assert declared <= set(L.EXPORTS) | declared
    for name in declared:
        assert hasattr(lib, name), f"libwmtp.so does not export {name}"
    assert set(L.EXPORTS) == declared


def test_version_and_status_strings(lib):
    assert lib.wmtp_version().decode().count(".") == 2
    assert lib.wmtp_status_string(0) == b"ok"
    for code in (-1, -2, -3, -4):
        assert lib.wmtp_status_string(code) != b"unknown status"


def _p(**kw):
    base = dict(num_heads_q=16, num_heads_kv=2, head_dim=256, page_size=64, sinks=4, window=2048,
                gamma_max=4, sm_scale=0.0)
    base.update(kw)
    return L.Params(**base)


def _full(lib, p, batch=1, num_q=None, kv=True):
    desc = L.PagedKVDesc(None, None, 8, None, 8, None) if kv else None
    size = c_size_t(0)
    if num_q is None:
        return lib.wmtp_draft_attn_full(byref(p) if p else None, batch, None, byref(desc) if desc else None,
                                        None, 1, None, None, byref(size), None, None)
    return lib.wmtp_verify_attn(byref(p) if p else None, batch, num_q, None, byref(desc) if desc else None,
                                None, 1, None, None, byref(size), None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=128), L.WMTP_ERR_UNSUPPORTED),
    (dict(head_dim=96), L.WMTP_ERR_UNSUPPORTED),
    (dict(num_heads_q=15), L.WMTP_ERR_INVALID_ARG),
    (dict(num_heads_kv=0), L.WMTP_ERR_INVALID_ARG),
    (dict(page_size=48), L.WMTP_ERR_UNSUPPORTED),
    (dict(page_size=8), L.WMTP_ERR_UNSUPPORTED),
    (dict(sm_scale=-1.0), L.WMTP_ERR_INVALID_ARG),
    (dict(sm_scale=float("nan")), L.WMTP_ERR_INVALID_ARG),
    (dict(num_heads_q=128, num_heads_kv=1), L.WMTP_ERR_UNSUPPORTED),  # a 128-row draft
    (dict(num_heads_q=140000, num_heads_kv=70000), L.WMTP_ERR_UNSUPPORTED),  # grid y limit
])
def test_paged_attention_rejects_bad_params(lib, kw, code):
    assert _full(lib, _p(**kw)) == code


def test_paged_attention_rejects_missing_pointers(lib):
    assert _full(lib, None) == L.WMTP_ERR_INVALID_ARG
    assert _full(lib, _p(), kv=False) == L.WMTP_ERR_INVALID_ARG
    assert _full(lib, _p(), batch=-1) == L.WMTP_ERR_INVALID_ARG
    assert _full(lib, _p(), num_q=0) == L.WMTP_ERR_INVALID_ARG
    assert _full(lib, _p(), num_q=17) == L.WMTP_ERR_UNSUPPORTED  # 17 * 8 = 136 rows
    assert _full(lib, _p(head_dim=64), num_q=9) == L.WMTP_ERR_UNSUPPORTED  # 72 rows need head_dim 256
    assert _full(lib, _p(), batch=65536) == L.WMTP_ERR_UNSUPPORTED  # grid z limit


def test_batch_zero_is_a_noop(lib):
    size = c_size_t(123)
    desc = L.PagedKVDesc(None, None, 8, None, 8, None)
    assert lib.wmtp_draft_attn_full(byref(_p()), 0, None, byref(desc), None, 1, None, None, byref(size),
                                    None, None) == 0
    assert size.value == 0


def test_ring_calls_reject_bad_params(lib):
    ring = L.RingDesc(None, None, None, None, None, None, None, None, 1)
    assert lib.wmtp_ring_reset(byref(_p(window=0)), byref(ring), None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_ring_reset(byref(_p(gamma_max=17)), byref(ring), None) == L.WMTP_ERR_UNSUPPORTED
    assert lib.wmtp_ring_reset(byref(_p()), byref(ring), None) == L.WMTP_ERR_INVALID_ARG  # null ptrs
    assert lib.wmtp_ring_append(byref(_p(sinks=-1)), byref(ring), None, None, None, None, 0, 0, None,
                                None) == L.WMTP_ERR_INVALID_ARG
    size = c_size_t(0)
    assert lib.wmtp_draft_attn_windowed(byref(_p()), None, byref(ring), None, 1, None, None, byref(size),
                                        None, None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_draft_attn_windowed(byref(_p()), None, None, None, 1, None, None, byref(size), None,
                                        None) == L.WMTP_ERR_INVALID_ARG


def test_combine_and_paged_write_reject_bad_args(lib):
    assert lib.wmtp_splitkv_combine(4, 256, 0, None, None, None, 1, None, None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_splitkv_combine(4, 6, 2, None, None, None, 1, None, None) == L.WMTP_ERR_UNSUPPORTED
    assert lib.wmtp_splitkv_combine(4, 8192, 2, None, None, None, 1, None, None) == L.WMTP_ERR_UNSUPPORTED
    assert lib.wmtp_splitkv_combine(4, 256, 2, None, None, None, 1, None, None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_splitkv_combine(0, 256, 2, None, None, None, 1, None, None) == 0
    desc = L.PagedKVDesc(None, None, 8, None, 8, None)
    assert lib.wmtp_paged_write(byref(_p()), 1, byref(desc), None, 1, None, None, None,
                                None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_paged_write(byref(_p(page_size=3)), 1, byref(desc), None, 1, None, None, None,
                                None) == L.WMTP_ERR_UNSUPPORTED
    assert lib.wmtp_paged_write(byref(_p()), 1, byref(desc), None, 0, None, None, None, None) == 0
    assert lib.wmtp_paged_write(byref(_p()), 65536, byref(desc), None, 1, None, None, None,
                                None) == L.WMTP_ERR_UNSUPPORTED  # grid y limit


def test_python_binding_raises_on_wrong_tensors():
    import torch
    p = w.params(16, 2, 256)
    with pytest.raises((TypeError, ValueError)):
        w.draft_attn_full(p, torch.zeros(1, 16, 256), None)


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(ImportError):
        L.load(str(tmp_path / "missing.so"))


def test_windowed_paged_and_slice_reject_bad_args(lib):
    desc = L.PagedKVDesc(None, None, 8, None, 8, None)
    size = c_size_t(0)
    # the windowed-over-pages draft needs window >= 1 and sinks >= 0
    for kw in (dict(window=0), dict(sinks=-1)):
        assert lib.wmtp_draft_attn_windowed_paged(byref(_p(**kw)), 1, None, byref(desc), None, 1, None, None,
                                                  byref(size), None, None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_draft_attn_windowed_paged(byref(_p(num_heads_q=15)), 1, None, byref(desc), None, 1, None,
                                              None, byref(size), None, None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_draft_attn_windowed_paged(byref(_p()), 0, None, byref(desc), None, 1, None, None,
                                              byref(size), None, None) == 0  # empty batch: size query only
    # a slice verify with a workspace needs the query positions
    ws = ctypes.create_string_buffer(512)
    have = c_size_t(256)
    assert lib.wmtp_verify_attn_slice(byref(_p()), 1, 4, None, byref(desc), None, None, 1, None,
                                      ctypes.addressof(ws) // 256 * 256 + 256, byref(have), None,
                                      None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_verify_attn_slice(byref(_p()), 1, 17, None, byref(desc), None, None, 1, None, None,
                                      byref(size), None, None) == L.WMTP_ERR_UNSUPPORTED  # 136 rows


def test_selftest_wait_rejects_misaligned_pointers(lib):
    # checked before anything is launched, so this runs without a GPU
    assert lib.wmtp_selftest_wait(0, None, 4, None) == L.WMTP_ERR_INVALID_ARG
    assert lib.wmtp_selftest_wait(0, 2, None, None) == L.WMTP_ERR_INVALID_ARG
    assert L.WAIT_LIMIT_CYCLES == 4_000_000_000


def test_verify_append_rejects_missing_new_tokens(lib):
    # checked before anything is launched, so this runs without a GPU
    desc = L.PagedKVDesc(None, None, 8, None, 8, None)
    ws = ctypes.create_string_buffer(512)
    have = c_size_t(256)
    base = ctypes.addressof(ws) // 256 * 256 + 256
    for k_new, v_new in ((None, base), (base, None), (None, None)):
        assert lib.wmtp_verify_attn_append(byref(_p()), 1, 4, None, k_new, v_new, byref(desc), None, 1, None,
                                           base, byref(have), None, None) == L.WMTP_ERR_INVALID_ARG
    # the size query needs no new tokens, and rejects what wmtp_verify_attn rejects
    size = c_size_t(0)
    assert lib.wmtp_verify_attn_append(byref(_p()), 1, 17, None, None, None, byref(desc), None, 1, None, None,
                                       byref(size), None, None) == L.WMTP_ERR_UNSUPPORTED  # 136 rows
    assert lib.wmtp_verify_attn_append(byref(_p()), 0, 4, None, None, None, byref(desc), None, 1, None, None,
                                       byref(size), None, None) == 0  # empty batch

"""The allocation-free native draft entry point, through the C ABI.

wmtp_draft_attn_full_noalloc serves callers that cannot give the library a
device workspace (runtimes that plan every device allocation before serving
starts; plugin hosts whose kernels receive only inputs and outputs).  It keeps
its split-KV scratch in a fixed array inside the library.  These tests check
the CUDA path against itself, not against the oracle (the workspace entry
point's own parity tests do that): two calls in a row give bit-identical
results to wmtp_draft_attn_full with a caller workspace (same split plan,
same kernels), a call changes the device's free memory by nothing, and a
request larger than the fixed array is refused.  This file is collected last
so that a failure here leaves every other test already run.
"""

from ctypes import byref, c_size_t, c_void_p

import pytest
import torch

import synth
import speculative_decode_draft_b200 as w
from speculative_decode_draft_b200 import _lib as L


pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def lib(cuda_device):
    from speculative_decode_draft_b200 import build
    build.build()
    return L.load()


def _desc(kv):
    return L.PagedKVDesc(kv.k_pool.data_ptr(), kv.v_pool.data_ptr(), kv.k_pool.shape[0],
                         kv.page_table.data_ptr(), kv.page_table.shape[1], kv.kv_len.data_ptr())


def _with_workspace(lib, p, q, kv, stream):
    B, Hq, D = q.shape
    desc = _desc(kv)
    size = c_size_t(0)
    assert lib.wmtp_draft_attn_full(byref(p), B, None, byref(desc), None, 1, None, None, byref(size),
                                    None, stream) == 0
    ws = torch.empty(max(size.value, 256), dtype=torch.uint8, device=DEV)
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    have = c_size_t(ws.numel())
    assert lib.wmtp_draft_attn_full(byref(p), B, q.data_ptr(), byref(desc), out.data_ptr(), 1, lse.data_ptr(),
                                    ws.data_ptr(), byref(have), None, stream) == 0
    return out, lse


def _noalloc(lib, p, q, kv, status, stream):
    B, Hq, D = q.shape
    desc = _desc(kv)
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    rc = lib.wmtp_draft_attn_full_noalloc(byref(p), B, q.data_ptr(), byref(desc), out.data_ptr(), 1,
                                          lse.data_ptr(), status.data_ptr(), stream)
    assert rc == 0, lib.wmtp_status_string(rc)
    return out, lse


@pytest.mark.parametrize("case", ["32k", "ragged"])
def test_noalloc_matches_workspace_entry_point_twice(lib, case):
    if case == "32k":
        wl = synth.workload("32k")
        lens, B, G, D, P, Hkv = [wl.context[0] + 1], 1, wl.group, wl.head_dim, wl.page_size, wl.num_heads_kv
    else:
        lens, B, G, D, P, Hkv = [100, 5000, 20000], 3, 8, 256, 64, 2
    p = w.params(G * Hkv, Hkv, D, page_size=P)
    kv = synth.paged_kv(7, B, Hkv, D, P, lens, max(lens) + 64, True, True, device=DEV)
    stream = c_void_p(torch.cuda.current_stream().cuda_stream)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for call, seed in enumerate((11, 12)):  # two calls in a row, different queries
        q = synth.queries(seed, (B, G * Hkv, D), device=DEV)
        ref_o, ref_l = _with_workspace(lib, p, q, kv, stream)
        o, l = _noalloc(lib, p, q, kv, status, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(o, ref_o), f"noalloc call {call}: output differs from the workspace entry point"
        assert torch.equal(l, ref_l), f"noalloc call {call}: lse differs from the workspace entry point"


def test_noalloc_call_allocates_no_device_memory(lib):
    B, G, D, P, Hkv = 2, 8, 256, 64, 2
    p = w.params(G * Hkv, Hkv, D, page_size=P)
    kv = synth.paged_kv(8, B, Hkv, D, P, [3000, 9000], 9064, True, True, device=DEV)
    stream = c_void_p(torch.cuda.current_stream().cuda_stream)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q = synth.queries(13, (B, G * Hkv, D), device=DEV)
    out = torch.empty(B, G * Hkv, D, dtype=torch.float32, device=DEV)
    lse = torch.empty(B, G * Hkv, dtype=torch.float32, device=DEV)
    desc = _desc(kv)

    def call():
        return lib.wmtp_draft_attn_full_noalloc(byref(p), B, q.data_ptr(), byref(desc), out.data_ptr(), 1,
                                                lse.data_ptr(), status.data_ptr(), stream)
    assert call() == 0  # warm-up: the library's code and the array are loaded by now
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    assert call() == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert int(status.item()) == 0


def test_noalloc_refuses_more_than_its_scratch(lib):
    # 8192 query rows with one split each need about 8.4 MB of partials
    p = w.params(64, 64, 256, page_size=64)
    desc = L.PagedKVDesc(256, 256, 64 * 128, 256, 1, 256)
    rc = lib.wmtp_draft_attn_full_noalloc(byref(p), 128, None, byref(desc), None, 1, None, None, None)
    assert rc == L.WMTP_ERR_WORKSPACE
    size = c_size_t(0)
    assert lib.wmtp_draft_attn_full(byref(p), 128, None, byref(desc), None, 1, None, None, byref(size), None,
                                    None) == 0
    assert size.value > L.NOALLOC_SCRATCH_BYTES

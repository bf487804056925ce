"""PyTorch-facing wrappers of the libwmtp C ABI (argument marshalling only).

Tensors are passed to the C ABI as raw device pointers; the wrappers check
dtype, device and contiguity, allocate outputs and the split-KV workspace with
PyTorch, and pass PyTorch's current CUDA stream.  Nothing here computes any
part of the attention path.
"""

from __future__ import annotations

import ctypes
from ctypes import byref, c_size_t, c_void_p
from dataclasses import dataclass

import torch

from . import _lib as L

BF16 = torch.bfloat16
I32 = torch.int32


def params(num_heads_q: int, num_heads_kv: int, head_dim: int, page_size: int = 64, sinks: int = 4,
           window: int = 2048, gamma_max: int = 8, sm_scale: float = 0.0) -> L.Params:
    """The wmtp_params struct (sm_scale 0 means 1/sqrt(head_dim))."""
    return L.Params(num_heads_q, num_heads_kv, head_dim, page_size, sinks, window, gamma_max, sm_scale)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, name: str, device=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream) -> c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


# ---------------------------------------------------------------- containers
@dataclass
class PagedCache:
    """One attention layer's paged KV cache (device tensors).

    k_pool, v_pool: bf16 ``[num_pages, Hkv, P, D]``; page_table int32
    ``[B, max_pages]``; kv_len int32 ``[B]``.
    """
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    page_table: torch.Tensor
    kv_len: torch.Tensor

    def desc(self) -> L.PagedKVDesc:
        for n in ("k_pool", "v_pool"):
            _need(getattr(self, n), BF16, n)
        for n in ("page_table", "kv_len"):
            _need(getattr(self, n), I32, n)
        return L.PagedKVDesc(self.k_pool.data_ptr(), self.v_pool.data_ptr(), self.k_pool.shape[0],
                             self.page_table.data_ptr(), self.page_table.shape[1], self.kv_len.data_ptr())


@dataclass
class Ring:
    """Per-sequence compact draft ring buffers (device tensors)."""
    k: torch.Tensor          # [B, Hkv, S+W, D] bf16
    v: torch.Tensor
    tags: torch.Tensor       # [B, S+W] int32
    len: torch.Tensor        # [B] int32
    committed: torch.Tensor  # [B] int32
    undo_k: torch.Tensor     # [B, gamma_max, Hkv, D] bf16
    undo_v: torch.Tensor
    undo_tags: torch.Tensor  # [B, gamma_max] int32

    @property
    def batch(self) -> int:
        return self.k.shape[0]

    @staticmethod
    def allocate(p: L.Params, batch: int, device, stream=None) -> "Ring":
        R = p.sinks + p.window
        g = max(p.gamma_max, 1)
        kw = dict(device=device)
        r = Ring(
            torch.empty(batch, p.num_heads_kv, R, p.head_dim, dtype=BF16, **kw),
            torch.empty(batch, p.num_heads_kv, R, p.head_dim, dtype=BF16, **kw),
            torch.empty(batch, R, dtype=I32, **kw),
            torch.empty(batch, dtype=I32, **kw),
            torch.empty(batch, dtype=I32, **kw),
            torch.empty(batch, g, p.num_heads_kv, p.head_dim, dtype=BF16, **kw),
            torch.empty(batch, g, p.num_heads_kv, p.head_dim, dtype=BF16, **kw),
            torch.empty(batch, g, dtype=I32, **kw),
        )
        ring_reset(p, r, stream=stream)
        return r

    def desc(self) -> L.RingDesc:
        for n in ("k", "v", "undo_k", "undo_v"):
            _need(getattr(self, n), BF16, n)
        for n in ("tags", "len", "committed", "undo_tags"):
            _need(getattr(self, n), I32, n)
        return L.RingDesc(self.k.data_ptr(), self.v.data_ptr(), self.tags.data_ptr(), self.len.data_ptr(),
                          self.committed.data_ptr(), self.undo_k.data_ptr(), self.undo_v.data_ptr(),
                          self.undo_tags.data_ptr(), self.batch)


# ---------------------------------------------------------------- workspace
_ws_cache: dict = {}


def _workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    key = (device.type, device.index)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def _run_attention(fn_name: str, call, out_shape, device, out_fp32, out, lse, workspace, status):
    lib = L.load()
    fn = getattr(lib, fn_name)
    size = c_size_t(0)
    L.check(fn_name, call(fn, None, None, None, None, byref(size), None))
    ws = workspace if workspace is not None else _workspace(device, size.value)
    if ws.numel() < size.value:
        raise ValueError(f"workspace needs {size.value} bytes, got {ws.numel()}")
    if out is None:
        out = torch.empty(out_shape, dtype=torch.float32 if out_fp32 else BF16, device=device)
    if lse is None:
        lse = torch.empty(out_shape[:-1], dtype=torch.float32, device=device)
    have = c_size_t(ws.numel())
    L.check(fn_name, call(fn, out.data_ptr(), lse.data_ptr(), ws.data_ptr(), None, byref(have),
                          _ptr(status)))
    return out, lse


def workspace_bytes(kind: str, p: L.Params, batch: int, num_q: int = 1, max_pages: int = 1,
                    num_pages: int = 1) -> int:
    """Bytes of split-KV workspace a call needs on the current device."""
    lib = L.load()
    size = c_size_t(0)
    if kind == "windowed":
        desc = L.RingDesc(256, 256, 256, 256, 256, 256, 256, 256, batch)  # sizes only: never dereferenced
        L.check(kind, lib.wmtp_draft_attn_windowed(byref(p), None, byref(desc), None, 1, None, None,
                                                   byref(size), None, None))
    else:
        desc = L.PagedKVDesc(None, None, num_pages, None, max_pages, None)
        if kind == "full":
            L.check(kind, lib.wmtp_draft_attn_full(byref(p), batch, None, byref(desc), None, 1, None, None,
                                                   byref(size), None, None))
        elif kind == "windowed_paged":
            L.check(kind, lib.wmtp_draft_attn_windowed_paged(byref(p), batch, None, byref(desc), None, 1, None,
                                                             None, byref(size), None, None))
        else:
            L.check(kind, lib.wmtp_verify_attn(byref(p), batch, num_q, None, byref(desc), None, 1, None, None,
                                               byref(size), None, None))
    return size.value


# ---------------------------------------------------------------- entry points
def draft_attn_full(p: L.Params, q: torch.Tensor, cache: PagedCache, *, out_fp32: bool = True,
                    out=None, lse=None, workspace=None, status=None, stream=None):
    """Native MTP draft attention: q ``[B, Hq, D]`` bf16 -> (out, lse)."""
    _need(q, BF16, "q")
    B, Hq, D = q.shape
    desc = cache.desc()
    st = _stream(stream)

    def call(fn, o, l, ws, _unused, size, stat):
        return fn(byref(p), B, None if ws is None else q.data_ptr(), byref(desc), o, int(out_fp32), l, ws,
                  size, stat, st)
    return _run_attention("wmtp_draft_attn_full", call, (B, Hq, D), q.device, out_fp32, out, lse,
                          workspace, status)


def draft_attn_windowed_paged(p: L.Params, q: torch.Tensor, cache: PagedCache, *, out_fp32: bool = True,
                              out=None, lse=None, workspace=None, status=None, stream=None):
    """Windowed-MTP draft attention read through the page table (sink +
    window positions of the paged cache, no ring): q ``[B, Hq, D]`` bf16."""
    _need(q, BF16, "q")
    B, Hq, D = q.shape
    desc = cache.desc()
    st = _stream(stream)

    def call(fn, o, l, ws, _unused, size, stat):
        return fn(byref(p), B, None if ws is None else q.data_ptr(), byref(desc), o, int(out_fp32), l, ws,
                  size, stat, st)
    return _run_attention("wmtp_draft_attn_windowed_paged", call, (B, Hq, D), q.device, out_fp32, out, lse,
                          workspace, status)


def verify_attn(p: L.Params, q: torch.Tensor, cache: PagedCache, *, out_fp32: bool = True, out=None,
                lse=None, workspace=None, status=None, stream=None, q_pos0: torch.Tensor | None = None):
    """Verify attention: q ``[B, num_q, Hq, D]`` bf16 -> (out, lse).

    ``q_pos0`` (int32 ``[B]``): the cache holds a slice of each sequence and
    query 0 sits at this position counted from the slice's first token
    (``wmtp_verify_attn_slice``); None means the cache holds the whole context
    and the queries are its last ``num_q`` positions."""
    _need(q, BF16, "q")
    B, Qn, Hq, D = q.shape
    desc = cache.desc()
    st = _stream(stream)
    if q_pos0 is not None:
        _need(q_pos0, I32, "q_pos0", q.device)

        def call_slice(fn, o, l, ws, _unused, size, stat):
            return fn(byref(p), B, Qn, None if ws is None else q.data_ptr(), byref(desc),
                      None if ws is None else q_pos0.data_ptr(), o, int(out_fp32), l, ws, size, stat, st)
        return _run_attention("wmtp_verify_attn_slice", call_slice, (B, Qn, Hq, D), q.device, out_fp32, out,
                              lse, workspace, status)

    def call(fn, o, l, ws, _unused, size, stat):
        return fn(byref(p), B, Qn, None if ws is None else q.data_ptr(), byref(desc), o, int(out_fp32), l,
                  ws, size, stat, st)
    return _run_attention("wmtp_verify_attn", call, (B, Qn, Hq, D), q.device, out_fp32, out, lse,
                          workspace, status)


def verify_attn_append(p: L.Params, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                       cache: PagedCache, *, out_fp32: bool = True, out=None, lse=None, workspace=None,
                       status=None, stream=None):
    """``paged_write`` of ``k_new/v_new [B, num_q, Hkv, D]`` at the last num_q
    positions of each sequence (``cache.kv_len`` includes them), then
    ``verify_attn``, in one call (``wmtp_verify_attn_append``)."""
    _need(q, BF16, "q")
    _need(k_new, BF16, "k_new", q.device)
    _need(v_new, BF16, "v_new", q.device)
    B, Qn, Hq, D = q.shape
    if tuple(k_new.shape[:2]) != (B, Qn) or k_new.shape != v_new.shape:
        raise ValueError(f"k_new/v_new must be [B, num_q, Hkv, D] = [{B}, {Qn}, ...], got {tuple(k_new.shape)}")
    desc = cache.desc()
    st = _stream(stream)

    def call(fn, o, l, ws, _unused, size, stat):
        live = ws is not None
        return fn(byref(p), B, Qn, q.data_ptr() if live else None, k_new.data_ptr() if live else None,
                  v_new.data_ptr() if live else None, byref(desc), o, int(out_fp32), l, ws, size, stat, st)
    return _run_attention("wmtp_verify_attn_append", call, (B, Qn, Hq, D), q.device, out_fp32, out, lse,
                          workspace, status)


def draft_attn_windowed(p: L.Params, q: torch.Tensor, ring: Ring, *, out_fp32: bool = True, out=None,
                        lse=None, workspace=None, status=None, stream=None):
    """Windowed-MTP draft attention over the rings: q ``[B, Hq, D]`` bf16."""
    _need(q, BF16, "q")
    B, Hq, D = q.shape
    if B != ring.batch:
        raise ValueError("q batch differs from ring batch")
    desc = ring.desc()
    st = _stream(stream)

    def call(fn, o, l, ws, _unused, size, stat):
        return fn(byref(p), None if ws is None else q.data_ptr(), byref(desc), o, int(out_fp32), l, ws, size,
                  stat, st)
    return _run_attention("wmtp_draft_attn_windowed", call, (B, Hq, D), q.device, out_fp32, out, lse,
                          workspace, status)


def ring_append(p: L.Params, ring: Ring, k_new: torch.Tensor | None, v_new: torch.Tensor | None,
                n_new: torch.Tensor | None, *, truncate_to: torch.Tensor | None = None,
                speculative: bool = False, status=None, stream=None) -> None:
    """Append ``k_new/v_new [B, max_new, Hkv, D]`` (rows ``< n_new[b]``) to the rings."""
    desc = ring.desc()
    max_new = 0
    if k_new is not None:
        _need(k_new, BF16, "k_new")
        _need(v_new, BF16, "v_new")
        _need(n_new, I32, "n_new")
        max_new = k_new.shape[1]
    if truncate_to is not None:
        _need(truncate_to, I32, "truncate_to")
    L.check("wmtp_ring_append", L.load().wmtp_ring_append(
        byref(p), byref(desc), _ptr(truncate_to), _ptr(n_new), _ptr(k_new), _ptr(v_new), max_new,
        int(speculative), _ptr(status), _stream(stream)))


def ring_reset(p: L.Params, ring: Ring, stream=None) -> None:
    desc = ring.desc()
    L.check("wmtp_ring_reset", L.load().wmtp_ring_reset(byref(p), byref(desc), _stream(stream)))


def splitkv_combine(part_o: torch.Tensor, part_lse: torch.Tensor, *, out_fp32: bool = True, out=None,
                    lse=None, stream=None):
    """Merge partials ``part_o [rows, nsplit, D]`` / ``part_lse [rows, nsplit]``."""
    _need(part_o, torch.float32, "part_o")
    _need(part_lse, torch.float32, "part_lse")
    rows, nsplit, D = part_o.shape
    if out is None:
        out = torch.empty(rows, D, dtype=torch.float32 if out_fp32 else BF16, device=part_o.device)
    if lse is None:
        lse = torch.empty(rows, dtype=torch.float32, device=part_o.device)
    L.check("wmtp_splitkv_combine", L.load().wmtp_splitkv_combine(
        rows, D, nsplit, part_o.data_ptr(), part_lse.data_ptr(), out.data_ptr(), int(out_fp32),
        lse.data_ptr(), _stream(stream)))
    return out, lse


def paged_write(p: L.Params, cache: PagedCache, pos0: torch.Tensor, k_new: torch.Tensor,
                v_new: torch.Tensor, *, status=None, stream=None) -> None:
    """Write ``k_new/v_new [B, n_new, Hkv, D]`` at positions ``pos0[b] + j``."""
    _need(pos0, I32, "pos0")
    _need(k_new, BF16, "k_new")
    _need(v_new, BF16, "v_new")
    desc = cache.desc()
    B, n_new = k_new.shape[:2]
    L.check("wmtp_paged_write", L.load().wmtp_paged_write(
        byref(p), B, byref(desc), pos0.data_ptr(), n_new, k_new.data_ptr(), v_new.data_ptr(), _ptr(status),
        _stream(stream)))


def new_status(device) -> torch.Tensor:
    """A zeroed device status word for the ``status=`` arguments."""
    return torch.zeros(1, dtype=I32, device=device)


def selftest_wait(arrive: bool, *, status=None, cycles=None, stream=None) -> None:
    """One bounded in-kernel wait (``wmtp_selftest_wait``).  Without ``arrive``
    nothing completes the barrier: the wait gives up after
    ``WAIT_LIMIT_CYCLES`` SM clocks and sets ``DEV_TIMEOUT`` in ``status``.
    ``cycles`` (int64 ``[1]``) receives the clocks the wait took."""
    if status is not None:
        _need(status, I32, "status")
    if cycles is not None:
        _need(cycles, torch.int64, "cycles")
    L.check("wmtp_selftest_wait", L.load().wmtp_selftest_wait(
        int(bool(arrive)), _ptr(status), _ptr(cycles), _stream(stream)))


# ---------------------------------------------------------------- serving-side helpers (host only)
class PagePool:
    """Free-list allocator over the page indices of one pool tensor
    (``wmtp_pool_*``; host memory only)."""

    def __init__(self, num_pages: int):
        self._lib = L.load()
        h = c_void_p()
        L.check("wmtp_pool_create", self._lib.wmtp_pool_create(int(num_pages), byref(h)))
        self._h = h

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.wmtp_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def free_count(self) -> int:
        return int(self._lib.wmtp_pool_free_count(self._h))

    def alloc(self, n: int) -> list[int]:
        """``n`` page indices; raises WmtpError (WMTP_ERR_WORKSPACE) if fewer are free."""
        buf = (ctypes.c_int32 * max(int(n), 1))()
        L.check("wmtp_pool_alloc", self._lib.wmtp_pool_alloc(self._h, int(n), buf))
        return list(buf[:int(n)])

    def release(self, pages) -> None:
        pages = list(pages)
        buf = (ctypes.c_int32 * max(len(pages), 1))(*pages)
        L.check("wmtp_pool_release", self._lib.wmtp_pool_release(self._h, len(pages), buf))


def plan_admission(p: L.Params, context: int, target_layers: int, draft_layers: int, windowed: bool,
                   kv_budget_bytes: int) -> dict:
    """Per-request KV footprint and the requests a budget admits (``wmtp_plan_admission``)."""
    out = L.Admission()
    L.check("wmtp_plan_admission", L.load().wmtp_plan_admission(
        byref(p), int(context), int(target_layers), int(draft_layers), int(bool(windowed)),
        int(kv_budget_bytes), byref(out)))
    return {name: int(getattr(out, name)) for name, _ in L.Admission._fields_}

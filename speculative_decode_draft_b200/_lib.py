"""ctypes binding of libwmtp (include/wmtp.h): argument marshalling only.

Every computation happens in the CUDA kernels behind the C ABI.  PyTorch is
used for device memory and streams.  If the shared library is missing, every
call raises: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_size_t, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwmtp.so")

# status codes and device status bits (include/wmtp.h)
WMTP_OK = 0
WMTP_ERR_INVALID_ARG = -1
WMTP_ERR_UNSUPPORTED = -2
WMTP_ERR_WORKSPACE = -3
WMTP_ERR_CUDA = -4
DEV_PAGE_OOB = 0x1
DEV_LEN_OOB = 0x2
DEV_RING_STATE = 0x4
DEV_UNDO_FULL = 0x8
DEV_TIMEOUT = 0x10
DEV_V_RANGE = 0x20  # reserved, never set
WAIT_LIMIT_CYCLES = 4000000000  # WMTP_WAIT_LIMIT_CYCLES

EXPORTS = (
    "wmtp_status_string",
    "wmtp_version",
    "wmtp_draft_attn_full",
    "wmtp_draft_attn_windowed",
    "wmtp_draft_attn_windowed_paged",
    "wmtp_ring_append",
    "wmtp_ring_reset",
    "wmtp_verify_attn",
    "wmtp_verify_attn_append",
    "wmtp_verify_attn_slice",
    "wmtp_splitkv_combine",
    "wmtp_paged_write",
    "wmtp_draft_attn_full_noalloc",
    "wmtp_pool_create",
    "wmtp_pool_destroy",
    "wmtp_pool_free_count",
    "wmtp_pool_alloc",
    "wmtp_pool_release",
    "wmtp_plan_admission",
    "wmtp_selftest_wait",
)

# Size of the fixed scratch array behind wmtp_draft_attn_full_noalloc.
NOALLOC_SCRATCH_BYTES = 4 << 20


class Params(ctypes.Structure):
    _fields_ = [
        ("num_heads_q", c_int32),
        ("num_heads_kv", c_int32),
        ("head_dim", c_int32),
        ("page_size", c_int32),
        ("sinks", c_int32),
        ("window", c_int32),
        ("gamma_max", c_int32),
        ("sm_scale", c_float),
    ]


class PagedKVDesc(ctypes.Structure):
    _fields_ = [
        ("k_pool", c_void_p),
        ("v_pool", c_void_p),
        ("num_pages", c_int32),
        ("page_table", c_void_p),
        ("max_pages", c_int32),
        ("kv_len", c_void_p),
    ]


class RingDesc(ctypes.Structure):
    _fields_ = [
        ("k", c_void_p),
        ("v", c_void_p),
        ("tags", c_void_p),
        ("len", c_void_p),
        ("committed", c_void_p),
        ("undo_k", c_void_p),
        ("undo_v", c_void_p),
        ("undo_tags", c_void_p),
        ("batch", c_int32),
    ]


class Admission(ctypes.Structure):
    _fields_ = [
        ("pages_per_layer", ctypes.c_int64),
        ("page_bytes", ctypes.c_int64),
        ("target_bytes", ctypes.c_int64),
        ("draft_bytes", ctypes.c_int64),
        ("bytes_per_request", ctypes.c_int64),
        ("max_requests", ctypes.c_int64),
    ]


class WmtpError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn} failed: {code} ({text})")
        self.code = code


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libwmtp.so (once) and declare the signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(
            f"libwmtp.so not found at {p}; build it with "
            "`python -m speculative_decode_draft_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(p)
    PP = POINTER(Params)
    PK = POINTER(PagedKVDesc)
    PR = POINTER(RingDesc)
    sz = POINTER(c_size_t)
    i32p = c_void_p
    lib.wmtp_status_string.restype = ctypes.c_char_p
    lib.wmtp_status_string.argtypes = [c_int32]
    lib.wmtp_version.restype = ctypes.c_char_p
    lib.wmtp_version.argtypes = []
    lib.wmtp_draft_attn_full.restype = c_int32
    lib.wmtp_draft_attn_full.argtypes = [PP, c_int32, c_void_p, PK, c_void_p, c_int32, c_void_p,
                                         c_void_p, sz, i32p, c_void_p]
    lib.wmtp_draft_attn_windowed_paged.restype = c_int32
    lib.wmtp_draft_attn_windowed_paged.argtypes = [PP, c_int32, c_void_p, PK, c_void_p, c_int32, c_void_p,
                                                   c_void_p, sz, i32p, c_void_p]
    lib.wmtp_verify_attn.restype = c_int32
    lib.wmtp_verify_attn.argtypes = [PP, c_int32, c_int32, c_void_p, PK, c_void_p, c_int32, c_void_p,
                                     c_void_p, sz, i32p, c_void_p]
    lib.wmtp_verify_attn_append.restype = c_int32
    lib.wmtp_verify_attn_append.argtypes = [PP, c_int32, c_int32, c_void_p, c_void_p, c_void_p, PK, c_void_p,
                                            c_int32, c_void_p, c_void_p, sz, i32p, c_void_p]
    lib.wmtp_verify_attn_slice.restype = c_int32
    lib.wmtp_verify_attn_slice.argtypes = [PP, c_int32, c_int32, c_void_p, PK, c_void_p, c_void_p, c_int32,
                                           c_void_p, c_void_p, sz, i32p, c_void_p]
    lib.wmtp_draft_attn_windowed.restype = c_int32
    lib.wmtp_draft_attn_windowed.argtypes = [PP, c_void_p, PR, c_void_p, c_int32, c_void_p, c_void_p, sz,
                                             i32p, c_void_p]
    lib.wmtp_ring_append.restype = c_int32
    lib.wmtp_ring_append.argtypes = [PP, PR, c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                     i32p, c_void_p]
    lib.wmtp_ring_reset.restype = c_int32
    lib.wmtp_ring_reset.argtypes = [PP, PR, c_void_p]
    lib.wmtp_splitkv_combine.restype = c_int32
    lib.wmtp_splitkv_combine.argtypes = [c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32,
                                         c_void_p, c_void_p]
    lib.wmtp_paged_write.restype = c_int32
    lib.wmtp_paged_write.argtypes = [PP, c_int32, PK, c_void_p, c_int32, c_void_p, c_void_p, i32p,
                                     c_void_p]
    lib.wmtp_draft_attn_full_noalloc.restype = c_int32
    lib.wmtp_draft_attn_full_noalloc.argtypes = [PP, c_int32, c_void_p, PK, c_void_p, c_int32, c_void_p,
                                                 i32p, c_void_p]
    lib.wmtp_pool_create.restype = c_int32
    lib.wmtp_pool_create.argtypes = [c_int32, POINTER(c_void_p)]
    lib.wmtp_pool_destroy.restype = None
    lib.wmtp_pool_destroy.argtypes = [c_void_p]
    lib.wmtp_pool_free_count.restype = c_int32
    lib.wmtp_pool_free_count.argtypes = [c_void_p]
    lib.wmtp_pool_alloc.restype = c_int32
    lib.wmtp_pool_alloc.argtypes = [c_void_p, c_int32, c_void_p]
    lib.wmtp_pool_release.restype = c_int32
    lib.wmtp_pool_release.argtypes = [c_void_p, c_int32, c_void_p]
    lib.wmtp_plan_admission.restype = c_int32
    lib.wmtp_plan_admission.argtypes = [PP, ctypes.c_int64, c_int32, c_int32, c_int32, ctypes.c_int64,
                                        POINTER(Admission)]
    lib.wmtp_selftest_wait.restype = c_int32
    lib.wmtp_selftest_wait.argtypes = [c_int32, c_void_p, c_void_p, c_void_p]
    if path is None:
        _lib = lib
    return lib


def check(fn: str, code: int) -> None:
    if code != WMTP_OK:
        raise WmtpError(fn, code, load().wmtp_status_string(code).decode())

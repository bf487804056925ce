"""Windowed-MTP draft/verify decode attention for NVIDIA B200 (sm_100a).

The hot path -- native and windowed MTP draft attention, the compact draft
ring buffer, causal verify attention and the split-KV combine -- runs in the
CUDA kernels of ``libwmtp.so`` behind the C ABI in ``include/wmtp.h``.  This
package is the thin PyTorch binding of that library.
"""

from ._lib import EXPORTS, WmtpError, load  # noqa: F401
from .api import (  # noqa: F401
    PagedCache,
    PagePool,
    Ring,
    draft_attn_full,
    draft_attn_windowed_paged,
    draft_attn_windowed,
    new_status,
    paged_write,
    params,
    plan_admission,
    ring_append,
    ring_reset,
    selftest_wait,
    splitkv_combine,
    verify_attn,
    verify_attn_append,
    workspace_bytes,
)

__version__ = "0.1.0"

"""Context-parallel verify: one sequence's context spread over several GPUs.

Each rank of a process group holds a contiguous range of every sequence's
positions in its own paged cache.  The verify queries (the last ``num_q``
positions of the sequence) attend each slice with the slice's causal limits
(``wmtp_verify_attn_slice``), the ranks exchange their (out, lse) pairs with
one all-gather of ``rows x (D + 1)`` fp32 values, and every rank merges them
with ``wmtp_splitkv_combine``.  The merge is exact: softmax attention over a
union of disjoint key sets is the log-sum-exp merge of the attentions over
each set.  The pages measure one GPU; this is the layout for contexts larger
than one GPU's memory.

Argument marshalling and the collective only: the attention and the merge run
in libwmtp's kernels.
"""

from __future__ import annotations

import torch

from . import _lib as L
from .api import PagedCache, splitkv_combine, verify_attn


def slice_query_positions(n_total: torch.Tensor, num_q: int, slice_start: torch.Tensor) -> torch.Tensor:
    """q_pos0 of every sequence for a slice that starts at global position
    ``slice_start``: the queries sit at ``n_total - num_q .. n_total - 1``."""
    return (n_total.to(torch.int64) - num_q - slice_start.to(torch.int64)).to(torch.int32).contiguous()


def gather_partials(o_local: torch.Tensor, lse_local: torch.Tensor, group=None):
    """All-gather every rank's (out, lse) in one collective and lay them out as
    combine partials: part_o ``[rows, world, D]``, part_lse ``[rows, world]``.

    Each rank contributes one ``rows x (D + 1)`` buffer (its output rows with
    the log-sum-exp appended, in the outputs' dtype: fp32 from the library).
    A gloo group gathers through host memory."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rows, D = o_local.shape
    packed = torch.cat([o_local, lse_local.to(o_local.dtype).reshape(rows, 1)], dim=1).contiguous()
    staged = packed.cpu() if (packed.is_cuda and dist.get_backend(group) == "gloo") else packed
    gathered = torch.empty((world,) + tuple(staged.shape), dtype=staged.dtype, device=staged.device)
    if staged.is_cuda:
        dist.all_gather_into_tensor(gathered, staged, group=group)
    else:
        dist.all_gather(list(gathered.unbind(0)), staged, group=group)
    g = gathered.to(o_local.device).permute(1, 0, 2)  # [rows, world, D + 1]
    return g[:, :, :D].contiguous(), g[:, :, D].contiguous()


def verify_attn_context_parallel(p: L.Params, q: torch.Tensor, local_cache: PagedCache,
                                 slice_start: torch.Tensor, n_total: torch.Tensor, *, group=None,
                                 out_fp32: bool = True, workspace=None, status=None):
    """Verify attention of ``q [B, num_q, Hq, D]`` over a context split across
    the ranks of ``group``.

    ``local_cache`` holds this rank's positions ``slice_start[b] ..
    slice_start[b] + kv_len[b] - 1`` of sequence b (its kv_len is the slice
    length); ``n_total[b]`` is the sequence's full length including the
    ``num_q`` new tokens.  Returns the merged (out, lse) on every rank.
    """
    import torch.distributed as dist
    B, Qn, Hq, D = q.shape
    q_pos0 = slice_query_positions(n_total, Qn, slice_start)
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return verify_attn(p, q, local_cache, q_pos0=q_pos0, out_fp32=out_fp32, workspace=workspace,
                           status=status)
    o, lse = verify_attn(p, q, local_cache, q_pos0=q_pos0, workspace=workspace, status=status)  # fp32 partial
    rows = B * Qn * Hq
    part_o, part_lse = gather_partials(o.view(rows, D), lse.view(rows), group)
    out, lse_all = splitkv_combine(part_o, part_lse, out_fp32=out_fp32)
    return out.view(B, Qn, Hq, D), lse_all.view(B, Qn, Hq)

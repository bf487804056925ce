"""Seeded synthetic inputs for the Windowed-MTP draft/verify attention path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the CUDA path's tests and the CPU oracle can take
their inputs from it.

Distributions (the pages fix none of them; the readings are stated here so a
reader can check them):

* Q ~ N(0, 1) rounded to bf16.
* K, V ~ N(0, 1) times a per-KV-head scale drawn uniformly from [0.5, 2]
  (separately for K and V, applied before the bf16 cast), except the ``tiny``
  workload, which is plain N(0, 1).
* Page tables: a random permutation of the pool's pages (identity for
  ``tiny``), drawn with ``numpy.random.default_rng(seed)``.
* Accepted-token counts per decode step: uniform on ``1 .. gamma+1`` from the
  same numpy generator.

Sizes follow the workloads named in the module-level ``WORKLOADS`` table.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_heads_q: int
    num_heads_kv: int
    head_dim: int
    page_size: int
    sinks: int
    window: int
    gamma: int
    verify_layers: int
    context: tuple          # committed KV length per sequence at step start
    kv_scale: bool          # per-head U[0.5, 2] scale on K and V
    shuffle_pages: bool
    seed: int
    steps: int = 1          # decode steps (ragged workload: 512)
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.num_heads_q // self.num_heads_kv

    @property
    def ring_slots(self) -> int:
        return self.sinks + self.window

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # batch 1, 1 draft + 1 target layer, 4 q heads / 1 kv head, D=64, 2,048
    # tokens, page 16, S=4, W=256, gamma=3, 4-query verify.
    "tiny": Workload("tiny", 1, 4, 1, 64, 16, 4, 256, 3, 1, (2048,), False, False, 1),
    # batch 1, GQA 16/2, D=256, 32,768 tokens, page 64 shuffled, S=4, W=2,048.
    "32k": Workload("32k", 1, 16, 2, 256, 64, 4, 2048, 3, 1, (32768,), True, True, 2),
    # 131,072 tokens, draft layer plus 10 verify layers.
    "128k": Workload("128k", 1, 16, 2, 256, 64, 4, 2048, 3, 10, (131072,), True, True, 3),
    # 1,048,576 tokens (~2 GiB bf16 KV per layer), draft plus 10 verify layers.
    "1m": Workload("1m", 1, 16, 2, 256, 64, 4, 2048, 3, 10, (1048576,), True, True, 4,
                   extra={"gammas": (3, 5), "windows": (1024, 4096)}),
    # 4 ragged sequences of 262,144 .. 1,048,576 tokens, 512 decode steps.
    "ragged4": Workload("ragged4", 4, 16, 2, 256, 64, 4, 2048, 3, 10, (), True, True, 5,
                        steps=512),
}


def ragged_lengths(seed: int, batch: int, lo: int = 262144, hi: int = 1048576) -> tuple:
    rng = np.random.default_rng(seed)
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=batch))


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    if name == "ragged4" and not w.context:
        w = w.with_(context=ragged_lengths(w.seed, w.batch))
    return w.with_(**overrides) if overrides else w


# ---------------------------------------------------------------------------
# random draws
# ---------------------------------------------------------------------------

def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, gen: torch.Generator, device, scale=None) -> torch.Tensor:
    """N(0,1) draws (fp32) times an optional broadcastable scale, then bf16."""
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if scale is not None:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def head_scales(gen: torch.Generator, num_heads: int, device) -> torch.Tensor:
    return 0.5 + 1.5 * torch.rand((num_heads,), generator=gen, device=device, dtype=torch.float32)


@dataclass
class PagedKV:
    """A paged K/V pool for one attention layer.

    k_pool, v_pool: bf16 ``[num_pages, Hkv, P, D]``; page_table int32
    ``[B, max_pages]``; kv_len int32 ``[B]``.
    """
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    page_table: torch.Tensor
    kv_len: torch.Tensor
    page_size: int

    @property
    def num_pages(self) -> int:
        return self.k_pool.shape[0]

    @property
    def max_pages(self) -> int:
        return self.page_table.shape[1]


def page_table(seed: int, batch: int, max_pages: int, shuffle: bool) -> np.ndarray:
    """int32 ``[batch, max_pages]``: a permutation of ``batch*max_pages`` pages."""
    total = batch * max_pages
    if shuffle:
        perm = np.random.default_rng(seed).permutation(total)
    else:
        perm = np.arange(total)
    return perm.reshape(batch, max_pages).astype(np.int32)


def paged_kv(seed: int, batch: int, num_heads_kv: int, head_dim: int, page_size: int,
             kv_len, capacity_tokens: int, kv_scale: bool, shuffle: bool,
             device="cpu") -> PagedKV:
    """Random pool with room for ``capacity_tokens`` per sequence.

    Every page of the pool is filled (used or not), so nothing uninitialised
    is ever read.
    """
    max_pages = -(-int(capacity_tokens) // page_size)
    num_pages = batch * max_pages
    gen = _gen(seed, device)
    ks = head_scales(gen, num_heads_kv, device).view(1, -1, 1, 1) if kv_scale else None
    vs = head_scales(gen, num_heads_kv, device).view(1, -1, 1, 1) if kv_scale else None
    shape = (num_pages, num_heads_kv, page_size, head_dim)
    k_pool = normal_bf16(shape, gen, device, ks)
    v_pool = normal_bf16(shape, gen, device, vs)
    pt = torch.from_numpy(page_table(seed, batch, max_pages, shuffle)).to(device)
    lens = torch.as_tensor(np.asarray(kv_len, dtype=np.int32).reshape(batch), device=device)
    return PagedKV(k_pool, v_pool, pt, lens, page_size)


def queries(seed: int, shape, device="cpu") -> torch.Tensor:
    """bf16 N(0,1) queries of any shape (``[B,Hq,D]`` or ``[B,Qn,Hq,D]``)."""
    return normal_bf16(tuple(shape), _gen(seed, device), device)


def new_tokens(seed: int, batch: int, n_new: int, num_heads_kv: int, head_dim: int,
               device="cpu", kv_scale: bool = False):
    """K/V of ``n_new`` new tokens per sequence: bf16 ``[B, n_new, Hkv, D]``."""
    gen = _gen(seed, device)
    ks = head_scales(gen, num_heads_kv, device).view(1, 1, -1, 1) if kv_scale else None
    vs = head_scales(gen, num_heads_kv, device).view(1, 1, -1, 1) if kv_scale else None
    shape = (batch, n_new, num_heads_kv, head_dim)
    return normal_bf16(shape, gen, device, ks), normal_bf16(shape, gen, device, vs)


def accept_counts(seed: int, steps: int, batch: int, gamma: int) -> np.ndarray:
    """Accepted tokens per decode step, uniform on ``1 .. gamma+1``: ``[steps, B]``."""
    return np.random.default_rng(seed + 7919).integers(1, gamma + 2, size=(steps, batch)).astype(np.int32)


def dense_from_paged(kv: PagedKV, b: int, length: int):
    """Gather positions ``0..length-1`` of sequence ``b`` into ``[length, Hkv, D]``
    (a layout helper for building rings from the same history)."""
    P = kv.page_size
    npg = -(-length // P)
    pages = kv.page_table[b, :npg].long()
    k = kv.k_pool[pages].permute(0, 2, 1, 3).reshape(npg * P, kv.k_pool.shape[1], -1)[:length]
    v = kv.v_pool[pages].permute(0, 2, 1, 3).reshape(npg * P, kv.v_pool.shape[1], -1)[:length]
    return k, v


def sm_scale_default(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)

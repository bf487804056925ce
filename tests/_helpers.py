"""Test helpers: conversions between device tensors and the oracle's numpy
inputs, and the parity metrics.  Nothing here computes attention."""

import numpy as np
import torch

import speculative_decode_draft_b200 as w

# Parity bar for floating-point outputs (fp32 output mode vs the fp64 oracle).
MAX_ABS = 2e-3
REL_L2 = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 tensor as uint16."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def rel_l2(x: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def assert_close(out: np.ndarray, ref: np.ndarray, what: str = "", max_abs=MAX_ABS, rel=REL_L2):
    err = float(np.abs(out - ref).max()) if out.size else 0.0
    r = rel_l2(out, ref)
    assert err <= max_abs and r <= rel, f"{what}: max-abs {err:.3e} (<= {max_abs}), rel-L2 {r:.3e} (<= {rel})"
    return err, r


def assert_lse_close(lse: np.ndarray, ref: np.ndarray, what: str = "", tol=1e-4):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(lse), fin), f"{what}: -inf pattern differs"
    if fin.any():
        err = float(np.abs(lse[fin] - ref[fin]).max())
        assert err <= tol, f"{what}: lse max-abs {err:.3e} > {tol}"


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (round to nearest even), back as fp64."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def bf16_ulp_diff(a_bf16: torch.Tensor, ref_f64: np.ndarray) -> int:
    """Largest distance in bf16 ulps between a bf16 tensor and rounded ref."""
    ra = bits(a_bf16).astype(np.int32)
    rb = bits(torch.from_numpy(np.ascontiguousarray(ref_f64)).to(torch.bfloat16)).astype(np.int32)

    def ordered(x):  # map sign-magnitude bf16 bits to a monotone integer line
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    return int(np.abs(ordered(ra) - ordered(rb)).max()) if ra.size else 0


def cache_of(kv) -> w.PagedCache:
    """synth.PagedKV -> the binding's PagedCache."""
    return w.PagedCache(kv.k_pool, kv.v_pool, kv.page_table, kv.kv_len)


def dense_kv_f64(kv, b: int, length: int, kv_head: int):
    """fp64 K, V ``[length, D]`` of one sequence and KV head (gathered on the
    device through the page table, converted on the host)."""
    P = kv.page_size
    npg = -(-length // P)
    pages = kv.page_table[b, :npg].long()
    k = kv.k_pool[pages, kv_head].reshape(npg * P, -1)[:length]
    v = kv.v_pool[pages, kv_head].reshape(npg * P, -1)[:length]
    return f64(k), f64(v)

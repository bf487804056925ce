// The compact draft ring buffer of Windowed-MTP, and the paged-cache writer.
//
// Ring ("Windowed-MTP ..." arxivlens view, Abstract and Technical
// contributions: a compact ring buffer keeps only the sink + window entries of
// the draft KV).  Per sequence: S + W slots; position p lives in slot p when
// p < S, else in slot S + (p - S) mod W.  Speculative appends save the entry
// they overwrite into an undo log so a rejected draft token can be rolled
// back exactly; a non-speculative call commits.  After every call the ring
// holds exactly positions {0..min(S,len)-1} U {max(S,len-W)..len-1}.
//
// Everything here is a byte copy, so the results are bit-exact.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "decode_attn.cuh"  // status bits, set_status

namespace wmtp {

constexpr int kRingThreads = 256;

struct RingArgs {
  uint4* k;  // [B][Hkv][R][D] bf16, addressed in 16-byte units
  uint4* v;
  int32_t* tags;  // [B][R]
  int32_t* len;   // [B]
  int32_t* committed;
  uint4* undo_k;  // [B][gmax][Hkv][D]
  uint4* undo_v;
  int32_t* undo_tags;  // [B][gmax]
  int batch, Hkv, D, S, W, R, gmax;
};

__device__ __forceinline__ int ring_slot(int p, int S, int W) { return p < S ? p : S + (p - S) % W; }

// 16-byte unit u of token row `slot`, KV head h, for sequence b.
__device__ __forceinline__ size_t ring_unit(const RingArgs& r, int b, int h, int slot, int c) {
  return ((static_cast<size_t>(b) * r.Hkv + h) * r.R + slot) * (r.D / 8) + c;
}
__device__ __forceinline__ size_t undo_unit(const RingArgs& r, int b, int j, int h, int c) {
  return ((static_cast<size_t>(b) * r.gmax + j) * r.Hkv + h) * (r.D / 8) + c;
}

// One CTA per sequence.
__global__ void __launch_bounds__(kRingThreads)
    ring_append_kernel(RingArgs r, const int32_t* __restrict__ truncate_to,
                       const int32_t* __restrict__ n_new, const uint4* __restrict__ k_new,
                       const uint4* __restrict__ v_new, int max_new, int speculative,
                       int32_t* status) {
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  __shared__ int s_ok, s_len, s_com, s_target, s_n;
  // launched as a programmatic dependent: wait (unconditionally, before any
  // memory access) for the work before it on the stream, then let the
  // attention kernel behind it get scheduled
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    const int len = r.len[b];
    const int com = r.committed[b];
    int ok = (com >= 0 && len >= com && len - com <= r.gmax) ? 1 : 0;
    const int tt = (truncate_to != nullptr) ? truncate_to[b] : -1;
    int target = len;
    if (ok && tt >= 0) {
      if (tt < com || tt > len)
        ok = 0;
      else
        target = tt;
    }
    const int n = (n_new != nullptr && max_new > 0) ? n_new[b] : 0;
    if (n < 0 || n > max_new) ok = 0;
    if (!ok) {
      set_status(status, kDevRingState);
    } else if (speculative && (target - com) + n > r.gmax) {
      ok = 0;
      set_status(status, kDevUndoFull);
    }
    s_ok = ok;
    s_len = len;
    s_com = com;
    s_target = target;
    s_n = n;
  }
  __syncthreads();
  if (!s_ok) return;
  const int com = s_com;
  const int target = s_target;
  const int n = s_n;
  const int upt = r.D / 8;          // 16-byte units per head row
  const int units = r.Hkv * upt;    // per token

  // 1. roll back speculative entries, newest first (two of them may share a
  //    slot when W is small, so this is sequential in p)
  for (int p = s_len - 1; p >= target; --p) {
    const int j = p - com;
    const int slot = ring_slot(p, r.S, r.W);
    for (int u = tid; u < units; u += kRingThreads) {
      const int h = u / upt, c = u % upt;
      r.k[ring_unit(r, b, h, slot, c)] = r.undo_k[undo_unit(r, b, j, h, c)];
      r.v[ring_unit(r, b, h, slot, c)] = r.undo_v[undo_unit(r, b, j, h, c)];
    }
    if (tid == 0) r.tags[static_cast<size_t>(b) * r.R + slot] = r.undo_tags[static_cast<size_t>(b) * r.gmax + j];
    __syncthreads();
  }

  // 2. append
  const int len = target;
  if (speculative) {
    for (int j = 0; j < n; ++j) {
      const int p = len + j;
      const int slot = ring_slot(p, r.S, r.W);
      const int ui = p - com;
      for (int u = tid; u < units; u += kRingThreads) {
        const int h = u / upt, c = u % upt;
        const size_t ri = ring_unit(r, b, h, slot, c);
        const size_t di = undo_unit(r, b, ui, h, c);
        const size_t si = (static_cast<size_t>(b) * max_new + j) * units + u;
        r.undo_k[di] = r.k[ri];
        r.undo_v[di] = r.v[ri];
        r.k[ri] = k_new[si];
        r.v[ri] = v_new[si];
      }
      if (tid == 0) {
        r.undo_tags[static_cast<size_t>(b) * r.gmax + ui] = r.tags[static_cast<size_t>(b) * r.R + slot];
        r.tags[static_cast<size_t>(b) * r.R + slot] = p;
      }
      __syncthreads();
    }
  } else {
    // only the tokens that survive in the final sink + window are written;
    // their slots are distinct, so this is order-free
    const int fin = len + n;
    const int a0 = len, a1 = min(r.S, fin);
    const int w0 = max(max(len, fin - r.W), r.S), w1 = fin;
    const int ns = max(a1 - a0, 0), nw = max(w1 - w0, 0);
    const long long total = static_cast<long long>(ns + nw) * units;
    for (long long idx = tid; idx < total; idx += kRingThreads) {
      const int i = static_cast<int>(idx / units);
      const int u = static_cast<int>(idx % units);
      const int p = (i < ns) ? a0 + i : w0 + (i - ns);
      const int j = p - len;
      const int slot = ring_slot(p, r.S, r.W);
      const int h = u / upt, c = u % upt;
      const size_t si = (static_cast<size_t>(b) * max_new + j) * units + u;
      r.k[ring_unit(r, b, h, slot, c)] = k_new[si];
      r.v[ring_unit(r, b, h, slot, c)] = v_new[si];
      if (u == 0) r.tags[static_cast<size_t>(b) * r.R + slot] = p;
    }
  }
  __syncthreads();
  if (tid == 0) {
    r.len[b] = len + n;
    if (!speculative) r.committed[b] = len + n;
  }
}

// Empty every ring: zero K/V and undo, tags -1, lengths 0.
__global__ void ring_reset_kernel(RingArgs r) {
  const size_t ring_units = static_cast<size_t>(r.batch) * r.Hkv * r.R * (r.D / 8);
  const size_t undo_units = static_cast<size_t>(r.batch) * r.gmax * r.Hkv * (r.D / 8);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < ring_units; i += stride) {
    r.k[i] = z;
    r.v[i] = z;
  }
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < undo_units; i += stride) {
    r.undo_k[i] = z;
    r.undo_v[i] = z;
  }
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
       i < static_cast<size_t>(r.batch) * r.R; i += stride)
    r.tags[i] = -1;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
       i < static_cast<size_t>(r.batch) * r.gmax; i += stride)
    r.undo_tags[i] = -1;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < static_cast<size_t>(r.batch);
       i += stride) {
    r.len[i] = 0;
    r.committed[i] = 0;
  }
}

// Write n_new tokens per sequence into a paged cache: grid (n_new, batch).
// `len_end`: NULL, or [batch] lengths whose last n_new positions are written
// (pos0 then unused): the append in front of a verify whose new tokens end
// the sequence.
__global__ void paged_write_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool, int num_pages,
                                   const int32_t* __restrict__ page_table, int max_pages, int P,
                                   int Hkv, int D, const int32_t* __restrict__ pos0, int n_new,
                                   const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                   int32_t* status, const int32_t* __restrict__ len_end) {
  const int j = blockIdx.x;
  const int b = blockIdx.y;
  // launched as a programmatic dependent: wait (unconditionally, before any
  // memory access) for the work before it on the stream, then let the
  // attention kernel behind it get scheduled
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int p = (len_end != nullptr ? len_end[b] - n_new : pos0[b]) + j;
  if (p < 0 || p >= max_pages * P) {
    if (threadIdx.x == 0) set_status(status, kDevLenOob);
    return;
  }
  const int pg = page_table[static_cast<size_t>(b) * max_pages + p / P];
  if (pg < 0 || pg >= num_pages) {
    if (threadIdx.x == 0) set_status(status, kDevPageOob);
    return;
  }
  const int row = p % P;
  const int upt = D / 8;
  for (int u = threadIdx.x; u < Hkv * upt; u += blockDim.x) {
    const int h = u / upt, c = u % upt;
    const size_t dst = ((static_cast<size_t>(pg) * Hkv + h) * P + row) * upt + c;
    const size_t src = ((static_cast<size_t>(b) * n_new + j) * Hkv + h) * upt + c;
    k_pool[dst] = k_new[src];
    v_pool[dst] = v_new[src];
  }
}

}  // namespace wmtp

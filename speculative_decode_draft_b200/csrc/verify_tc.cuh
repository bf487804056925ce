// Verify attention on the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
//
// The target verifies gamma+1 draft tokens with causal attention over its
// full paged KV ("Windowed-MTP ..." arxivlens view, Abstract: verification
// stays full-context).  All rows = (gamma+1) x G query heads of one KV head
// share each K/V byte; with G = 8 that is 16..72 rows against every token
// for gamma = 1..8.
//
// Per CTA = (split, KV head, sequence), head_dim 256, 64-token tiles, with
// the rows as the MMA M dimension (padded to M = 64, or to M = 128 for blocks
// of 65..128 rows such as gamma = 8 with G = 8) and everything but K and V
// kept in tensor memory (512 columns; the M=64 layout uses lanes 0..15 of
// each of the four lane quadrants, M=128 all 32):
//   columns   0..127  Q            bf16 pairs, the A operand of S = Q K^T
//   columns 128..255  S / P x 2    fp32 scores of a tile; after the softmax
//                                  columns 0..31 of the buffer hold P as fp16
//                                  pairs, the A operand of P V
//   columns 256..511  O            fp32 output accumulator, 256 head dims
// Row r of the block sits in TMEM lane 32 (r % 4) + r / 4 (M row
// 16 (r % 4) + r / 4 for M=64, 32 (r % 4) + r / 4 for M=128), so the rows
// spread over the four lane quadrants and each softmax warp owns a quarter of
// them.
//
// Roles:
//   warp 0     streams K and V tiles (64 x 256 bf16 each, 128-byte swizzle)
//              into two shared-memory rings (KS and VS tiles deep) with TMA,
//              one lane per ring; a K tile is released as soon as its
//              S = Q K^T has completed, a V tile only after its O += P V, so K
//              loads run ahead of the softmax;
//   warp 1     allocates the tensor memory; one lane issues S = Q K^T (M rows,
//              N=64, K from shared memory, K-major);
//   warp 10    one lane issues O += P V (M rows, N=256, V read MN-major
//              straight from the TMA tile).  A lane issues a small tcgen05.mma only
//              every ~66 cycles, so the two streams issue from two lanes;
//   warps 2-5  stage Q into TMEM, then run the softmax, one thread per row:
//              the row's scores come out of TMEM, the maximum and sum are
//              taken inside the thread, and P goes back into TMEM in fp16;
//   warps 6-9  convert each landed V tile in place from bf16 to fp16 (and
//              zero its rows past the sequence end).
// The value product is therefore fp16 x fp16 -> fp32: P carries a relative
// rounding of at most 2^-11 (bf16 would give 2^-8 and miss a 1e-3 relative-L2
// bound), and V is exact for every |v| < 2^16 (below 2^-17 the absolute error
// stays under 2^-25); a larger |v| saturates and raises WMTP_DEV_V_RANGE.
// P is stored as 2^(s - m_ref + 7): the largest weight is then 2^15 (inside
// fp16's 65504) and weights stay normal fp16 numbers down to 2^-21 of the
// reference maximum.  Without the offset, a weight below 2^-14 would fall
// into fp16's subnormal range, where the rounding is absolute (2^-25); a
// large sea of nearly equal small weights next to one dominant key (an
// attention sink) would then be rounded the same way and bias the output.  One
// fp16 MMA per 16 tokens (an N=256 MMA keeps the tensor pipe ~134 cycles)
// instead of a bf16 hi + lo pair is what keeps PV well under the HBM time of
// a tile.
// The reference maximum of a row is raised only when the tile maximum
// exceeds it by more than 2^8 (with the 2^7 offset, weights then stay at or
// below 2^15), and only then is that row of O rescaled in TMEM, after the
// previous PV completed.
//
// Every mbarrier wait is bounded; a wait that gives up raises
// WMTP_DEV_TIMEOUT and stops the pipeline; the producers still wait (bounded)
// for their copies in flight and the issuing lanes for their MMAs, and the
// tensor memory is freed before the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "decode_attn.cuh"
#include "ptx.cuh"

namespace wmtp {

constexpr int kTcThreads = 352;       // producers, QK issuer, 4 softmax warps, 4 V converter warps, PV issuer
constexpr int kPvWarp = 10;
constexpr int kBarTmem = 3;           // named barrier: MMA + softmax warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;
constexpr uint32_t kColS = 128;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.f;   // lazy rescale threshold (log2 units)
constexpr float kPShiftLog2 = 7.f;    // P = 2^(s - m_ref + 7) <= 2^15 in fp16

template <int KS, int VS>
struct TcPlan {
  static constexpr int kChunkBytes = 64 * 128;           // 64 tokens x 128 B
  static constexpr int kTileBytes = 4 * kChunkBytes;      // one K or V tile, D = 256
  static constexpr int kOffK = 0;                         // K ring: KS tiles
  static constexpr int kOffV = KS * kTileBytes;           // V ring: VS tiles
  static constexpr int kOffBar = (KS + VS) * kTileBytes;
  // k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], v_ready[VS], s_full[2],
  // p_full[2], o_done, mma_final, q_ready, pv_done[2]
  static constexpr int kNumBars = 2 * KS + 3 * VS + 9;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort
  static constexpr int kBytes = kOffMisc + 8;
  static constexpr int kAlloc = kBytes + 1024;
};

// Depths of the K and V rings (64-token tiles).  K tiles leave as soon as QK
// has read them and V tiles only after the softmax and PV, yet 2 + 4 measured
// slower than 3 + 3 on B200 (398-404 against 393-396 us per 1M layer).
constexpr int kTcKStages = 3;
constexpr int kTcVStages = 3;

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag != 0) return false;
    if (clock64() - t0 > ptx::kWaitLimitCycles) return false;
  }
}

// M: MMA rows (64 or 128); the block's rows must not exceed it.
template <int KS, int VS, int M>
__global__ void __launch_bounds__(kTcThreads, 1)
    verify_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const DecodeArgs a) {
  using Plan = TcPlan<KS, VS>;
  constexpr int D = 256;
  static_assert(M == 64 || M == 128, "MMA rows: 64 or 128");
  constexpr int kLanesPerQuadrant = M / 4;  // TMEM lanes of each quadrant that hold rows

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t bar0 = sbase + Plan::kOffBar;
  const uint32_t bar_k_full = bar0;
  const uint32_t bar_k_empty = bar_k_full + 8 * KS;
  const uint32_t bar_v_full = bar_k_empty + 8 * KS;
  const uint32_t bar_v_empty = bar_v_full + 8 * VS;
  const uint32_t bar_v_ready = bar_v_empty + 8 * VS;
  const uint32_t bar_s_full = bar_v_ready + 8 * VS;
  const uint32_t bar_p_full = bar_s_full + 16;
  const uint32_t bar_o_done = bar_p_full + 16;
  const uint32_t bar_final = bar_o_done + 8;
  const uint32_t bar_q_ready = bar_final + 8;
  const uint32_t bar_pv_done = bar_q_ready + 8;  // [2]: PV of the tiles using S/P buffer 0 / 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Plan::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Plan::kOffMisc + 4);

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- set-up: barriers and tensor memory
  if (threadIdx.x == 0) {
    for (int s = 0; s < KS; ++s) {
      ptx::mbar_init(bar_k_full + 8 * s, 1);
      ptx::mbar_init(bar_k_empty + 8 * s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      ptx::mbar_init(bar_v_full + 8 * s, 1);
      ptx::mbar_init(bar_v_empty + 8 * s, 1);
      ptx::mbar_init(bar_v_ready + 8 * s, 4);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar_s_full + 8 * i, 1);
      ptx::mbar_init(bar_p_full + 8 * i, 4);
    }
    ptx::mbar_init(bar_o_done, 1);
    ptx::mbar_init(bar_final, 2);  // one commit from each MMA-issuing lane
    ptx::mbar_init(bar_pv_done, 1);
    ptx::mbar_init(bar_pv_done + 8, 1);
    ptx::mbar_init(bar_q_ready, 4);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  // every global-memory access comes after this: with a programmatic launch
  // the set-up above overlaps the previous kernel's tail
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- token range of this split
  int n_tok = a.kv_len[b];
  if (n_tok != 0 &&
      ((a.q_pos0 == nullptr && n_tok < a.num_q) || n_tok < 0 || n_tok > a.max_pages * a.page_size)) {
    if (threadIdx.x == 0 && split == 0 && kvh == 0) set_status(a.status, kDevLenOob);
    n_tok = 0;
  }
  const int ntiles = (n_tok + kTileTokens - 1) / kTileTokens;
  const int tps = (ntiles + a.nsplit - 1) / a.nsplit;
  const int t_begin = min(split * tps, ntiles);
  const int t_end = min(t_begin + tps, ntiles);
  const int my_tiles = t_end - t_begin;
  // start the page-table reads of the first tiles now; the producers' own
  // loads then hit L2
  if (warp == 0 && lane < VS && lane < my_tiles) {
    const int* pte = a.page_table + static_cast<size_t>(b) * a.max_pages +
                     ((t_begin + lane) * kTileTokens) / a.page_size;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(pte));
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  // softmax-thread identity: TMEM lane m = 32 q + lane holds row 4 lane + q
  const int q = warp & 3;
  const int row = 4 * lane + q;
  const bool row_active = warp >= 2 && warp < 6 && lane < kLanesPerQuadrant && row < a.rows;
  const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;

  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // =================================================================== producers
  // lane 0 loads K tiles, lane 1 loads V tiles; each has its own ring
  if (warp == 0) {
    if (lane < 2 && my_tiles > 0) {
      const bool is_k = lane == 0;
      const CUtensorMap* tmap = is_k ? &tmap_k : &tmap_v;
      ptx::prefetch_tmap(tmap);
      const uint64_t pol = ptx::policy_evict_first();
      const int box_rows = min(a.page_size, kTileTokens);
      const int boxes = kTileTokens / box_rows;
      const int oob_z = a.num_pages * a.Hkv;  // past the tensor: zero fill
      const uint32_t bar_full = is_k ? bar_k_full : bar_v_full;
      const uint32_t bar_empty = is_k ? bar_k_empty : bar_v_empty;
      const uint32_t ring = sbase + (is_k ? Plan::kOffK : Plan::kOffV);
      const int nst = is_k ? KS : VS;  // stages of this lane's ring
      int issued = 0;
      for (int k = 0; k < my_tiles; ++k) {
        const int stage = k % nst;
        if (!tc_wait(bar_empty + 8 * stage, ((k / nst) & 1) ^ 1, abort_flag)) {
          if (*abort_flag == 0) set_status(a.status, kDevTimeout);
          *abort_flag = 1;
          break;
        }
        const int tok0 = (t_begin + k) * kTileTokens;
        const uint32_t dst = ring + stage * Plan::kTileBytes;
        const uint32_t fb = bar_full + 8 * stage;
        int zs[4], ys[4];
        int valid = 1;
        for (int j = 0; j < boxes; ++j) {
          const int tok = tok0 + j * box_rows;
          zs[j] = oob_z;
          ys[j] = 0;
          if (tok >= n_tok) continue;
          const int lp = tok / a.page_size;
          const int pg = a.page_table[static_cast<size_t>(b) * a.max_pages + lp];
          if (pg < 0 || pg >= a.num_pages) {
            valid = 0;
          } else {
            zs[j] = pg * a.Hkv + kvh;
            ys[j] = tok - lp * a.page_size;
          }
        }
        if (is_k && !valid) set_status(a.status, kDevPageOob);
        ptx::mbar_arrive_expect_tx(fb, Plan::kTileBytes);
        for (int j = 0; j < boxes; ++j) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            ptx::tma_load_3d(dst + c * Plan::kChunkBytes + j * box_rows * 128, tmap, fb, c * 64, ys[j], zs[j], pol);
        }
        issued = k + 1;
      }
      // no copy may still be writing shared memory when the CTA exits (after
      // an abort the consumers stop early): wait, bounded, for the last load
      // of each stage
      for (int k = max(issued - nst, 0); k < issued; ++k)
        if (!ptx::mbar_wait(bar_full + 8 * (k % nst), (k / nst) & 1)) set_status(a.status, kDevTimeout);
    }
    return;
  }

  // =================================================================== V converters
  if (warp >= 6 && warp < kPvWarp) {
    const int cw = warp - 6;  // one 8 KB column chunk (64 head dims) of the V tile per warp
    uint32_t vexp = 0;        // per-half maximum of the bf16 exponent fields seen
    for (int k = 0; k < my_tiles; ++k) {
      const int stage = k % VS;
      if (!__all_sync(0xffffffffu, tc_wait(bar_v_full + 8 * stage, (k / VS) & 1, abort_flag))) {
        if (lane == 0) set_status(a.status, kDevTimeout);
        *abort_flag = 1;
        break;
      }
      const int tok0 = (t_begin + k) * kTileTokens;
      const int rows_valid = min(kTileTokens, n_tok - tok0);
      const uint32_t chunk = sbase + Plan::kOffV + stage * Plan::kTileBytes + cw * Plan::kChunkBytes;
#pragma unroll 4
      for (int u = lane; u < Plan::kChunkBytes / 16; u += 32) {
        const uint32_t addr = chunk + 16 * u;
        uint4 w;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                     : "r"(addr));
        if (u / 8 < rows_valid) {  // 8 sixteen-byte units per 128-byte row
          vexp = __vmaxu2(vexp, __vmaxu2(w.x & 0x7f807f80u, w.y & 0x7f807f80u));
          vexp = __vmaxu2(vexp, __vmaxu2(w.z & 0x7f807f80u, w.w & 0x7f807f80u));
          w.x = ptx::bf16x2_to_f16x2_sat(w.x);
          w.y = ptx::bf16x2_to_f16x2_sat(w.y);
          w.z = ptx::bf16x2_to_f16x2_sat(w.z);
          w.w = ptx::bf16x2_to_f16x2_sat(w.w);
        } else {  // past the end of the sequence: zero, so 0-weight rows add 0
          w = make_uint4(0, 0, 0, 0);
        }
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w.x), "r"(w.y), "r"(w.z),
                     "r"(w.w)
                     : "memory");
      }
      ptx::fence_proxy_async_smem();  // generic writes before the tensor core reads
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_v_ready + 8 * stage);
    }
    // a bf16 exponent field of 143 or more means |v| >= 2^16
    if ((vexp & 0xffffu) >= (143u << 7) || (vexp >> 16) >= (143u << 7)) set_status(a.status, kDevVRange);
    return;
  }

  // =================================================================== PV issuer
  // O += P(k) V(k) for every tile, issued by its own lane: a single lane
  // issues a small tcgen05.mma only every ~66 cycles, so the QK and PV
  // streams run from two lanes and overlap in the tensor pipe.
  if (warp == kPvWarp) {
    if (lane == 0 && my_tiles > 0) {
      constexpr uint32_t kIdescPV = tc::idesc_f16_f32(M, 256, 0, 1);     // A (P, TMEM), B (V) MN-major, fp16
      const uint64_t v_desc0 = tc::smem_desc_sw128(sbase + Plan::kOffV, Plan::kChunkBytes, 1024);
      bool ok = true;
      for (int k = 0; ok && k < my_tiles; ++k) {
        ok = tc_wait(bar_p_full + 8 * (k & 1), (k >> 1) & 1, abort_flag) &&
             tc_wait(bar_v_ready + 8 * (k % VS), (k / VS) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        const uint64_t vd = v_desc0 + (static_cast<uint64_t>((k % VS) * Plan::kTileBytes) >> 4);
        const uint32_t p_tmem = tmem_base + kColS + (k & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          const uint64_t bd = vd + (static_cast<uint32_t>(kk * 2048) >> 4);
          tc::mma_ts(tmem_base + kColO, p_tmem + 8 * kk, bd, kIdescPV, (k > 0 || kk > 0) ? 1u : 0u);
        }
        tc::commit(bar_v_empty + 8 * (k % VS));
        tc::commit(bar_o_done);
        tc::commit(bar_pv_done + 8 * (k & 1));
      }
      if (!ok) {
        if (*abort_flag == 0) set_status(a.status, kDevTimeout);
        *abort_flag = 1;
      }
      // mma_final completes when both issuing lanes' MMAs have all completed
      tc::commit(bar_final);
      if (!ptx::mbar_wait(bar_final, 0)) set_status(a.status, kDevTimeout);
    }
    return;
  }

  // =================================================================== QK issuer
  if (warp == 1) {
    if (lane == 0 && my_tiles > 0) {
      // M = 64 whenever the rows fit: an M=64 MMA costs the same issue time
      // as M=128 for half the tensor work (and power)
      constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(M, 64, 0, 0);     // A (Q, TMEM), B (K) K-major
      // descriptor start addresses are in 16-byte units in the low bits, so
      // moving an operand by n bytes adds n >> 4 to the descriptor
      const uint64_t k_desc0 = tc::smem_desc_sw128(sbase + Plan::kOffK, 16, 1024);
      // Q is staged into TMEM by the softmax warps while the first K/V tiles
      // are in flight
      bool ok = tc_wait(bar_q_ready, 0, abort_flag);
      for (int k = 0; ok && k < my_tiles; ++k) {
        // S/P buffer k & 1 last held P(k-2): PV(k-2), issued by the other
        // lane, must have completed (its phase of pv_done; the next phase
        // needs P(k), which needs this S)
        if (k >= 2 && !(ok = tc_wait(bar_pv_done + 8 * (k & 1), ((k - 2) >> 1) & 1, abort_flag))) break;
        if (!(ok = tc_wait(bar_k_full + 8 * (k % KS), (k / KS) & 1, abort_flag))) break;
        tc::fence_after_sync();
        const uint64_t kd = k_desc0 + (static_cast<uint64_t>((k % KS) * Plan::kTileBytes) >> 4);
        const uint32_t d_tmem = tmem_base + kColS + (k & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * Plan::kChunkBytes + (kk & 3) * 32;
          tc::mma_ts(d_tmem, tmem_base + kColQ + 8 * kk, kd + (ka >> 4), kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc::commit(bar_s_full + 8 * (k & 1));
        tc::commit(bar_k_empty + 8 * (k % KS));
      }
      if (!ok) {
        if (*abort_flag == 0) set_status(a.status, kDevTimeout);
        *abort_flag = 1;
      }
      // wait (bounded) until every MMA of both issuing lanes has completed,
      // so the tensor memory is never freed under a running MMA
      tc::commit(bar_final);
      if (!ptx::mbar_wait(bar_final, 0)) set_status(a.status, kDevTimeout);
    }
    __syncwarp();
  } else {
    // ================================================================= softmax
    {
      // Q row into TMEM columns 0..127 (bf16 pairs), zeros for padding rows;
      // every load is issued before the first store so the row costs one
      // global-memory round trip
      const __nv_bfloat16* src =
          row_active ? a.q + ((static_cast<size_t>(b) * a.num_q + row / a.G) * a.Hq + kvh * a.G + row % a.G) * D
                     : nullptr;
      uint4 v[D / 8];
#pragma unroll
      for (int j = 0; j < D / 8; ++j)
        v[j] = row_active ? *reinterpret_cast<const uint4*>(src + 8 * j) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t wq[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          wq[4 * j] = v[8 * c + j].x;
          wq[4 * j + 1] = v[8 * c + j].y;
          wq[4 * j + 2] = v[8 * c + j].z;
          wq[4 * j + 3] = v[8 * c + j].w;
        }
        tc::tmem_st32(tmem_base + lane_addr + kColQ + 32 * c, wq);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_q_ready);
    }
    // query i attends positions <= q_first + i of this cache (q_first is
    // kv_len - num_q unless the call covers a slice of a longer sequence)
    const int q_first = a.q_pos0 != nullptr ? a.q_pos0[b] : n_tok - a.num_q;
    const int lim = row_active ? min(n_tok, q_first + row / a.G + 1) : n_tok;  // causal limit of this row
    const int first_masked_tok = min(n_tok, q_first + 1);
    float m_ref = -INFINITY;  // reference maximum (log2 units)
    float l_run = 0.f;
    bool failed = false;

    for (int k = 0; k < my_tiles; ++k) {
      const int sb = k & 1;
      // S(k) complete implies K(k) landed.  (The K ring itself is not waited
      // on here: its stage may already hold a later tile, so a parity wait on
      // it would be ambiguous.)
      const bool ok = __all_sync(0xffffffffu, tc_wait(bar_s_full + 8 * sb, (k >> 1) & 1, abort_flag));
      if (!ok) {
        failed = true;
        break;  // this warp stops; the MMA warp times out or sees the abort
      }
      tc::fence_after_sync();
      const int tok0 = (t_begin + k) * kTileTokens;
      // a tile with a page outside the pool is skipped (the producers loaded
      // zeros for it and raised WMTP_DEV_PAGE_OOB)
      bool tile_ok = true;
      for (int tok = tok0; tok < min(tok0 + kTileTokens, n_tok); tok += min(a.page_size, kTileTokens)) {
        const int pg = a.page_table[static_cast<size_t>(b) * a.max_pages + tok / a.page_size];
        tile_ok = tile_ok && pg >= 0 && pg < a.num_pages;
      }
      const uint32_t s_addr = tmem_base + lane_addr + kColS + sb * 64;

      uint32_t sraw[64];
      tc::tmem_ld32(s_addr, sraw);
      tc::tmem_ld32(s_addr + 32, sraw + 32);
      float x[64];
      float mx = -INFINITY;
      if (tok0 + kTileTokens <= first_masked_tok) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          x[j] = tile_ok ? __uint_as_float(sraw[j]) * a.scale_log2 : -INFINITY;
          mx = fmaxf(mx, x[j]);
        }
      } else {  // tile holding the causal tail and/or the end of the sequence
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int t = tok0 + j;
          x[j] = (tile_ok && t < lim && t < n_tok) ? __uint_as_float(sraw[j]) * a.scale_log2 : -INFINITY;
          mx = fmaxf(mx, x[j]);
        }
      }
      // raise the reference maximum only when the tile exceeds it by more
      // than 2^8; rows whose reference moved rescale their O row and sum
      float alpha = 1.f;
      bool moved = false;
      if (mx > m_ref + kRescaleLog2 || (m_ref == -INFINITY && mx != -INFINITY)) {
        alpha = (m_ref == -INFINITY) ? 0.f : ptx::ex2(m_ref - mx);
        moved = m_ref != -INFINITY;
        m_ref = mx;
      }
      const float base = (m_ref == -INFINITY) ? 0.f : m_ref - kPShiftLog2;
      if (__any_sync(0xffffffffu, moved)) {
        // PV(k-1) must have finished before O is rewritten.  S(k) arriving
        // implies PV(k-2) completed (issued before QK(k)), so the pending
        // o_done phase is PV(k-1)'s and a parity wait is unambiguous.
        if (!__all_sync(0xffffffffu, tc_wait(bar_o_done, (k - 1) & 1, abort_flag))) {
          failed = true;
          break;
        }
        tc::fence_after_sync();
        const float f = moved ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(tmem_base + lane_addr + kColO + 32 * c, o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          tc::tmem_st32(tmem_base + lane_addr + kColO + 32 * c, o);
        }
      }
      // P = 2^(x - m_ref + 7) as fp16 pairs, back into the S columns
      float sum = 0.f;
      uint32_t ph[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float p0 = ptx::ex2(x[2 * j] - base);  // 2^-inf = 0 for masked entries
        const float p1 = ptx::ex2(x[2 * j + 1] - base);
        sum += p0 + p1;
        ph[j] = ptx::pack_f16x2(p0, p1);
      }
      l_run = l_run * alpha + sum;
      tc::tmem_st32(s_addr, ph);

      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_p_full + 8 * sb);
    }

    // ---- finish: normalised partial output and log-sum-exp of this row
    if (!failed && my_tiles > 0) {
      // mma_final completes once, when every MMA of the CTA has completed (a
      // parity wait on o_done could not tell PV(n-2)'s phase from PV(n)'s
      // once both PV(n-2) and PV(n-1) have completed)
      if (!__all_sync(0xffffffffu, tc_wait(bar_final, 0, abort_flag))) failed = true;
      tc::fence_after_sync();
    }
    failed = __any_sync(0xffffffffu, failed || *abort_flag != 0);
    if (failed) {
      if (lane == 0) set_status(a.status, kDevTimeout);
      *abort_flag = 1;
    }
    const float inv = (l_run > 0.f && !failed) ? 1.f / l_run : 0.f;
    const size_t grow =
        row_active ? (static_cast<size_t>(b) * a.num_q + row / a.G) * a.Hq + kvh * a.G + row % a.G : 0;
    float* dst = a.part_o + (grow * a.nsplit + split) * D;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {  // two 128-column TMEM loads per row
      uint32_t o[128];
      if (my_tiles > 0 && !failed) {
        tc::tmem_ld128(tmem_base + lane_addr + kColO + 128 * c, o);
      } else {
#pragma unroll
        for (int j = 0; j < 128; ++j) o[j] = 0u;
      }
      if (row_active) {
#pragma unroll
        for (int j = 0; j < 128; j += 4)
          *reinterpret_cast<float4*>(dst + 128 * c + j) =
              make_float4(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv,
                          __uint_as_float(o[j + 2]) * inv, __uint_as_float(o[j + 3]) * inv);
      }
    }
    if (row_active) {
      // m_ref is in log2 units of the scaled score; l_run carries the 2^7
      // offset of P
      a.part_lse[grow * a.nsplit + split] =
          (l_run > 0.f && !failed) ? (m_ref - kPShiftLog2) * 0.69314718055994531f + logf(l_run) : -INFINITY;
    }
    tc::fence_before_sync();
  }

  // ---- every MMA has completed (the MMA lane waited for its final commit);
  // free the tensor memory
  ptx::named_bar_sync(kBarTmem, 160);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace wmtp

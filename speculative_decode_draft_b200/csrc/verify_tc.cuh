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
// each of the four lane quadrants, M=128 all 32).  For M = 64, Q sits in
// shared memory and the scores have three TMEM buffers; for M = 128 (Q is
// twice as large) Q sits in TMEM and the scores have two:
//   M = 64:  columns 0..191 S / P x 3, columns 256..511 O
//   M = 128: columns 0..127 Q (bf16 pairs), 128..255 S / P x 2, 256..511 O
// An S buffer holds a tile's fp32 scores; after the softmax its columns 0..31
// hold P_hi and 32..63 P_lo as bf16 pairs (P = hi + lo).  A block of up to
// 32 rows uses only half of the M = 64 lanes, so there P_lo goes to the
// row's spare lane (M row + 8) in columns 0..31 and one MMA per 16 tokens
// takes both; O's spare-lane rows then hold the P_lo products, added to
// their row at the end.  O is the fp32 output accumulator, 256 head dims.
// QK(k) may overwrite buffer k % NB only once PV(k - NB) has read it, so
// with three buffers the QK of a tile no longer waits for the PV of the
// tile just before the previous one.
// Row r of the block sits in TMEM lane 32 (r % 4) + r / 4 (M row
// 16 (r % 4) + r / 4 for M=64, 32 (r % 4) + r / 4 for M=128), so the rows
// spread over the four lane quadrants and each pair of softmax warps owns a
// quarter of them.
//
// Roles (12 warps):
//   warps 0, 3 stream K (warp 0) and V (warp 3) tiles (64 x 256 bf16 each,
//              128-byte swizzle) into two shared-memory rings (KS and VS tiles
//              deep) with TMA, one lane each; a K tile is released as soon as
//              its S = Q K^T has completed, a V tile after its O += P V.  The
//              two producers sit in different warps so that neither one's
//              barrier wait holds up the other's issue;
//   warp 1     allocates the tensor memory; one lane issues S = Q K^T (M rows,
//              N=64, K from shared memory, K-major);
//   warp 2     one lane issues O += P V (M rows, N=256, V read MN-major
//              straight from the TMA tile, bf16).  A lane issues a small
//              tcgen05.mma only every ~66 cycles, so the two streams issue
//              from two lanes;
//   warps 4-11 stage Q, then run the softmax: two warps per TMEM lane
//              quadrant (warp % 4), one per half of the tile's 64 columns
//              (and of O's 256).  A warp covers the rows of its quadrant with
//              sixteen-lane TMEM accesses: four threads share a row and take
//              8 of its half's 32 scores each, so every lane works even when
//              a quadrant holds only 8 rows (gamma = 3, G = 8).  Row maxima
//              meet through two shuffles, then between the two halves
//              through shared memory and a two-warp mbarrier; both halves
//              then take the same rescale decisions.  P goes back into TMEM.
//              The softmax is the per-tile critical path once a quadrant
//              holds more than 8 rows (gamma >= 5), so it gets eight warps.
// The value product is bf16 x bf16 -> fp32 on two MMAs per 16 tokens: P is
// split into P_hi = bf16(p) and P_lo = bf16(p - P_hi), |p - P_hi - P_lo| <=
// 2^-16 p (a single bf16 P, 2^-8, would miss a 1e-3 relative-L2 bound), and V
// enters in its own bf16 format, exactly and at any magnitude.
// The reference maximum of a row is raised only when the tile maximum
// exceeds it by more than 2^8 (weights then stay at or below 2^8), and only
// then is that row of O rescaled in TMEM, after the previous PV completed.
//
// Accumulation runs: a tensor-core accumulation adds each product to the
// fp32 accumulator at the accumulator's precision, so a product far smaller
// than the running sum loses low-order bits.  Over a long split of nearly
// equal weights and values of one sign (a flat stretch of attention) that
// loss is systematic, ~n 2^-25 of the result after n products.  Every
// kRunTiles tiles the softmax threads therefore fold the accumulator into the
// split's fp32 partial in global memory (exact fp32 adds) and the next PV
// starts a fresh accumulation; a run then spans at most 16,384 tokens
// (kRunTiles, shared with the mma.sync kernel).
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

constexpr int kTcThreads = 384;       // K producer, QK issuer, PV issuer, V producer, 8 softmax warps
constexpr int kPvWarp = 2;
constexpr int kVWarp = 3;
constexpr int kSmWarp0 = 4;           // softmax warps 4..11
constexpr int kSmThreads = 256;
constexpr int kBarTmem = 3;           // named barrier: QK issuer + softmax warps
constexpr int kBarSoftmax = 4;        // named barrier: the softmax warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.f;   // lazy rescale threshold (log2 units)

// QS: Q in shared memory (three score buffers) or in TMEM (two).
template <int KS, int VS, bool QS>
struct TcPlan {
  static constexpr int kNB = QS ? 3 : 2;                  // S / P buffers in TMEM
  static constexpr int kChunkBytes = 64 * 128;           // 64 tokens (or rows) x 128 B
  static constexpr int kTileBytes = 4 * kChunkBytes;      // one K or V tile (or Q), D = 256
  static constexpr int kOffK = 0;                         // K ring: KS tiles
  static constexpr int kOffV = KS * kTileBytes;           // V ring: VS tiles
  static constexpr int kOffQ = (KS + VS) * kTileBytes;    // Q (QS only), 64 rows, K-major, 128-byte swizzle
  static constexpr int kH = QS ? 1 : 2;                  // sixteen-lane groups of a quadrant (M / 64)
  static constexpr int kOffBar = kOffQ + (QS ? kTileBytes : 0);
  // k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[NB], p_full[NB],
  // pv_done[NB], mma_final, q_ready, pair[4 quadrants][2 parities]
  static constexpr int kNumBars = 2 * KS + 2 * VS + 3 * kNB + 2 + 8;
  // values the two softmax warps of a quadrant exchange (row maxima, row
  // sums): [parity][half][quadrant][kH][sub-row][8 row groups] floats
  static constexpr int kOffXch = kOffBar + kNumBars * 8;
  static constexpr int kXchBytes = 2 * 2 * 4 * kH * 2 * 8 * 4;
  static constexpr int kOffMisc = kOffXch + kXchBytes;     // tmem base, abort, split page validity
  static constexpr int kBytes = kOffMisc + 12;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "dynamic shared memory above the 227 KB a CTA may have");
};

// Depths of the K and V rings (64-token tiles).
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

// p0, p1 -> bf16 hi pair and lo pair (p = hi + lo to 2^-16 relative); the
// first value goes to the low half of each word.
__device__ __forceinline__ void split_pack(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  hi = ptx::pack_bf16x2(p0, p1);
  lo = ptx::pack_bf16x2(p0 - ptx::bf16lo_to_f32(hi), p1 - ptx::bf16hi_to_f32(hi));
}

// M: MMA rows (64 or 128); the block's rows must not exceed it.  M = 64
// keeps Q in shared memory and three score buffers, M = 128 Q in TMEM and two.
template <int KS, int VS, int M>
__global__ void __launch_bounds__(kTcThreads, 1)
    verify_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const DecodeArgs a) {
  constexpr bool QS = M == 64;
  using Plan = TcPlan<KS, VS, QS>;
  constexpr int NB = Plan::kNB;
  constexpr uint32_t kColQ = 0;            // TMEM Q (M = 128)
  constexpr uint32_t kColS = QS ? 0 : 128;  // first score buffer
  constexpr int D = 256;
  static_assert(M == 64 || M == 128, "MMA rows: 64 or 128");
  constexpr int H = Plan::kH;  // sixteen-lane groups of a quadrant that hold rows

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t bar0 = sbase + Plan::kOffBar;
  const uint32_t bar_k_full = bar0;
  const uint32_t bar_k_empty = bar_k_full + 8 * KS;
  const uint32_t bar_v_full = bar_k_empty + 8 * KS;
  const uint32_t bar_v_empty = bar_v_full + 8 * VS;
  const uint32_t bar_s_full = bar_v_empty + 8 * VS;  // [NB]
  const uint32_t bar_p_full = bar_s_full + 8 * NB;    // [NB]
  const uint32_t bar_pv_done = bar_p_full + 8 * NB;   // [NB]: PV of the tiles using S/P buffer b
  const uint32_t bar_final = bar_pv_done + 8 * NB;
  const uint32_t bar_q_ready = bar_final + 8;
  const uint32_t bar_pair = bar_q_ready + 8;          // [quadrant][parity]
  volatile int* split_bad = reinterpret_cast<volatile int*>(smem + Plan::kOffMisc + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Plan::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Plan::kOffMisc + 4);

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- set-up: barriers and tensor memory
  // each producer initialises its own ring's barriers, so it can issue its
  // first load before the block-wide barrier below
  if (threadIdx.x == kVWarp * 32) {
    for (int s = 0; s < VS; ++s) {
      ptx::mbar_init(bar_v_full + 8 * s, 1);
      ptx::mbar_init(bar_v_empty + 8 * s, 1);
    }
    ptx::fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < KS; ++s) {
      ptx::mbar_init(bar_k_full + 8 * s, 1);
      ptx::mbar_init(bar_k_empty + 8 * s, 1);
    }
    for (int i = 0; i < NB; ++i) {
      ptx::mbar_init(bar_s_full + 8 * i, 1);
      ptx::mbar_init(bar_p_full + 8 * i, kSmThreads / 32);
      ptx::mbar_init(bar_pv_done + 8 * i, 1);
    }
    ptx::mbar_init(bar_final, 2);  // one commit from each MMA-issuing lane
    ptx::mbar_init(bar_q_ready, kSmThreads / 32);
    for (int i = 0; i < 8; ++i) ptx::mbar_init(bar_pair + 8 * i, 2);  // the two warps of a quadrant
    *abort_flag = 0;
    *split_bad = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  // every global-memory access comes after this: with a programmatic launch
  // the set-up above overlaps the previous kernel's tail
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // ---- Q first: the softmax warps' loads leave before any K/V load of the
  // CTA.  Thread `lane` of softmax warp (q, half) holds head dims
  // 128 half .. 128 half + 127 of row 4 lane + q (zeros for padding rows);
  // every load is issued before the first use.
  const int q = warp & 3;                   // the TMEM lane quadrant of a softmax warp
  const int half = (warp - kSmWarp0) >> 2;  // its column half
  const bool softmax_warp = warp >= kSmWarp0;
  uint4 qv[D / 16];
  if (softmax_warp) {
    const int row = 4 * lane + q;
    const bool q_active = lane < M / 4 && row < a.rows;
    const __nv_bfloat16* src =
        q_active ? a.q + ((static_cast<size_t>(b) * a.num_q + row / a.G) * a.Hq + kvh * a.G + row % a.G) * D +
                       (D / 2) * half
                 : nullptr;
#pragma unroll
    for (int j = 0; j < D / 16; ++j)
      qv[j] = q_active ? *reinterpret_cast<const uint4*>(src + 8 * j) : make_uint4(0, 0, 0, 0);
  }
  // the page-table entries of this split's first tiles, guessed from the
  // cache's capacity (exact when the sequence fills it), head for L2 while
  // kv_len is read
  if (warp == 0 && lane < KS) {
    const int nt_cap = (a.max_pages * a.page_size + kTileTokens - 1) / kTileTokens;
    const int t = split * ((nt_cap + a.nsplit - 1) / a.nsplit) + lane;
    if (t < nt_cap)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a.page_table + static_cast<size_t>(b) * a.max_pages +
                                                        (t * kTileTokens) / a.page_size));
  }
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
  // Blocks of up to 32 rows fill only the sub-row j = 0 lanes of an M = 64
  // MMA (rows 16 (r % 4) + r / 4 < 8 of each quadrant's sixteen).  P_lo of a
  // row then sits in the row's spare lane (+8), so P_hi and P_lo go through
  // one MMA per 16 tokens, and O's spare-lane rows hold the P_lo products,
  // which the epilogue adds to their row.
  const bool stacked = QS && a.rows <= 32;

  // ---- producers: warp 0 loads K tiles, warp 3 V tiles (lane 0 each), each
  // into its own ring.  Tile k of a ring goes to stage k % depth.
  const bool is_k = warp == 0;
  const CUtensorMap* tmap = is_k ? &tmap_k : &tmap_v;
  const uint32_t bar_full = is_k ? bar_k_full : bar_v_full;
  const uint32_t bar_empty = is_k ? bar_k_empty : bar_v_empty;
  const int nst = is_k ? KS : VS;  // stages of this lane's ring
  const int box_rows = min(a.page_size, kTileTokens);
  const int boxes = kTileTokens / box_rows;
  // the page-table entries of tile k (boxes of them; -1 past the sequence),
  // read one tile ahead of their use so the round trip overlaps the wait for
  // a free stage
  auto pages_of = [&](int k, int (&pg)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tok = (t_begin + k) * kTileTokens + j * box_rows;
      pg[j] = (k < my_tiles && j < boxes && tok < n_tok)
                  ? a.page_table[static_cast<size_t>(b) * a.max_pages + tok / a.page_size]
                  : -1;
    }
  };
  auto produce = [&](int k, const int (&pg)[4], uint64_t pol) {
    const int tok0 = (t_begin + k) * kTileTokens;
    const int oob_z = a.num_pages * a.Hkv;  // past the tensor: zero fill
    const uint32_t dst = sbase + (is_k ? Plan::kOffK : Plan::kOffV) + (k % nst) * Plan::kTileBytes;
    const uint32_t fb = bar_full + 8 * (k % nst);
    int zs[4], ys[4];
    int valid = 1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tok = tok0 + j * box_rows;
      zs[j] = oob_z;
      ys[j] = 0;
      if (j >= boxes || tok >= n_tok) continue;
      if (pg[j] < 0 || pg[j] >= a.num_pages) {
        valid = 0;
      } else {
        zs[j] = pg[j] * a.Hkv + kvh;
        ys[j] = tok % a.page_size;
      }
    }
    if (is_k && !valid) set_status(a.status, kDevPageOob);
    ptx::mbar_arrive_expect_tx(fb, Plan::kTileBytes);
    for (int j = 0; j < boxes; ++j) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        ptx::tma_load_3d(dst + c * Plan::kChunkBytes + j * box_rows * 128, tmap, fb, c * 64, ys[j], zs[j], pol);
    }
  };
  // The fused append: the new rows (positions n_tok - num_q .. n_tok - 1)
  // that fall in this CTA's tiles go into the pools before any of its tiles
  // is loaded -- K by warp 0, V by warp 3, all lanes, every load of a lane
  // before its stores.  Each lane orders its stores before the async proxy,
  // then the warp converges before lane 0 issues a bulk copy.  Only the CTA
  // that loads a tile reads its new rows.  A row on a page outside the pool
  // is skipped (the tile's loads raise WMTP_DEV_PAGE_OOB).
  if (a.k_new != nullptr && (warp == 0 || warp == kVWarp) && my_tiles > 0) {
    const int new_lo = n_tok - a.num_q;
    const int lo = max(new_lo, t_begin * kTileTokens), hi = min(n_tok, t_end * kTileTokens);
    if (lo < hi) {
      constexpr int kUnits = D / 8;  // 16-byte units of a row
      const uint4* src = reinterpret_cast<const uint4*>(is_k ? a.k_new : a.v_new);
      uint4* pool = reinterpret_cast<uint4*>(is_k ? a.k_pool_w : a.v_pool_w);
      const int n_units = (hi - lo) * kUnits;
      // four units a lane per round: every load of the round before its stores
      for (int u0 = 0; u0 < n_units; u0 += 4 * 32) {
        uint4 val[4];
        size_t dst[4];
        bool ok[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int u = u0 + i * 32 + lane;
          ok[i] = u < n_units;
          if (!ok[i]) continue;
          const int pos = lo + u / kUnits, c = u % kUnits;
          const int pg = a.page_table[static_cast<size_t>(b) * a.max_pages + pos / a.page_size];
          ok[i] = pg >= 0 && pg < a.num_pages;
          dst[i] = ((static_cast<size_t>(pg) * a.Hkv + kvh) * a.page_size + pos % a.page_size) * kUnits + c;
          val[i] = src[((static_cast<size_t>(b) * a.num_q + (pos - new_lo)) * a.Hkv + kvh) * kUnits + c];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (ok[i]) pool[dst[i]] = val[i];
      }
      ptx::fence_proxy_async_global();
    }
    __syncwarp();
  }
  // tile 0 of each ring goes out before the block-wide barrier (the
  // producers initialised their own barriers), and the page-table lines of
  // the next tiles head for L2
  int issued_pre = 0;
  if ((warp == 0 || warp == kVWarp) && lane == 0 && my_tiles > 0) {
    ptx::prefetch_tmap(tmap);
    int pg0[4];
    pages_of(0, pg0);
    produce(0, pg0, ptx::policy_evict_first());
    issued_pre = 1;
  }
  if (warp == 0 && lane >= 1 && lane <= VS && lane < my_tiles) {
    const int* pte = a.page_table + static_cast<size_t>(b) * a.max_pages +
                     ((t_begin + lane) * kTileTokens) / a.page_size;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(pte));
  }
  // Q of M = 64 goes to shared memory now (K-major with the 128-byte swizzle
  // the K tiles have: chunk c (head dims 64 c .. 64 c + 63) of MMA row m at
  // c * 8 KB + 128 m, 16-byte unit u at position u ^ (m % 8))
  if constexpr (QS) {
    if (softmax_warp && lane < 16) {
      const int m = 16 * q + lane;
#pragma unroll
      for (int jj = 0; jj < D / 16; ++jj) {
        const int j = (D / 16) * half + jj;  // 16-byte unit of the row
        const uint32_t dst = sbase + Plan::kOffQ + (j >> 3) * Plan::kChunkBytes + m * 128 + (((j & 7) ^ (m & 7)) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(qv[jj].x), "r"(qv[jj].y),
                     "r"(qv[jj].z), "r"(qv[jj].w)
                     : "memory");
      }
    }
    if (softmax_warp) ptx::fence_proxy_async_smem();  // generic writes before the tensor core reads
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // =================================================================== producers
  if (warp == 0 || warp == kVWarp) {
    if (lane == 0 && my_tiles > 0) {
      const uint64_t pol = ptx::policy_evict_first();
      int issued = issued_pre;
      int pg_cur[4], pg_nxt[4];
      pages_of(issued, pg_cur);
      for (int k = issued; k < my_tiles; ++k) {
        // entries four tiles ahead head for L2; the next tile's are read now
        const int ahead = (t_begin + k + 4) * kTileTokens;
        if (k + 4 < my_tiles && ahead < n_tok)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.page_table + static_cast<size_t>(b) * a.max_pages +
                                                            ahead / a.page_size));
        pages_of(k + 1, pg_nxt);
        if (!tc_wait(bar_empty + 8 * (k % nst), ((k / nst) & 1) ^ 1, abort_flag)) {
          if (*abort_flag == 0) set_status(a.status, kDevTimeout);
          *abort_flag = 1;
          break;
        }
        produce(k, pg_cur, pol);
        issued = k + 1;
#pragma unroll
        for (int j = 0; j < 4; ++j) pg_cur[j] = pg_nxt[j];
      }
      // no copy may still be writing shared memory when the CTA exits (after
      // an abort the consumers stop early): wait, bounded, for the last load
      // of each stage
      for (int k = max(issued - nst, 0); k < issued; ++k)
        if (!ptx::mbar_wait(bar_full + 8 * (k % nst), (k / nst) & 1)) set_status(a.status, kDevTimeout);
    }
    return;
  }

  // =================================================================== PV issuer
  // O += P(k) V(k) for every tile, issued by its own lane: a single lane
  // issues a small tcgen05.mma only every ~66 cycles, so the QK and PV
  // streams run from two lanes and overlap in the tensor pipe.  Per 16
  // tokens two MMAs, P_hi V and P_lo V, or one for a stacked block (P_hi and
  // P_lo in the same columns, different lanes).  The first MMA of a run
  // starts a fresh accumulation (the softmax threads have folded the
  // previous run).
  if (warp == kPvWarp) {
    if (lane == 0 && my_tiles > 0) {
      constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(M, 256, 0, 1);    // A (P, TMEM), B (V) MN-major
      const uint64_t v_desc0 = tc::smem_desc_sw128(sbase + Plan::kOffV, Plan::kChunkBytes, 1024);
      bool ok = true;
      for (int k = 0; ok && k < my_tiles; ++k) {
        ok = tc_wait(bar_p_full + 8 * (k % NB), (k / NB) & 1, abort_flag) &&
             tc_wait(bar_v_full + 8 * (k % VS), (k / VS) & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        const uint64_t vd = v_desc0 + (static_cast<uint64_t>((k % VS) * Plan::kTileBytes) >> 4);
        const uint32_t p_tmem = tmem_base + kColS + (k % NB) * 64;
        const uint32_t fresh = (k % kRunTiles) == 0 ? 0u : 1u;  // 0: overwrite O
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          // 16 tokens = 8 columns of bf16 pairs; V rows 16 kk .. 16 kk + 15
          const uint64_t bd = vd + (static_cast<uint32_t>(kk * 2048) >> 4);
          tc::mma_ts(tmem_base + kColO, p_tmem + 8 * kk, bd, kIdescPV, kk > 0 ? 1u : fresh);
          if (!stacked) tc::mma_ts(tmem_base + kColO, p_tmem + 32 + 8 * kk, bd, kIdescPV, 1u);
        }
        tc::commit(bar_v_empty + 8 * (k % VS));
        tc::commit(bar_pv_done + 8 * (k % NB));
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
      constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(M, 64, 0, 0);     // A (Q), B (K) K-major
      // descriptor start addresses are in 16-byte units in the low bits, so
      // moving an operand by n bytes adds n >> 4 to the descriptor
      const uint64_t k_desc0 = tc::smem_desc_sw128(sbase + Plan::kOffK, 16, 1024);
      const uint64_t q_desc0 = tc::smem_desc_sw128(sbase + Plan::kOffQ, 16, 1024);  // QS only
      // Q is staged into TMEM by the softmax warps while the first K/V tiles
      // are in flight
      bool ok = tc_wait(bar_q_ready, 0, abort_flag);
      for (int k = 0; ok && k < my_tiles; ++k) {
        // S/P buffer k % NB last held P(k-NB): PV(k-NB), issued by the other
        // lane, must have completed (its phase of pv_done; the next phase
        // needs P(k), which needs this S)
        if (k >= NB && !(ok = tc_wait(bar_pv_done + 8 * (k % NB), ((k - NB) / NB) & 1, abort_flag))) break;
        if (!(ok = tc_wait(bar_k_full + 8 * (k % KS), (k / KS) & 1, abort_flag))) break;
        tc::fence_after_sync();
        const uint64_t kd = k_desc0 + (static_cast<uint64_t>((k % KS) * Plan::kTileBytes) >> 4);
        const uint32_t d_tmem = tmem_base + kColS + (k % NB) * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * Plan::kChunkBytes + (kk & 3) * 32;
          if constexpr (QS)
            tc::mma_ss(d_tmem, q_desc0 + (ka >> 4), kd + (ka >> 4), kIdescQK, kk > 0 ? 1u : 0u);
          else
            tc::mma_ts(d_tmem, tmem_base + kColQ + 8 * kk, kd + (ka >> 4), kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc::commit(bar_s_full + 8 * (k % NB));
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
    // Warps (q, 0) and (q, 1) share the rows of lane quadrant q; half `half`
    // takes tile columns 32 half .. 32 half + 31 and O columns
    // 128 half .. 128 half + 127.
    const uint32_t qlane = static_cast<uint32_t>(32 * q) << 16;
    {
      // Q of M = 128 goes into TMEM lane 32 q + lane, columns
      // 64 half .. 64 half + 63 (bf16 pairs of this half's head dims); Q of
      // M = 64 is already in shared memory
      if constexpr (!QS) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t wq[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            wq[4 * j] = qv[8 * cc + j].x;
            wq[4 * j + 1] = qv[8 * cc + j].y;
            wq[4 * j + 2] = qv[8 * cc + j].z;
            wq[4 * j + 3] = qv[8 * cc + j].w;
          }
          tc::tmem_st32(tmem_base + qlane + kColQ + 64 * half + 32 * cc, wq);
        }
        tc::fence_before_sync();
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_q_ready);
    }

    // Sixteen-lane view: in group h this thread covers TMEM lanes
    // 16 h + lane / 4 (sub-row j = 0) and 16 h + lane / 4 + 8 (j = 1) of the
    // quadrant, and of this half's 32 columns of a tile columns
    // 32 half + 8 r + 2 (lane % 4) + {0, 1} (r = 0..3).  The four threads
    // lane / 4 * 4 + {0..3} share both rows.
    const int cq = 2 * (lane & 3);
    int row_of[H][2];
    bool act[H][2];    // this thread's row exists
    bool any_r[H][2];  // some row of this warp's (group, sub-row) exists (warp-uniform)
    int lim[H][2];     // causal limit (exclusive)
    const int q_first = a.q_pos0 != nullptr ? a.q_pos0[b] : n_tok - a.num_q;
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int ln = 16 * h + 8 * j + (lane >> 2);  // lane inside the quadrant
        row_of[h][j] = 4 * ln + q;
        act[h][j] = row_of[h][j] < a.rows;
        any_r[h][j] = 4 * (16 * h + 8 * j) + q < a.rows;
        lim[h][j] = act[h][j] ? min(n_tok, q_first + row_of[h][j] / a.G + 1) : n_tok;
      }
    const int first_masked_tok = min(n_tok, q_first + 1);

    float m_ref[H][2], l_run[H][2], m_g[H][2];
    bool have_g[H][2];
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m_ref[h][j] = -INFINITY;
        l_run[h][j] = 0.f;  // this thread's share (8 of this half's 32 columns of every tile)
        m_g[h][j] = -INFINITY;
        have_g[h][j] = false;
      }
    bool failed = false;

    // the split's partial slot of one of this thread's rows
    auto dst_of = [&](int h, int j) -> float* {
      const int r = row_of[h][j];
      const size_t grow = (static_cast<size_t>(b) * a.num_q + r / a.G) * a.Hq + kvh * a.G + r % a.G;
      return a.part_o + (grow * a.nsplit + split) * D;
    };
    // O columns 64 cb .. 64 cb + 63 of group h; this half owns cb = 2 half, 2 half + 1
    auto o_addr = [&](int h, int cb) -> uint32_t {
      return tmem_base + qlane + (static_cast<uint32_t>(16 * h) << 16) + kColO + 64 * cb;
    };
    auto s_addr_of = [&](int h, int sb) -> uint32_t {
      return tmem_base + qlane + (static_cast<uint32_t>(16 * h) << 16) + kColS + sb * 64;
    };
    // Exchange with the other half of the quadrant.  Step s (tile s, or
    // my_tiles for the row sums at the end) writes slots of parity s & 1 and
    // completes a phase of pair barrier (q, s & 1); a warp reaches step s + 2
    // only after its partner has arrived at step s + 1, so by then the
    // partner has read the slots of step s.
    float* xch = reinterpret_cast<float*>(smem + Plan::kOffXch);
    auto xslot = [&](int s, int hf, int h, int j) -> float* {
      return xch + (((((s & 1) * 2 + hf) * 4 + q) * H + h) * 2 + j) * 8 + (lane >> 2);
    };
    auto pair_sync = [&](int s) -> bool {
      const uint32_t bar = bar_pair + 8 * (2 * q + (s & 1));
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar);
      const bool ok = __all_sync(0xffffffffu, tc_wait(bar, (s >> 1) & 1, abort_flag));
      tc::fence_after_sync();
      return ok;
    };

    // Page validity, once for the whole split: a tile with a page outside the
    // pool is skipped (the producers load zeros for it and raise
    // WMTP_DEV_PAGE_OOB).  In the common case every entry is valid and no tile
    // needs a check; otherwise the tiles read their entries as they go.
    {
      const int box_rows = min(a.page_size, kTileTokens);
      const int first = t_begin * kTileTokens, last = min(t_end * kTileTokens, n_tok);
      bool ok = true;
      for (int tok = first + (threadIdx.x - kSmWarp0 * 32) * box_rows; tok < last; tok += kSmThreads * box_rows) {
        const int pg = a.page_table[static_cast<size_t>(b) * a.max_pages + tok / a.page_size];
        ok = ok && pg >= 0 && pg < a.num_pages;
      }
      if (!__all_sync(0xffffffffu, ok) && lane == 0) *split_bad = 1;
      ptx::named_bar_sync(kBarSoftmax, kSmThreads);
    }
    const bool split_ok = *split_bad == 0;

    for (int k = 0; k < my_tiles && !failed; ++k) {
      const int sb = k % NB;
      // S(k) complete implies K(k) landed.  (The K ring itself is not waited
      // on here: its stage may already hold a later tile, so a parity wait on
      // it would be ambiguous.)
      if (!__all_sync(0xffffffffu, tc_wait(bar_s_full + 8 * sb, (k / NB) & 1, abort_flag))) {
        failed = true;
        break;  // this warp stops; the MMA warps time out or see the abort
      }
      tc::fence_after_sync();
      const int tok0 = (t_begin + k) * kTileTokens;
      const bool run_start = k > 0 && (k % kRunTiles) == 0;
      bool o_ready = false;  // PV(k-1) known complete
      if (run_start) {
        // fold the finished run into the split's fp32 partial, in units of
        // the current reference: G = G 2^(m_g - m_ref) + O; PV(k) then starts
        // a fresh accumulation.  PV(k-1) completes the pv_done phase of its
        // buffer; the buffer's next phase needs P(k-1+NB), so the wait is
        // unambiguous.  Each half folds its own O columns.
        if (!__all_sync(0xffffffffu, tc_wait(bar_pv_done + 8 * ((k - 1) % NB), ((k - 1) / NB) & 1, abort_flag))) {
          failed = true;
          break;
        }
        tc::fence_after_sync();
        o_ready = true;
#pragma unroll
        for (int h = 0; h < H; ++h) {
          if (!(any_r[h][0] || any_r[h][1])) continue;
          float gs[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) gs[j] = have_g[h][j] ? ptx::ex2(m_g[h][j] - m_ref[h][j]) : 0.f;
#pragma unroll 1
          for (int cb = 2 * half; cb < 2 * half + 2; ++cb) {
            uint32_t o[32];
            tc::tmem_ld_16x256b_x8(o_addr(h, cb), o);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              if (!act[h][j] || m_ref[h][j] == -INFINITY) continue;
              float* d = dst_of(h, j) + 64 * cb + cq;
#pragma unroll
              for (int r = 0; r < 8; ++r) {
                float2* g = reinterpret_cast<float2*>(d + 8 * r);
                const float2 old = have_g[h][j] ? *g : make_float2(0.f, 0.f);
                float o0 = __uint_as_float(o[4 * r + 2 * j]), o1 = __uint_as_float(o[4 * r + 2 * j + 1]);
                if (stacked) {  // j = 0: add the spare lane's P_lo products
                  o0 += __uint_as_float(o[4 * r + 2]);
                  o1 += __uint_as_float(o[4 * r + 3]);
                }
                *g = make_float2(old.x * gs[j] + o0, old.y * gs[j] + o1);
              }
            }
          }
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (m_ref[h][j] != -INFINITY) {
              m_g[h][j] = m_ref[h][j];
              have_g[h][j] = true;
            }
        }
      }
      bool tile_ok = true;
      if (!split_ok) {
        for (int tok = tok0; tok < min(tok0 + kTileTokens, n_tok); tok += min(a.page_size, kTileTokens)) {
          const int pg = a.page_table[static_cast<size_t>(b) * a.max_pages + tok / a.page_size];
          tile_ok = tile_ok && pg >= 0 && pg < a.num_pages;
        }
      }
      const bool masked_tile = tok0 + kTileTokens > first_masked_tok || !tile_ok;
      // V rows past the end of the sequence hold stale pool bytes: zero them
      // before PV reads the tile, so their 0 weights add exactly 0
      if (tok0 + kTileTokens > n_tok) {
        const int stage = k % VS;
        if (!__all_sync(0xffffffffu, tc_wait(bar_v_full + 8 * stage, (k / VS) & 1, abort_flag))) {
          failed = true;
          break;
        }
        const int r0 = max(n_tok - tok0, 0);
        const uint32_t vt = sbase + Plan::kOffV + stage * Plan::kTileBytes;
        // 16-byte unit c (0..31) of token row r: chunk c / 8, unit c % 8 (a
        // whole row is zeroed, so the swizzle does not matter)
        for (int u = threadIdx.x - kSmWarp0 * 32; u < (kTileTokens - r0) * 32; u += kSmThreads) {
          const int r = r0 + u / 32, c = u % 32;
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vt + (c >> 3) * Plan::kChunkBytes +
                                                                       r * 128 + ((c & 7) << 4)),
                       "r"(0)
                       : "memory");
        }
        ptx::fence_proxy_async_smem();
      }

      // this half's scores, scaled to log2 units (masked entries -inf), and
      // their row maxima
      float x[H][2][8];
      float mx[H][2];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        mx[h][0] = mx[h][1] = -INFINITY;
        if (!(any_r[h][0] || any_r[h][1])) continue;
        uint32_t sraw[16];
        tc::tmem_ld_16x256b_x4(s_addr_of(h, sb) + 32 * half, sraw);
        // sub-row groups without any row are skipped (warp-uniform); a tile
        // without masked positions takes the short path
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (!any_r[h][j]) continue;
          if (!masked_tile) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                x[h][j][2 * r + e] = __uint_as_float(sraw[4 * r + 2 * j + e]) * a.scale_log2;
          } else {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int t = tok0 + 32 * half + 8 * r + cq + e;
                const float s = __uint_as_float(sraw[4 * r + 2 * j + e]) * a.scale_log2;
                x[h][j][2 * r + e] = (tile_ok && t < lim[h][j] && t < n_tok) ? s : -INFINITY;
              }
          }
          // pairwise maximum (a tree keeps the dependent chain short)
          float t4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) t4[i] = fmaxf(x[h][j][2 * i], x[h][j][2 * i + 1]);
          float m = fmaxf(fmaxf(t4[0], t4[2]), fmaxf(t4[1], t4[3]));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
          mx[h][j] = m;
        }
      }
      // the other half's maxima (both halves then hold the tile maximum of
      // every row and take the same decisions below).  The S columns this
      // warp reads are the P columns its partner writes: both loads complete
      // before the exchange, both stores come after it.
      if ((lane & 3) == 0) {
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (any_r[h][j]) *xslot(k, half, h, j) = mx[h][j];
      }
      if (!pair_sync(k)) {
        failed = true;
        break;
      }
#pragma unroll
      for (int h = 0; h < H; ++h)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          if (any_r[h][j]) mx[h][j] = fmaxf(mx[h][j], *xslot(k, half ^ 1, h, j));

#pragma unroll
      for (int h = 0; h < H; ++h) {
        uint32_t ph[8], pl[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) ph[i] = pl[i] = 0u;
        if (any_r[h][0] || any_r[h][1]) {
          // raise the reference maximum only when the tile exceeds it by more
          // than 2^8; rows whose reference moved rescale their O row and sum
          float alpha[2] = {1.f, 1.f};
          bool moved = false;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (mx[h][j] > m_ref[h][j] + kRescaleLog2 || (m_ref[h][j] == -INFINITY && mx[h][j] != -INFINITY)) {
              alpha[j] = (m_ref[h][j] == -INFINITY) ? 0.f : ptx::ex2(m_ref[h][j] - mx[h][j]);
              moved = moved || m_ref[h][j] != -INFINITY;
              m_ref[h][j] = mx[h][j];
            }
            l_run[h][j] *= alpha[j];
          }
          // a new run starts from an empty accumulator: nothing to rescale
          if (!run_start && __any_sync(0xffffffffu, moved)) {
            // PV(k-1) must have finished before O is rewritten (the pv_done
            // phase of its buffer, as for the fold above)
            if (!o_ready) {
              if (!__all_sync(0xffffffffu, tc_wait(bar_pv_done + 8 * ((k - 1) % NB), ((k - 1) / NB) & 1,
                                                   abort_flag))) {
                failed = true;
                break;
              }
              tc::fence_after_sync();
              o_ready = true;
            }
#pragma unroll 1
            for (int cb = 2 * half; cb < 2 * half + 2; ++cb) {
              uint32_t o[32];
              tc::tmem_ld_16x256b_x8(o_addr(h, cb), o);
#pragma unroll
              for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                  for (int e = 0; e < 2; ++e)
                    o[4 * r + 2 * j + e] =
                        __float_as_uint(__uint_as_float(o[4 * r + 2 * j + e]) * (stacked ? alpha[0] : alpha[j]));
              tc::tmem_st_16x256b_x8(o_addr(h, cb), o);
            }
          }
          // P = 2^(x - m_ref) as bf16 hi + lo pairs: token pair
          // 16 half + 4 r + lane % 4 of the tile, back into the S columns
          // (P_hi in columns 0..31, P_lo in 32..63; in a stacked block P_lo
          // in the row's spare lane, columns 0..31)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (!any_r[h][j]) continue;
            const float base = (m_ref[h][j] == -INFINITY) ? 0.f : m_ref[h][j];
            float ps[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const float p0 = ptx::ex2(x[h][j][2 * r] - base);  // 2^-inf = 0 for masked entries
              const float p1 = ptx::ex2(x[h][j][2 * r + 1] - base);
              ps[r] = p0 + p1;
              split_pack(p0, p1, ph[2 * r + j], pl[2 * r + j]);
            }
            l_run[h][j] += (ps[0] + ps[2]) + (ps[1] + ps[3]);
          }
        }
        const uint32_t s_addr = s_addr_of(h, sb);
        if (stacked) {
          // P_hi in the row's lane, P_lo in its spare lane, same columns
          uint32_t pk[8];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            pk[2 * r] = ph[2 * r];
            pk[2 * r + 1] = pl[2 * r];
          }
          tc::tmem_st_16x128b_x4(s_addr + 16 * half, pk);
        } else {
          tc::tmem_st_16x128b_x4_pair(s_addr + 16 * half, ph, s_addr + 32 + 16 * half, pl);
        }
      }
      if (failed) break;

      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_p_full + 8 * sb);
    }

    // ---- finish: normalised partial output and log-sum-exp of each row
    if (!failed && my_tiles > 0) {
      // mma_final completes once, when every MMA of the CTA has completed
      if (!__all_sync(0xffffffffu, tc_wait(bar_final, 0, abort_flag))) failed = true;
      tc::fence_after_sync();
    }
    // the row sums: the four threads of a row hold a quarter of this half's
    // share, the other half's warp the rest
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float l = l_run[h][j];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        l_run[h][j] = l;
      }
    if (!failed) {
      if ((lane & 3) == 0) {
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (any_r[h][j]) *xslot(my_tiles, half, h, j) = l_run[h][j];
      }
      if (!pair_sync(my_tiles)) {
        failed = true;
      } else {
#pragma unroll
        for (int h = 0; h < H; ++h)
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (any_r[h][j]) l_run[h][j] += *xslot(my_tiles, half ^ 1, h, j);
      }
    }
    failed = __any_sync(0xffffffffu, failed || *abort_flag != 0);
    if (failed) {
      if (lane == 0) set_status(a.status, kDevTimeout);
      *abort_flag = 1;
    }
#pragma unroll
    for (int h = 0; h < H; ++h) {
      float inv[2], gs[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        inv[j] = (l_run[h][j] > 0.f && !failed) ? 1.f / l_run[h][j] : 0.f;
        gs[j] = (have_g[h][j] && !failed) ? ptx::ex2(m_g[h][j] - m_ref[h][j]) : 0.f;
      }
      if (!(any_r[h][0] || any_r[h][1])) continue;
#pragma unroll 1
      for (int cb = 2 * half; cb < 2 * half + 2; ++cb) {
        uint32_t o[32];
        if (my_tiles > 0 && !failed) {
          tc::tmem_ld_16x256b_x8(o_addr(h, cb), o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (!act[h][j]) continue;
          float* d = dst_of(h, j) + 64 * cb + cq;
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            float2* g = reinterpret_cast<float2*>(d + 8 * r);
            const float2 old = (have_g[h][j] && !failed) ? *g : make_float2(0.f, 0.f);
            float o0 = __uint_as_float(o[4 * r + 2 * j]), o1 = __uint_as_float(o[4 * r + 2 * j + 1]);
            if (stacked) {  // j = 0: add the spare lane's P_lo products
              o0 += __uint_as_float(o[4 * r + 2]);
              o1 += __uint_as_float(o[4 * r + 3]);
            }
            *g = make_float2((old.x * gs[j] + o0) * inv[j], (old.y * gs[j] + o1) * inv[j]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (half == 0 && act[h][j] && (lane & 3) == 0) {
          const int r = row_of[h][j];
          const size_t grow = (static_cast<size_t>(b) * a.num_q + r / a.G) * a.Hq + kvh * a.G + r % a.G;
          // m_ref is in log2 units of the scaled score
          a.part_lse[grow * a.nsplit + split] = (l_run[h][j] > 0.f && !failed)
                                                    ? m_ref[h][j] * 0.69314718055994531f + logf(l_run[h][j])
                                                    : -INFINITY;
        }
      }
    }
    tc::fence_before_sync();
  }

  // ---- every MMA has completed (the MMA lanes waited for their final
  // commit); free the tensor memory
  ptx::named_bar_sync(kBarTmem, 32 + kSmThreads);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace wmtp

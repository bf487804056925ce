// Split-KV decode attention for Windowed-MTP draft and verify steps (sm_100a).
//
// One kernel template serves the attention calls of a decode step:
//   * native draft  : 1 query x G heads over the draft layer's paged cache
//                     ("Windowed-MTP ..." arxivlens view, Abstract: the draft
//                     head reads the full KV cache in each draft forward);
//   * windowed draft: the same query over the compact sink + window ring
//                     (same Abstract; readpriors post, What happened), or
//                     over the sink + window positions of the paged cache
//                     (paged_window: only the tiles holding those positions
//                     are loaded);
//   * verify        : gamma+1 causal queries x G heads over a target layer's
//                     paged cache (same Abstract: verification stays
//                     full-context) for blocks outside the tcgen05 verify
//                     kernel's range (head_dim 64, or 8 or fewer rows); with
//                     q_pos0 the cache may hold a slice of a longer context.
//
// Work decomposition: CTA = (split, kv head, sequence).  All query rows that
// share the KV head (rows = num_q * G, padded to NT*8) are processed together,
// so each K/V byte is read from HBM once per call.
//
// Warp roles (5 warps): warps 0-3 compute, warp 4 is the TMA producer.  The
// producer streams 64-token tiles of K and V (64 x D bf16 each) into a ring of
// STAGES shared-memory stages with 3-D tiled TMA loads (128-byte swizzle),
// completing on per-stage "full" mbarriers; compute warps release a stage on
// its "empty" mbarrier.
//
// Per 64-token tile, the compute warps:
//   1. S^T = K Q^T on tensor cores (mma.sync m16n8k16, bf16 in, fp32 out):
//      warp w takes tokens 16w..16w+15 against every query row;
//   2. share per-row tile maxima through shared memory (named barrier), then
//      p = 2^(s*scale*log2e - m), rescale running sums and outputs;
//   3. write P as two bf16 terms (p = hi + lo, |p - hi - lo| <= 2^-16 p) so
//      the PV product keeps ~fp32 weight precision, named barrier;
//   4. O^T += V^T P^T on tensor cores, warp w owning head-dim columns
//      [w*D/4, (w+1)*D/4).
// At the end each CTA writes its split's fp32 partial output and log-sum-exp;
// a combine kernel merges the splits.  The kernel is launched as a
// programmatic dependent: barrier set-up runs before griddepcontrol.wait,
// every global-memory access after it.
//
// Masking is by selection (score := -inf), never by multiplication, and V rows
// past the valid length are zeroed in shared memory, so stale or non-finite
// bytes beyond a sequence never reach the output.
//
// Accumulation runs: a tensor-core MMA adds its products to the fp32
// accumulator at the accumulator's precision, so products far smaller than
// the running sum lose low-order bits.  Over a long split of nearly equal
// weights and values of one sign that loss is systematic (~n 2^-25 of the
// result after n tokens).  Every kRunTiles tiles the accumulator is therefore
// folded into the split's fp32 partial in global memory with exact fp32 adds
// and restarted, so one accumulation spans at most 16,384 tokens.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace wmtp {

constexpr int kTileTokens = 64;
constexpr int kComputeWarps = 4;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kThreads = 32 * (kComputeWarps + 1);
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kPPitchBytes = 144;  // one P row: 64 bf16 + 16 bytes of padding
constexpr int kBarCompute = 1;     // named barrier id of the compute warps
constexpr int kRunTiles = 256;     // tiles per accumulation run (16,384 tokens)

// Status bits (mirror include/wmtp.h).
constexpr int kDevPageOob = 0x1;
constexpr int kDevLenOob = 0x2;
constexpr int kDevRingState = 0x4;
constexpr int kDevUndoFull = 0x8;
constexpr int kDevTimeout = 0x10;

struct DecodeArgs {
  const __nv_bfloat16* q;  // [B][num_q][Hq][D]
  int num_q, Hq, Hkv, G, rows;
  // paged source
  const int32_t* page_table;  // [B][max_pages]
  const int32_t* kv_len;      // [B]
  int max_pages, num_pages, page_size;
  // ring source
  const int32_t* ring_tags;  // [B][R]
  const int32_t* ring_len;   // [B]
  int ring_slots, sinks, window;
  // paged source only: 1 = attend the sink + window positions of the pages
  // (the windowed draft read through the page table), 0 = every position
  int paged_window;
  // paged source only: [B] position of query 0 counted from this cache's first
  // token (a slice of a longer sequence), or NULL for kv_len - num_q
  const int32_t* q_pos0;
  // outputs
  float* part_o;    // [B*num_q*Hq][nsplit][D]
  float* part_lse;  // [B*num_q*Hq][nsplit]
  int nsplit;
  float scale_log2;  // sm_scale * log2(e)
  int32_t* status;
  // tcgen05 verify only, or NULL: the num_q new tokens' K/V ([B][num_q][Hkv][D]
  // bf16), written into the pools (k_pool_w, v_pool_w: [num_pages][Hkv][P][D])
  // at positions kv_len - num_q .. kv_len - 1 before their tiles are loaded
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pool_w;
  __nv_bfloat16* v_pool_w;
};

__device__ __forceinline__ void set_status(int32_t* status, int bits) {
  if (status != nullptr) atomicOr(status, bits);
}

// ---------------------------------------------------------------- smem plan
template <int D, int NT, int STAGES>
struct SmemPlan {
  static constexpr int kRows = NT * 8;
  static constexpr int kChunks = D / 64;            // 128-byte-wide column chunks
  static constexpr int kChunkBytes = kTileTokens * 128;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQChunkBytes = kRows * 128;
  static constexpr int kQBytes = kChunks * kQChunkBytes;
  static constexpr int kPBytes = 2 * kRows * kPPitchBytes;  // hi and lo
  static constexpr int kRedBytes = kComputeWarps * kRows * 4 + 16 * 4;
  static constexpr int kOffK = 0;
  static constexpr int kOffQ = STAGES * kStageBytes;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffRed = kOffP + kPBytes;
  static constexpr int kOffBar = (kOffRed + kRedBytes + 7) / 8 * 8;
  static constexpr int kOffFlags = kOffBar + 2 * STAGES * 8;
  static constexpr int kBytes = kOffFlags + STAGES * 4;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1 KB
};

constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block on sm_100

template <int D, int NT>
constexpr int pick_stages() {
  return (SmemPlan<D, NT, 6>::kAlloc <= kSmemLimit && D == 64)  ? 6
         : (SmemPlan<D, NT, 3>::kAlloc <= kSmemLimit)            ? 3
                                                                 : 2;
}

// Swizzled byte offset of 16-byte unit `unit` (0..7) of row `row` inside a
// 128-byte-wide chunk; matches the TMA 128B swizzle for 1 KB-aligned chunks.
__device__ __forceinline__ uint32_t swz(int row, int unit) {
  return static_cast<uint32_t>(row * 128 + ((unit ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------- kernel
template <int D, int NT, int STAGES, bool RING>
__global__ void __launch_bounds__(kThreads, 1)
    decode_attn_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const DecodeArgs a) {
  using Plan = SmemPlan<D, NT, STAGES>;
  constexpr int kRows = Plan::kRows;
  constexpr int kMT = D / 64;  // 16-column m-tiles of O^T per compute warp
  static_assert(D == 64 || D == 256, "head_dim must be 64 or 256");
  static_assert(NT >= 1 && NT <= 8, "rows must be 1..64");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t s_q = sbase + Plan::kOffQ;
  const uint32_t s_p = sbase + Plan::kOffP;
  float* red = reinterpret_cast<float*>(smem + Plan::kOffRed);
  int* abort_flag = reinterpret_cast<int*>(smem + Plan::kOffRed + kComputeWarps * kRows * 4);
  const uint32_t bar_full = sbase + Plan::kOffBar;
  const uint32_t bar_empty = bar_full + STAGES * 8;
  volatile int* stage_flag = reinterpret_cast<volatile int*>(smem + Plan::kOffFlags);

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // barriers first: with a programmatic launch this overlaps the previous
  // kernel's tail; every global-memory access comes after griddepcontrol.wait
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(bar_full + 8 * s, 1);
      ptx::mbar_init(bar_empty + 8 * s, kComputeWarps);
    }
    ptx::fence_mbar_init();
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // ---- the token range of this split (uniform across the CTA)
  int n_tok = 0;
  int seq_len = 0;
  if (RING) {
    seq_len = a.ring_len[b];
    if (seq_len < 0) {
      if (threadIdx.x == 0 && split == 0 && kvh == 0) set_status(a.status, kDevRingState);
      seq_len = 0;
    }
    n_tok = min(seq_len, a.ring_slots);
  } else {
    seq_len = a.kv_len[b];
    if (seq_len != 0 &&
        ((a.q_pos0 == nullptr && seq_len < a.num_q) || seq_len < 0 || seq_len > a.max_pages * a.page_size)) {
      if (threadIdx.x == 0 && split == 0 && kvh == 0) set_status(a.status, kDevLenOob);
      seq_len = 0;
    }
    n_tok = seq_len;
  }
  // Windowed paged mode: the attended positions are [0, pw_sink_end) and
  // [pw_lo_win, n_tok).  Tiles holding none of them are skipped: virtual tile v
  // maps to tile v for the ns sink tiles, then to tw0 + (v - ns).
  const bool pwin = !RING && a.paged_window != 0;
  const int pw_sink_end = pwin ? min(a.sinks, n_tok) : n_tok;
  const int pw_lo_win = pwin ? max(a.sinks, n_tok - a.window) : n_tok;
  const int ns = pwin ? (pw_sink_end + kTileTokens - 1) / kTileTokens : 0;
  const int tw0 = pwin ? max(ns, pw_lo_win / kTileTokens) : 0;
  const int ntiles = pwin ? ns + max(0, (n_tok + kTileTokens - 1) / kTileTokens - tw0)
                          : (n_tok + kTileTokens - 1) / kTileTokens;
  auto tile_of = [&](int v) { return (!pwin || v < ns) ? v : tw0 + (v - ns); };
  // position of query 0 in this cache: query i attends positions <= q_first + i
  const int q_first = (!RING && a.q_pos0 != nullptr) ? a.q_pos0[b] : n_tok - a.num_q;
  const int tps = (ntiles + a.nsplit - 1) / a.nsplit;
  const int t_begin = min(split * tps, ntiles);
  const int t_end = min(t_begin + tps, ntiles);
  const int my_tiles = t_end - t_begin;

  // ---- producer: tile k of the split goes to stage k % STAGES
  const int box_rows = RING ? kTileTokens : min(a.page_size, kTileTokens);
  const int boxes = kTileTokens / box_rows;
  // the page-table entries of tile k (boxes of them; -1 past the sequence),
  // read one tile ahead of their use so the round trip overlaps the wait for
  // a free stage
  auto pages_of = [&](int k, int (&pg)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tok = tile_of(t_begin + k) * kTileTokens + j * box_rows;
      pg[j] = (!RING && k < my_tiles && j < boxes && tok < n_tok)
                  ? a.page_table[static_cast<size_t>(b) * a.max_pages + tok / a.page_size]
                  : -1;
    }
  };
  auto produce = [&](int k, const int (&pg)[4]) {
    const uint64_t pol = ptx::policy_evict_first();
    const int stage = k % STAGES;
    const int oob_z = RING ? 0x7fffffff : a.num_pages * a.Hkv;  // past the tensor: zero fill
    const int tile = tile_of(t_begin + k);
    const uint32_t kdst = sbase + Plan::kOffK + stage * Plan::kStageBytes;
    const uint32_t vdst = kdst + Plan::kTileBytes;
    const uint32_t fb = bar_full + 8 * stage;
    int valid = 1;
    if (RING) {
      stage_flag[stage] = 1;
      ptx::mbar_arrive_expect_tx(fb, Plan::kStageBytes);
      const int z = b * a.Hkv + kvh;
#pragma unroll
      for (int c = 0; c < Plan::kChunks; ++c) {
        ptx::tma_load_3d(kdst + c * Plan::kChunkBytes, &tmap_k, fb, c * 64, tile * kTileTokens, z, pol);
        ptx::tma_load_3d(vdst + c * Plan::kChunkBytes, &tmap_v, fb, c * 64, tile * kTileTokens, z, pol);
      }
    } else {
      // resolve the pages of this tile first, so the validity flag is
      // published together with the barrier arrival
      int zs[4];
      int ys[4];
      const int tok0 = tile * kTileTokens;
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
      if (!valid) set_status(a.status, kDevPageOob);
      stage_flag[stage] = valid;
      ptx::mbar_arrive_expect_tx(fb, Plan::kStageBytes);
      for (int j = 0; j < boxes; ++j) {
#pragma unroll
        for (int c = 0; c < Plan::kChunks; ++c) {
          const uint32_t off = c * Plan::kChunkBytes + j * box_rows * 128;
          ptx::tma_load_3d(kdst + off, &tmap_k, fb, c * 64, ys[j], zs[j], pol);
          ptx::tma_load_3d(vdst + off, &tmap_v, fb, c * 64, ys[j], zs[j], pol);
        }
      }
    }
  };
  __syncthreads();
  // let the dependent combine kernel get scheduled while this grid runs; it
  // waits in-kernel until this grid has finished and its writes are visible
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // =================================================================== producer
  if (warp == kProducerWarp) {
    if (lane == 0 && my_tiles > 0) {
      ptx::prefetch_tmap(&tmap_k);
      ptx::prefetch_tmap(&tmap_v);
      int issued = 0;
      int pg_cur[4], pg_nxt[4];
      pages_of(0, pg_cur);
      for (int k = 0; k < my_tiles; ++k) {
        // entries four tiles ahead head for L2; the next tile's are read now
        if (!RING && k + 4 < my_tiles) {
          const int ahead = tile_of(t_begin + k + 4) * kTileTokens;
          if (ahead < n_tok)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.page_table + static_cast<size_t>(b) * a.max_pages +
                                                              ahead / a.page_size));
        }
        pages_of(k + 1, pg_nxt);
        const int stage = k % STAGES;
        const uint32_t par = ((k / STAGES) & 1) ^ 1;
        if (!ptx::mbar_wait(bar_empty + 8 * stage, par)) {
          set_status(a.status, kDevTimeout);
          break;
        }
        produce(k, pg_cur);
        issued = k + 1;
#pragma unroll
        for (int j = 0; j < 4; ++j) pg_cur[j] = pg_nxt[j];
      }
      // no copy may still be writing shared memory when the CTA exits (after
      // a timeout the consumers stop early): wait, bounded, for the last load
      // of each stage
      for (int k = max(issued - STAGES, 0); k < issued; ++k)
        if (!ptx::mbar_wait(bar_full + 8 * (k % STAGES), (k / STAGES) & 1)) set_status(a.status, kDevTimeout);
    }
    return;
  }

  // =================================================================== compute
  const int tid = threadIdx.x;  // 0..127
  const int g = lane >> 2;      // mma group id
  const int t4 = lane & 3;      // thread in group

  // ---- Q rows of this KV head into shared memory (swizzled like K chunks)
  {
    constexpr int kUnitsPerRow = D / 8;
    for (int u = tid; u < kRows * kUnitsPerRow; u += kComputeThreads) {
      const int r = u / kUnitsPerRow;
      const int j = u % kUnitsPerRow;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (r < a.rows) {
        const int qi = r / a.G;
        const int gg = r % a.G;
        const __nv_bfloat16* src =
            a.q + ((static_cast<size_t>(b) * a.num_q + qi) * a.Hq + kvh * a.G + gg) * D + j * 8;
        val = *reinterpret_cast<const uint4*>(src);
      }
      const uint32_t dst = s_q + (j >> 3) * Plan::kQChunkBytes + swz(r, j & 7);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(val.x), "r"(val.y),
                   "r"(val.z), "r"(val.w)
                   : "memory");
    }
  }
  if (tid == 0) abort_flag[0] = 0;
  ptx::named_bar_sync(kBarCompute, kComputeThreads);

  // ---- per-thread row bookkeeping: rows nt*8 + 2*t4 + j, j in {0,1}
  int lim[NT][2];  // exclusive token limit (causal); only used on masked tiles
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int row = nt * 8 + 2 * t4 + j;
      if (RING || row >= a.rows)
        lim[nt][j] = n_tok;
      else
        lim[nt][j] = min(n_tok, q_first + row / a.G + 1);
    }

  float o_acc[kMT][NT][4];
  float m_run[NT][2];
  float l_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o_acc[mt][nt][e] = 0.f;
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
  }

  const int dbase = warp * (D / 4);
  // the accumulator folded so far (in the split's partial slot, units of
  // 2^m_g) for each of this thread's rows
  float m_g[NT][2];
  bool have_g[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_g[nt][0] = m_g[nt][1] = -INFINITY;
    have_g[nt][0] = have_g[nt][1] = false;
  }
  auto row_dst = [&](int row) -> float* {
    const size_t grow = (static_cast<size_t>(b) * a.num_q + row / a.G) * a.Hq + kvh * a.G + row % a.G;
    return a.part_o + (grow * a.nsplit + split) * D;
  };
  const int first_masked_tok = RING ? -1 : min(n_tok, q_first + 1);  // tokens >= this may be masked

  for (int k = 0; k < my_tiles; ++k) {
    if (k > 0 && (k % kRunTiles) == 0) {
      // fold the finished run: G = G 2^(m_g - m_run) + O, then restart O
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int row = nt * 8 + 2 * t4 + j;
          if (row >= a.rows || m_run[nt][j] == -INFINITY) continue;
          const float gs = have_g[nt][j] ? ptx::ex2(m_g[nt][j] - m_run[nt][j]) : 0.f;
          float* dst = row_dst(row);
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt) {
            const int d = dbase + 16 * mt + g;
            dst[d] = (have_g[nt][j] ? dst[d] * gs : 0.f) + o_acc[mt][nt][j];
            dst[d + 8] = (have_g[nt][j] ? dst[d + 8] * gs : 0.f) + o_acc[mt][nt][j + 2];
            o_acc[mt][nt][j] = 0.f;
            o_acc[mt][nt][j + 2] = 0.f;
          }
          m_g[nt][j] = m_run[nt][j];
          have_g[nt][j] = true;
        }
    }
    const int stage = k % STAGES;
    const uint32_t par = (k / STAGES) & 1;
    const bool got = ptx::mbar_wait(bar_full + 8 * stage, par);
    const uint32_t kst = sbase + Plan::kOffK + stage * Plan::kStageBytes;
    const uint32_t vst = kst + Plan::kTileBytes;
    const int tile = tile_of(t_begin + k);
    const int tok0 = tile * kTileTokens;
    const bool tile_ok = got && stage_flag[stage] != 0;

    // zero V rows past the valid length (tail tile only)
    if (got && tok0 + kTileTokens > n_tok) {
      const int r0 = max(n_tok - tok0, 0);
      constexpr int kUnits = D / 8;
      for (int u = tid; u < (kTileTokens - r0) * kUnits; u += kComputeThreads) {
        const int r = r0 + u / kUnits;
        const int j = u % kUnits;
        const uint32_t dst = vst + (j >> 3) * Plan::kChunkBytes + r * 128 + ((j & 7) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0) : "memory");
      }
      ptx::fence_proxy_async_smem();
    }

    // ---- 1. S^T = K Q^T for tokens [16*warp, 16*warp + 16)
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
    if (tile_ok) {
      float s2[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s2[nt][e] = 0.f;
      const int krow = 16 * warp + ((lane >> 3) & 1) * 8 + (lane & 7);
      const int kunit_hi = lane >> 4;  // 0 or 1: second 8 columns of the k-step
#pragma unroll
      for (int kk2 = 0; kk2 < D / 32; ++kk2) {
        uint32_t a0[4], a1[4];
        {
          const int d0 = kk2 * 32;
          const int u0 = ((d0 & 63) >> 3) + kunit_hi;
          const int u1 = (((d0 + 16) & 63) >> 3) + kunit_hi;
          ptx::ldsm_x4(kst + (d0 >> 6) * Plan::kChunkBytes + swz(krow, u0), a0);
          ptx::ldsm_x4(kst + ((d0 + 16) >> 6) * Plan::kChunkBytes + swz(krow, u1), a1);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t bq[4];
          const int qrow = nt * 8 + (lane & 7);
          const int d = kk2 * 32 + (lane >> 3) * 8;
          ptx::ldsm_x4(s_q + (d >> 6) * Plan::kQChunkBytes + swz(qrow, (d & 63) >> 3), bq);
          ptx::mma_bf16_16816(s[nt], a0, bq[0], bq[1]);
          // one row tile: a second accumulator breaks the dependency chain;
          // several row tiles already interleave independent chains
          if (NT == 1)
            ptx::mma_bf16_16816(s2[nt], a1, bq[2], bq[3]);
          else
            ptx::mma_bf16_16816(s[nt], a1, bq[2], bq[3]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
    }

    // ---- scale and mask; S^T element e: token g (+8 for e>=2), row 2*t4 + (e&1)
    const int tokA = tok0 + 16 * warp + g;
    const int tokB = tokA + 8;
    bool need_mask = !tile_ok || RING || pwin || (tok0 + kTileTokens > first_masked_tok);
    if (!need_mask) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] *= a.scale_log2;
    } else {
      bool okA = tile_ok, okB = tile_ok;
      if (RING) {
        const int R = a.ring_slots;
        const int lo_win = max(a.sinks, seq_len - a.window);
        const int sink_end = min(a.sinks, seq_len);
        const int tagA = (tokA < R) ? a.ring_tags[static_cast<size_t>(b) * R + tokA] : -1;
        const int tagB = (tokB < R) ? a.ring_tags[static_cast<size_t>(b) * R + tokB] : -1;
        okA = okA && tokA < n_tok && tagA >= 0 && tagA < seq_len && (tagA < sink_end || tagA >= lo_win);
        okB = okB && tokB < n_tok && tagB >= 0 && tagB < seq_len && (tagB < sink_end || tagB >= lo_win);
      } else if (pwin) {
        okA = okA && (tokA < pw_sink_end || (tokA >= pw_lo_win && tokA < n_tok));
        okB = okB && (tokB < pw_sink_end || (tokB >= pw_lo_win && tokB < n_tok));
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = (e < 2) ? tokA : tokB;
          const bool ok = ((e < 2) ? okA : okB) && tok < lim[nt][e & 1];
          s[nt][e] = ok ? s[nt][e] * a.scale_log2 : -INFINITY;
        }
    }

    // ---- 2. tile row maxima, shared across the compute warps
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float mx = fmaxf(s[nt][j], s[nt][j + 2]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (g == 0) red[warp * kRows + nt * 8 + 2 * t4 + j] = mx;
      }
    if (lane == 0 && !got) abort_flag[0] = 1;
    ptx::named_bar_sync(kBarCompute, kComputeThreads);
    if (abort_flag[0] != 0) {
      if (tid == 0) set_status(a.status, kDevTimeout);
      break;  // every compute warp takes this branch after the same barrier
    }

    float p[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int row = nt * 8 + 2 * t4 + j;
        float tm = red[row];
#pragma unroll
        for (int w = 1; w < kComputeWarps; ++w) tm = fmaxf(tm, red[w * kRows + row]);
        const float m_new = fmaxf(m_run[nt][j], tm);
        const float base = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = ptx::ex2(m_run[nt][j] - base);
        m_run[nt][j] = m_new;
        p[nt][j] = ptx::ex2(s[nt][j] - base);
        p[nt][j + 2] = ptx::ex2(s[nt][j + 2] - base);
        l_run[nt][j] = l_run[nt][j] * alpha + p[nt][j] + p[nt][j + 2];
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
          o_acc[mt][nt][j] *= alpha;
          o_acc[mt][nt][j + 2] *= alpha;
        }
      }

    // ---- 3. P (hi + lo bf16) into shared memory, [row][token] with 144 B pitch
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t hA = ptx::pack_bf16x2(p[nt][0], p[nt][1]);
      const uint32_t hB = ptx::pack_bf16x2(p[nt][2], p[nt][3]);
      const uint32_t lA = ptx::pack_bf16x2(p[nt][0] - ptx::bf16lo_to_f32(hA), p[nt][1] - ptx::bf16hi_to_f32(hA));
      const uint32_t lB = ptx::pack_bf16x2(p[nt][2] - ptx::bf16lo_to_f32(hB), p[nt][3] - ptx::bf16hi_to_f32(hB));
      const uint32_t row_off = (nt * 8 + g) * kPPitchBytes + (16 * warp + 2 * t4) * 2;
      const uint32_t hi = s_p + row_off;
      const uint32_t lo = s_p + kRows * kPPitchBytes + row_off;
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(hi), "r"(ptx::movmatrix_trans(hA)) : "memory");
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(hi + 16), "r"(ptx::movmatrix_trans(hB)) : "memory");
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(lo), "r"(ptx::movmatrix_trans(lA)) : "memory");
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(lo + 16), "r"(ptx::movmatrix_trans(lB)) : "memory");
    }
    ptx::named_bar_sync(kBarCompute, kComputeThreads);

    // ---- 4. O^T[d][row] += V^T P^T for this warp's columns
#pragma unroll
    for (int ks = 0; ks < kTileTokens / 16; ++ks) {
      uint32_t bp[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int prow = nt * 8 + (lane & 7);
        const int pcol = 16 * ks + ((lane >> 3) & 1) * 8;
        const int buf = lane >> 4;
        ptx::ldsm_x4(s_p + buf * kRows * kPPitchBytes + prow * kPPitchBytes + pcol * 2, bp[nt]);
      }
      const int vtok = 16 * ks + (lane >> 4) * 8 + (lane & 7);
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) {
        const int d = dbase + 16 * mt + ((lane >> 3) & 1) * 8;
        uint32_t av[4];
        ptx::ldsm_x4_trans(vst + (d >> 6) * Plan::kChunkBytes + swz(vtok, (d & 63) >> 3), av);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          ptx::mma_bf16_16816(o_acc[mt][nt], av, bp[nt][0], bp[nt][1]);
          ptx::mma_bf16_16816(o_acc[mt][nt], av, bp[nt][2], bp[nt][3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar_empty + 8 * stage);
  }

  // ---- finish: row sums across lanes and warps, normalise, write partials
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[nt][j];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[nt][j] = l;
    }
  ptx::named_bar_sync(kBarCompute, kComputeThreads);  // everyone is done reading red
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (g == 0) red[warp * kRows + nt * 8 + 2 * t4 + j] = l_run[nt][j];
  ptx::named_bar_sync(kBarCompute, kComputeThreads);

#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int row = nt * 8 + 2 * t4 + j;
      if (row >= a.rows) continue;
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) l += red[w * kRows + row];
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const size_t grow = (static_cast<size_t>(b) * a.num_q + row / a.G) * a.Hq + kvh * a.G + row % a.G;
      float* dst = row_dst(row);
      const bool hg = have_g[nt][j];
      const float gs = hg ? ptx::ex2(m_g[nt][j] - m_run[nt][j]) : 0.f;
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) {
        const int d = dbase + 16 * mt + g;
        dst[d] = ((hg ? dst[d] * gs : 0.f) + o_acc[mt][nt][j]) * inv;
        dst[d + 8] = ((hg ? dst[d + 8] * gs : 0.f) + o_acc[mt][nt][j + 2]) * inv;
      }
      if (warp == 0 && g == 0) {
        // m_run is in log2 units of the scaled score
        a.part_lse[grow * a.nsplit + split] =
            (l > 0.f) ? m_run[nt][j] * 0.69314718055994531f + logf(l) : -INFINITY;
      }
    }
}

}  // namespace wmtp

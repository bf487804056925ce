// libwmtp: the C ABI declared in include/wmtp.h.
//
// Host side only: argument validation, workspace sizing, TMA tensor-map
// encoding and kernel launches.  Every step of the attention path runs in the
// kernels of decode_attn.cuh, combine.cuh and ring.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "combine.cuh"
#include "decode_attn.cuh"
#include "ring.cuh"
#include "verify_tc.cuh"
#include "wmtp.h"

namespace wmtp {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxRows = 64;             // rows per KV head of the mma.sync kernel
constexpr int kMaxRowsTc = 128;          // rows per KV head of the tcgen05 verify
constexpr int kMaxGammaMax = 16;
constexpr int kMaxVerifyWaves = 8;      // CTAs per SM in turn for the tcgen05 verify of a batch
constexpr int kMinTilesPerSplit = 16;   // extra waves only while full-capacity splits keep this many tiles
constexpr size_t kWsAlign = 256;
constexpr int kMaxGridYZ = 65535;       // gridDim.y / gridDim.z limit

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------- device info
struct DeviceInfo {
  int sms = 0;
};

DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

wmtp_status current_device(int* dev, DeviceInfo* info) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return WMTP_ERR_CUDA;
  const int d = *dev;
  std::call_once(g_dev_once[d], [d]() {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d) == cudaSuccess) g_dev[d].sms = sms;
  });
  if (g_dev[d].sms <= 0) return WMTP_ERR_CUDA;
  *info = g_dev[d];
  return WMTP_OK;
}

// ---------------------------------------------------------------- launches
// Dynamic shared-memory opt-in of one kernel, set once per device.  Only a
// success is remembered: a failed attempt (its error cleared from this
// library's runtime state) is retried by the next call.  Concurrent first
// calls from several host threads serialise on the mutex.
struct SmemAttrOnce {
  std::atomic<bool> done[kMaxDevices];
  std::mutex mu;
};

template <typename Kern>
wmtp_status ensure_smem_attr(SmemAttrOnce& once, Kern kern, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WMTP_ERR_CUDA;
  if (once.done[dev].load(std::memory_order_acquire)) return WMTP_OK;
  std::lock_guard<std::mutex> lock(once.mu);
  if (once.done[dev].load(std::memory_order_relaxed)) return WMTP_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
    (void)cudaGetLastError();
    return WMTP_ERR_CUDA;
  }
  once.done[dev].store(true, std::memory_order_release);
  return WMTP_OK;
}

// A launch whose success is read from the launch call itself, never from
// cudaGetLastError (which would also report an unrelated earlier error left
// on this thread, after the kernel had been queued).  `programmatic`: launch
// as a programmatic dependent of the previous work on the stream (the kernel
// must execute griddepcontrol.wait before its first memory access).
template <typename... Exp, typename... Act>
wmtp_status launch_plain(bool programmatic, void (*kern)(Exp...), dim3 grid, dim3 block, cudaStream_t st,
                         Act&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = programmatic ? attr : nullptr;
  cfg.numAttrs = programmatic ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...) == cudaSuccess ? WMTP_OK : WMTP_ERR_CUDA;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

EncodeTiledFn encoder() {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

// A [dim2][dim1][D] bf16 tensor, loaded in boxes of 64 columns x box_rows rows
// with the 128-byte swizzle the kernels read with.
wmtp_status encode_map(CUtensorMap* m, void* base, int D, long long dim1, long long dim2, int box_rows) {
  EncodeTiledFn enc = encoder();
  if (enc == nullptr) return WMTP_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(dim1),
                        static_cast<cuuint64_t>(dim2)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(dim1) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WMTP_OK : WMTP_ERR_CUDA;
}

// ---------------------------------------------------------------- validation
bool supported_page(int p) { return p == 16 || p == 32 || p == 64 || p == 128 || p == 256; }

wmtp_status check_params(const wmtp_params* p, int num_q) {
  if (p == nullptr) return WMTP_ERR_INVALID_ARG;
  if (p->num_heads_q <= 0 || p->num_heads_kv <= 0 || num_q <= 0) return WMTP_ERR_INVALID_ARG;
  if (p->num_heads_q % p->num_heads_kv != 0) return WMTP_ERR_INVALID_ARG;
  if (p->num_heads_kv > kMaxGridYZ) return WMTP_ERR_UNSUPPORTED;
  if (!(p->sm_scale >= 0.f) || !std::isfinite(p->sm_scale)) return WMTP_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 256) return WMTP_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(p->num_heads_q / p->num_heads_kv) * num_q;
  // up to 64 rows on the mma.sync kernel; the tcgen05 verify (head_dim 256,
  // two or more queries) takes up to 128
  if (rows > (p->head_dim == 256 && num_q >= 2 ? kMaxRowsTc : kMaxRows)) return WMTP_ERR_UNSUPPORTED;
  return WMTP_OK;
}

float scale_log2(const wmtp_params* p) {
  const float s = (p->sm_scale > 0.f) ? p->sm_scale : 1.f / std::sqrt(static_cast<float>(p->head_dim));
  return s * 1.4426950408889634f;
}

// ---------------------------------------------------------------- launch plan
struct LaunchPlan {
  int nsplit = 1;
  size_t off_lse = 0;
  size_t bytes = 0;
};

template <int D, int NT>
int ctas_per_sm() {
  constexpr int alloc = SmemPlan<D, NT, pick_stages<D, NT>()>::kAlloc;
  const int per = 233472 / (alloc + 1024);
  return per < 1 ? 1 : per;
}

int ctas_per_sm_rt(int D, int NT) {
#define WMTP_CPS(DD, N) \
  if (D == DD && NT == N) return ctas_per_sm<DD, N>();
#define WMTP_CPS_D(DD) WMTP_CPS(DD, 1) WMTP_CPS(DD, 2) WMTP_CPS(DD, 3) WMTP_CPS(DD, 4) \
  WMTP_CPS(DD, 5) WMTP_CPS(DD, 6) WMTP_CPS(DD, 7) WMTP_CPS(DD, 8)
  WMTP_CPS_D(64)
  WMTP_CPS_D(256)
#undef WMTP_CPS_D
#undef WMTP_CPS
  return 1;
}

// `waves`: how many CTAs each SM runs in turn.  One wave splits the batch's
// work evenly only when the sequences have similar lengths; with w = B waves
// every sequence gets the same number of splits and each SM runs one CTA of
// every sequence, so its total work follows the sum of the lengths whatever
// they are (used by the tcgen05 verify, which is bound per SM by its MMA issue
// chain; the bandwidth-bound kernels rebalance through the memory system).
LaunchPlan make_plan(int sms, int B, int Hkv, long long rows_total, int D, int ctas_per_sm, long long max_tiles,
                     int waves = 1) {
  LaunchPlan pl;
  const long long slots = static_cast<long long>(sms) * ctas_per_sm * waves;
  long long per = slots / (static_cast<long long>(B) * Hkv);
  if (waves > 1 && per > max_tiles / kMinTilesPerSplit) per = max_tiles / kMinTilesPerSplit;
  if (per < 1) per = 1;
  if (per > max_tiles) per = max_tiles;
  if (per < 1) per = 1;
  pl.nsplit = static_cast<int>(per);
  const size_t po = static_cast<size_t>(rows_total) * pl.nsplit * D * sizeof(float);
  pl.off_lse = align_up(po, kWsAlign);
  pl.bytes = pl.off_lse + align_up(static_cast<size_t>(rows_total) * pl.nsplit * sizeof(float), kWsAlign);
  return pl;
}

// Launch an attention kernel as a programmatic dependent of whatever the
// stream ran before: its barrier and tensor-memory set-up may overlap that
// kernel's tail, and it executes griddepcontrol.wait before its first
// global-memory access, so stream order is kept for every byte it reads.
template <typename Kern>
wmtp_status launch_programmatic(Kern kern, dim3 grid, int threads, int smem, cudaStream_t st,
                                const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tk, tv, a) == cudaSuccess ? WMTP_OK : WMTP_ERR_CUDA;
}

// ---------------------------------------------------------------- dispatch
template <int D, int NT, bool RING>
wmtp_status launch_decode_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, int B,
                            cudaStream_t st) {
  constexpr int S = pick_stages<D, NT>();
  constexpr int alloc = SmemPlan<D, NT, S>::kAlloc;
  static_assert(alloc <= kSmemLimit, "shared-memory plan exceeds the sm_100 per-block limit");
  auto kern = decode_attn_kernel<D, NT, S, RING>;
  static SmemAttrOnce once;
  const wmtp_status s = ensure_smem_attr(once, kern, alloc);
  if (s != WMTP_OK) return s;
  return launch_programmatic(kern, dim3(a.nsplit, a.Hkv, B), kThreads, alloc, st, tk, tv, a);
}

template <bool RING>
wmtp_status launch_decode(int D, int NT, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                          int B, cudaStream_t st) {
#define WMTP_CASE(DD, N) \
  if (D == DD && NT == N) return launch_decode_t<DD, N, RING>(tk, tv, a, B, st);
#define WMTP_CASE_D(DD) WMTP_CASE(DD, 1) WMTP_CASE(DD, 2) WMTP_CASE(DD, 3) WMTP_CASE(DD, 4) \
  WMTP_CASE(DD, 5) WMTP_CASE(DD, 6) WMTP_CASE(DD, 7) WMTP_CASE(DD, 8)
  WMTP_CASE_D(64)
  WMTP_CASE_D(256)
#undef WMTP_CASE_D
#undef WMTP_CASE
  return WMTP_ERR_UNSUPPORTED;
}

template <int M>
wmtp_status launch_verify_tc_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, int B,
                               cudaStream_t st) {
  constexpr int alloc = TcPlan<kTcKStages, kTcVStages, M == 64>::kAlloc;
  static_assert(alloc <= kSmemLimit, "shared-memory plan exceeds the sm_100 per-block limit");
  auto kern = verify_tc_kernel<kTcKStages, kTcVStages, M>;
  static SmemAttrOnce once;
  const wmtp_status s = ensure_smem_attr(once, kern, alloc);
  if (s != WMTP_OK) return s;
  return launch_programmatic(kern, dim3(a.nsplit, a.Hkv, B), kTcThreads, alloc, st, tk, tv, a);
}

// M = 64 MMAs while the rows fit (half the tensor work of M = 128 at the
// same issue cost), M = 128 for 65..128 rows.
wmtp_status launch_verify_tc(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, int B,
                             cudaStream_t st) {
  return a.rows <= 64 ? launch_verify_tc_t<64>(tk, tv, a, B, st) : launch_verify_tc_t<128>(tk, tv, a, B, st);
}

// Verify blocks of head_dim 256 with 9..128 query rows run on tcgen05.
bool use_verify_tc(int D, int num_q, int rows) { return D == 256 && num_q >= 2 && rows >= 9 && rows <= kMaxRowsTc; }

// `after_decode`: launched right behind a decode kernel on the same stream, as
// its programmatic dependent (the combine waits in-kernel for the partials).
wmtp_status launch_combine(int rows, int D, int nsplit, const float* po, const float* pl, void* out,
                           int out_fp32, float* lse_out, cudaStream_t st, bool after_decode) {
  if (rows <= 0) return WMTP_OK;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(rows, (D + kCombineCols - 1) / kCombineCols, 1);
  cfg.blockDim = dim3(kCombineThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_decode ? 1 : 0;
  cudaError_t e = out_fp32 ? cudaLaunchKernelEx(&cfg, splitkv_combine_kernel<true>, po, pl, nsplit, D, out, lse_out)
                           : cudaLaunchKernelEx(&cfg, splitkv_combine_kernel<false>, po, pl, nsplit, D, out,
                                                lse_out);
  return e == cudaSuccess ? WMTP_OK : WMTP_ERR_CUDA;
}

// Shared tail of the three attention entry points.
template <bool RING>
wmtp_status run_attention(const wmtp_params* p, int B, int num_q, const void* q, const CUtensorMap* tk,
                          const CUtensorMap* tv, DecodeArgs a, long long max_tiles, void* out,
                          int out_fp32, float* lse_out, void* workspace, size_t* workspace_bytes,
                          cudaStream_t st, bool maps_ready) {
  int dev = 0;
  DeviceInfo info;
  wmtp_status s = current_device(&dev, &info);
  if (s != WMTP_OK) return s;
  const int D = p->head_dim;
  const int G = p->num_heads_q / p->num_heads_kv;
  const int rows = num_q * G;
  const int NT = (rows + 7) / 8;
  const long long rows_total = static_cast<long long>(B) * num_q * p->num_heads_q;
  if (rows_total > 0x7fffffffLL) return WMTP_ERR_UNSUPPORTED;  // the combine's grid x
  const bool tc = !RING && use_verify_tc(D, num_q, rows);
  const int waves = tc ? (B < kMaxVerifyWaves ? B : kMaxVerifyWaves) : 1;
  const int per_sm = tc ? 1 : ctas_per_sm_rt(D, NT);  // the tcgen05 verify holds a whole SM
  LaunchPlan pl = make_plan(info.sms, B, p->num_heads_kv, rows_total, D, per_sm, max_tiles < 1 ? 1 : max_tiles,
                            waves);
  if (workspace == nullptr) {
    *workspace_bytes = pl.bytes;
    return WMTP_OK;
  }
  if (*workspace_bytes < pl.bytes || !aligned(workspace, kWsAlign)) return WMTP_ERR_WORKSPACE;
  if (q == nullptr || out == nullptr || !aligned(q, 16) || !aligned(out, 16)) return WMTP_ERR_INVALID_ARG;
  if (!maps_ready) return WMTP_ERR_CUDA;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.num_q = num_q;
  a.Hq = p->num_heads_q;
  a.Hkv = p->num_heads_kv;
  a.G = G;
  a.rows = rows;
  a.nsplit = pl.nsplit;
  a.scale_log2 = scale_log2(p);
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.off_lse);
  if (tc) {
    s = launch_verify_tc(*tk, *tv, a, B, st);  // writes a.k_new / a.v_new itself
  } else {
    if (a.k_new != nullptr) {
      // the mma.sync verify's shapes: the append as its own launch in front
      s = launch_plain(true, paged_write_kernel, dim3(num_q, B), dim3(128), st, reinterpret_cast<uint4*>(a.k_pool_w),
                       reinterpret_cast<uint4*>(a.v_pool_w), a.num_pages, a.page_table, a.max_pages, a.page_size,
                       a.Hkv, D, static_cast<const int32_t*>(nullptr), num_q,
                       reinterpret_cast<const uint4*>(a.k_new), reinterpret_cast<const uint4*>(a.v_new), a.status,
                       a.kv_len);
      if (s != WMTP_OK) return s;
      a.k_new = a.v_new = nullptr;
    }
    s = launch_decode<RING>(D, NT, *tk, *tv, a, B, st);
  }
  if (s != WMTP_OK) return s;
  return launch_combine(static_cast<int>(rows_total), D, pl.nsplit, a.part_o, a.part_lse, out, out_fp32,
                        lse_out, st, true);
}

// `window`: attend only the sink + window positions of the pages (num_q 1).
// `k_new`, `v_new` (verify only): the num_q new tokens' K/V, written at the
// sequence's last num_q positions before they are read -- inside the tcgen05
// verify kernel, else by a paged write launched in front of it.
wmtp_status paged_attention(const wmtp_params* p, int32_t batch, int32_t num_q, const void* q,
                            const wmtp_paged_kv* kv, void* out, int32_t out_fp32, float* lse_out,
                            void* workspace, size_t* workspace_bytes, int32_t* status_word, void* stream,
                            bool window = false, const int32_t* q_pos0 = nullptr, const void* k_new = nullptr,
                            const void* v_new = nullptr) {
  wmtp_status s = check_params(p, num_q);
  if (s != WMTP_OK) return s;
  if (window && (num_q != 1 || p->sinks < 0 || p->window < 1)) return WMTP_ERR_INVALID_ARG;
  if (batch < 0 || kv == nullptr || workspace_bytes == nullptr) return WMTP_ERR_INVALID_ARG;
  if (batch > kMaxGridYZ) return WMTP_ERR_UNSUPPORTED;
  if (!supported_page(p->page_size)) return WMTP_ERR_UNSUPPORTED;
  if (kv->num_pages <= 0 || kv->max_pages <= 0) return WMTP_ERR_INVALID_ARG;
  const long long max_tokens = static_cast<long long>(kv->max_pages) * p->page_size;
  if (max_tokens > (1LL << 30)) return WMTP_ERR_UNSUPPORTED;
  if (static_cast<long long>(kv->num_pages) * p->num_heads_kv > 0x7fffffffLL) return WMTP_ERR_UNSUPPORTED;
  if (batch == 0) {
    if (workspace == nullptr) *workspace_bytes = 0;
    return WMTP_OK;
  }
  long long max_tiles = (max_tokens + kTileTokens - 1) / kTileTokens;
  if (window) {  // at most the sink tiles plus the tiles the window touches
    const long long wt =
        (p->sinks + kTileTokens - 1) / kTileTokens + (p->window + kTileTokens - 1) / kTileTokens + 1;
    if (wt < max_tiles) max_tiles = wt;
  }
  CUtensorMap tk, tv;
  bool ready = false;
  if (workspace != nullptr) {
    if (kv->k_pool == nullptr || kv->v_pool == nullptr || kv->page_table == nullptr || kv->kv_len == nullptr)
      return WMTP_ERR_INVALID_ARG;
    if (!aligned(kv->k_pool, 16) || !aligned(kv->v_pool, 16)) return WMTP_ERR_INVALID_ARG;
    const int box = p->page_size < kTileTokens ? p->page_size : kTileTokens;
    const long long dim2 = static_cast<long long>(kv->num_pages) * p->num_heads_kv;
    s = encode_map(&tk, kv->k_pool, p->head_dim, p->page_size, dim2, box);
    if (s != WMTP_OK) return s;
    s = encode_map(&tv, kv->v_pool, p->head_dim, p->page_size, dim2, box);
    if (s != WMTP_OK) return s;
    ready = true;
  }
  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.page_table = kv->page_table;
  a.kv_len = kv->kv_len;
  a.max_pages = kv->max_pages;
  a.num_pages = kv->num_pages;
  a.page_size = p->page_size;
  a.status = status_word;
  a.paged_window = window ? 1 : 0;
  a.q_pos0 = q_pos0;
  a.sinks = p->sinks;
  a.window = p->window;
  if (k_new != nullptr && workspace != nullptr) {
    if (!aligned(k_new, 16) || !aligned(v_new, 16)) return WMTP_ERR_INVALID_ARG;
    a.k_new = static_cast<const __nv_bfloat16*>(k_new);
    a.v_new = static_cast<const __nv_bfloat16*>(v_new);
    a.k_pool_w = static_cast<__nv_bfloat16*>(kv->k_pool);
    a.v_pool_w = static_cast<__nv_bfloat16*>(kv->v_pool);
  }
  return run_attention<false>(p, batch, num_q, q, &tk, &tv, a, max_tiles, out, out_fp32, lse_out, workspace,
                              workspace_bytes, static_cast<cudaStream_t>(stream), ready);
}

RingArgs ring_args(const wmtp_params* p, const wmtp_ring* r) {
  RingArgs a;
  a.k = static_cast<uint4*>(r->k);
  a.v = static_cast<uint4*>(r->v);
  a.tags = r->tags;
  a.len = r->len;
  a.committed = r->committed;
  a.undo_k = static_cast<uint4*>(r->undo_k);
  a.undo_v = static_cast<uint4*>(r->undo_v);
  a.undo_tags = r->undo_tags;
  a.batch = r->batch;
  a.Hkv = p->num_heads_kv;
  a.D = p->head_dim;
  a.S = p->sinks;
  a.W = p->window;
  a.R = p->sinks + p->window;
  a.gmax = p->gamma_max;
  return a;
}

wmtp_status check_ring(const wmtp_params* p, const wmtp_ring* r) {
  if (p == nullptr || r == nullptr) return WMTP_ERR_INVALID_ARG;
  if (p->num_heads_kv <= 0 || p->sinks < 0 || p->window < 1) return WMTP_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 256) return WMTP_ERR_UNSUPPORTED;
  if (p->gamma_max < 0 || p->gamma_max > kMaxGammaMax) return WMTP_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->sinks) + p->window > (1 << 24)) return WMTP_ERR_UNSUPPORTED;
  if (r->batch < 0) return WMTP_ERR_INVALID_ARG;
  if (r->batch > 0 && (r->k == nullptr || r->v == nullptr || r->tags == nullptr || r->len == nullptr ||
                       r->committed == nullptr))
    return WMTP_ERR_INVALID_ARG;
  if (r->batch > 0 && p->gamma_max > 0 &&
      (r->undo_k == nullptr || r->undo_v == nullptr || r->undo_tags == nullptr))
    return WMTP_ERR_INVALID_ARG;
  if (!aligned(r->k, 16) || !aligned(r->v, 16) || !aligned(r->undo_k, 16) || !aligned(r->undo_v, 16))
    return WMTP_ERR_INVALID_ARG;
  return WMTP_OK;
}

}  // namespace
}  // namespace wmtp

using namespace wmtp;

extern "C" {

const char* wmtp_status_string(int32_t status) {
  switch (status) {
    case WMTP_OK: return "ok";
    case WMTP_ERR_INVALID_ARG: return "invalid argument";
    case WMTP_ERR_UNSUPPORTED: return "unsupported shape";
    case WMTP_ERR_WORKSPACE: return "workspace too small or misaligned";
    case WMTP_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

const char* wmtp_version(void) { return "0.1.0"; }

wmtp_status wmtp_draft_attn_full(const wmtp_params* params, int32_t batch, const void* q,
                                 const wmtp_paged_kv* kv, void* out, int32_t out_fp32, float* lse_out,
                                 void* workspace, size_t* workspace_bytes, int32_t* status_word,
                                 void* stream) {
  return paged_attention(params, batch, 1, q, kv, out, out_fp32, lse_out, workspace, workspace_bytes,
                         status_word, stream);
}

wmtp_status wmtp_draft_attn_windowed_paged(const wmtp_params* params, int32_t batch, const void* q,
                                           const wmtp_paged_kv* kv, void* out, int32_t out_fp32,
                                           float* lse_out, void* workspace, size_t* workspace_bytes,
                                           int32_t* status_word, void* stream) {
  return paged_attention(params, batch, 1, q, kv, out, out_fp32, lse_out, workspace, workspace_bytes,
                         status_word, stream, true);
}

wmtp_status wmtp_verify_attn_slice(const wmtp_params* params, int32_t batch, int32_t num_q, const void* q,
                                   const wmtp_paged_kv* kv, const int32_t* q_pos0, void* out, int32_t out_fp32,
                                   float* lse_out, void* workspace, size_t* workspace_bytes, int32_t* status_word,
                                   void* stream) {
  if (workspace != nullptr && q_pos0 == nullptr) return WMTP_ERR_INVALID_ARG;
  return paged_attention(params, batch, num_q, q, kv, out, out_fp32, lse_out, workspace, workspace_bytes,
                         status_word, stream, false, q_pos0);
}

wmtp_status wmtp_verify_attn(const wmtp_params* params, int32_t batch, int32_t num_q, const void* q,
                             const wmtp_paged_kv* kv, void* out, int32_t out_fp32, float* lse_out,
                             void* workspace, size_t* workspace_bytes, int32_t* status_word, void* stream) {
  return paged_attention(params, batch, num_q, q, kv, out, out_fp32, lse_out, workspace, workspace_bytes,
                         status_word, stream);
}

wmtp_status wmtp_verify_attn_append(const wmtp_params* params, int32_t batch, int32_t num_q, const void* q,
                                    const void* k_new, const void* v_new, const wmtp_paged_kv* kv, void* out,
                                    int32_t out_fp32, float* lse_out, void* workspace, size_t* workspace_bytes,
                                    int32_t* status_word, void* stream) {
  if (workspace != nullptr && batch > 0 && (k_new == nullptr || v_new == nullptr)) return WMTP_ERR_INVALID_ARG;
  return paged_attention(params, batch, num_q, q, kv, out, out_fp32, lse_out, workspace, workspace_bytes,
                         status_word, stream, false, nullptr, k_new, v_new);
}

wmtp_status wmtp_draft_attn_windowed(const wmtp_params* params, const void* q, const wmtp_ring* ring,
                                     void* out, int32_t out_fp32, float* lse_out, void* workspace,
                                     size_t* workspace_bytes, int32_t* status_word, void* stream) {
  wmtp_status s = check_params(params, 1);
  if (s != WMTP_OK) return s;
  s = check_ring(params, ring);
  if (s != WMTP_OK) return s;
  if (workspace_bytes == nullptr) return WMTP_ERR_INVALID_ARG;
  const int B = ring->batch;
  if (B > kMaxGridYZ) return WMTP_ERR_UNSUPPORTED;
  if (B == 0) {
    if (workspace == nullptr) *workspace_bytes = 0;
    return WMTP_OK;
  }
  const int R = params->sinks + params->window;
  const long long max_tiles = (R + kTileTokens - 1) / kTileTokens;
  CUtensorMap tk, tv;
  bool ready = false;
  if (workspace != nullptr) {
    const long long dim2 = static_cast<long long>(B) * params->num_heads_kv;
    s = encode_map(&tk, ring->k, params->head_dim, R, dim2, kTileTokens);
    if (s != WMTP_OK) return s;
    s = encode_map(&tv, ring->v, params->head_dim, R, dim2, kTileTokens);
    if (s != WMTP_OK) return s;
    ready = true;
  }
  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.ring_tags = ring->tags;
  a.ring_len = ring->len;
  a.ring_slots = R;
  a.sinks = params->sinks;
  a.window = params->window;
  a.status = status_word;
  return run_attention<true>(params, B, 1, q, &tk, &tv, a, max_tiles, out, out_fp32, lse_out, workspace,
                             workspace_bytes, static_cast<cudaStream_t>(stream), ready);
}

wmtp_status wmtp_ring_append(const wmtp_params* params, const wmtp_ring* ring, const int32_t* truncate_to,
                             const int32_t* n_new, const void* k_new, const void* v_new, int32_t max_new,
                             int32_t speculative, int32_t* status_word, void* stream) {
  wmtp_status s = check_ring(params, ring);
  if (s != WMTP_OK) return s;
  if (max_new < 0) return WMTP_ERR_INVALID_ARG;
  if (max_new > 0 && (n_new == nullptr || k_new == nullptr || v_new == nullptr)) return WMTP_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return WMTP_ERR_INVALID_ARG;
  if (speculative && params->gamma_max == 0 && max_new > 0) return WMTP_ERR_INVALID_ARG;
  if (ring->batch == 0) return WMTP_OK;
  RingArgs a = ring_args(params, ring);
  return launch_plain(true, ring_append_kernel, dim3(ring->batch), dim3(kRingThreads), static_cast<cudaStream_t>(stream),
                      a, truncate_to, n_new, static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                      max_new, speculative ? 1 : 0, status_word);
}

wmtp_status wmtp_ring_reset(const wmtp_params* params, const wmtp_ring* ring, void* stream) {
  wmtp_status s = check_ring(params, ring);
  if (s != WMTP_OK) return s;
  if (ring->batch == 0) return WMTP_OK;
  RingArgs a = ring_args(params, ring);
  return launch_plain(false, ring_reset_kernel, dim3(256), dim3(256), static_cast<cudaStream_t>(stream), a);
}

wmtp_status wmtp_splitkv_combine(int32_t rows, int32_t head_dim, int32_t nsplit, const float* part_o,
                                 const float* part_lse, void* out, int32_t out_fp32, float* lse_out,
                                 void* stream) {
  if (rows < 0 || nsplit <= 0) return WMTP_ERR_INVALID_ARG;
  if (head_dim <= 0 || head_dim % 4 != 0 || head_dim > 4096) return WMTP_ERR_UNSUPPORTED;
  if (rows > 0 && (part_o == nullptr || part_lse == nullptr || out == nullptr)) return WMTP_ERR_INVALID_ARG;
  if (!aligned(part_o, 16) || !aligned(out, 16)) return WMTP_ERR_INVALID_ARG;
  return launch_combine(rows, head_dim, nsplit, part_o, part_lse, out, out_fp32, lse_out,
                        static_cast<cudaStream_t>(stream), false);
}

wmtp_status wmtp_paged_write(const wmtp_params* params, int32_t batch, const wmtp_paged_kv* kv,
                             const int32_t* pos0, int32_t n_new, const void* k_new, const void* v_new,
                             int32_t* status_word, void* stream) {
  if (params == nullptr || kv == nullptr || batch < 0 || n_new < 0) return WMTP_ERR_INVALID_ARG;
  if (params->num_heads_kv <= 0 || !supported_page(params->page_size)) return WMTP_ERR_UNSUPPORTED;
  if (params->head_dim <= 0 || params->head_dim % 8 != 0) return WMTP_ERR_UNSUPPORTED;
  if (batch == 0 || n_new == 0) return WMTP_OK;
  if (batch > kMaxGridYZ) return WMTP_ERR_UNSUPPORTED;
  if (kv->k_pool == nullptr || kv->v_pool == nullptr || kv->page_table == nullptr || pos0 == nullptr ||
      k_new == nullptr || v_new == nullptr)
    return WMTP_ERR_INVALID_ARG;
  if (!aligned(kv->k_pool, 16) || !aligned(kv->v_pool, 16) || !aligned(k_new, 16) || !aligned(v_new, 16))
    return WMTP_ERR_INVALID_ARG;
  return launch_plain(true, paged_write_kernel, dim3(n_new, batch), dim3(128), static_cast<cudaStream_t>(stream),
                      static_cast<uint4*>(kv->k_pool), static_cast<uint4*>(kv->v_pool), kv->num_pages,
                      kv->page_table, kv->max_pages, params->page_size, params->num_heads_kv, params->head_dim,
                      pos0, n_new, static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                      status_word, static_cast<const int32_t*>(nullptr));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of wmtp_draft_attn_full.
//
// Some callers cannot hand this library a workspace: runtimes that plan every
// device allocation up front and forbid new ones once serving starts, and
// plugin hosts whose kernel interface passes only inputs and outputs.  For
// them the split-KV partials live in the fixed array below instead of a
// caller-provided buffer.  Every GPU that loads this library holds the array
// until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t wmtp_noalloc_scratch[WMTP_NOALLOC_SCRATCH_BYTES];

namespace wmtp {
namespace {

// Device address of the array on each device.  In host code the array's name
// is only a host-side stand-in, so the real address is fetched once per
// device, with that device current, and passed to the kernels.
// Only a successful lookup is kept; a failed one (for example inside a stream
// capture) clears its error from this library's runtime state and is retried
// by the next call.
std::atomic<void*> g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

void* noalloc_scratch(int dev) {
  void* ptr = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (ptr != nullptr) return ptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ptr = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
  if (ptr != nullptr) return ptr;
  if (cudaGetSymbolAddress(&ptr, wmtp_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
  return ptr;
}

}  // namespace
}  // namespace wmtp

extern "C" wmtp_status wmtp_draft_attn_full_noalloc(const wmtp_params* params, int32_t batch, const void* q,
                                                    const wmtp_paged_kv* kv, void* out, int32_t out_fp32,
                                                    float* lse_out, int32_t* status_word, void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WMTP_ERR_CUDA;
  void* scratch = noalloc_scratch(dev);
  if (scratch == nullptr) return WMTP_ERR_CUDA;
  size_t need = 0;
  wmtp_status s = paged_attention(params, batch, 1, q, kv, out, out_fp32, lse_out, nullptr, &need,
                                  status_word, stream);
  if (s != WMTP_OK) return s;
  if (need > static_cast<size_t>(WMTP_NOALLOC_SCRATCH_BYTES)) return WMTP_ERR_WORKSPACE;
  if (batch == 0) return WMTP_OK;
  size_t have = WMTP_NOALLOC_SCRATCH_BYTES;
  return paged_attention(params, batch, 1, q, kv, out, out_fp32, lse_out, scratch, &have, status_word,
                         stream);
}

// Log-sum-exp merge of split-KV partial attention results.
//
// Not on the pages: the standard identity behind split-KV ("flash-decoding")
// decode attention.  With m = max_s lse_s and w_s = e^(lse_s - m):
//   o = sum_s w_s o_s / sum_s w_s,   lse = m + ln sum_s w_s.
// Splits with lse = -inf (no attended keys) get weight 0; a row whose splits
// are all empty yields o = 0, lse = -inf.
//
// Layout of the work: CTA = (row, 128-column block).  Each of the 8 warps
// takes every 8th split; a lane owns 4 consecutive columns (one float4 per
// split), so a warp reads 512 contiguous bytes per split and the 8 warps keep
// many independent loads in flight.  Warp partial sums meet in shared memory.
//
// The kernel is launched as a programmatic dependent of the decode kernel:
// it may start while the decode kernel drains and waits (griddepcontrol.wait)
// until the partials are complete and visible.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace wmtp {

constexpr int kCombineWarps = 8;
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kCombineCols = 128;  // columns per CTA (32 lanes x float4)

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <bool OUT_F32>
__global__ void __launch_bounds__(kCombineThreads)
    splitkv_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                           int nsplit, int D, void* __restrict__ out, float* __restrict__ lse_out) {
  __shared__ float4 s_acc[kCombineWarps][32];
  __shared__ float s_den[kCombineWarps];
  grid_dependency_wait();

  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int col = blockIdx.y * kCombineCols + lane * 4;
  const float* pl = part_lse + static_cast<size_t>(row) * nsplit;

  // row maximum of the split log-sum-exps (every warp computes it)
  float m = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) m = fmaxf(m, pl[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (m != -INFINITY) {
    const float* po = part_o + static_cast<size_t>(row) * nsplit * D + col;
    const bool active = col < D;
    int s = warp;
    // two splits per iteration keep two independent loads in flight per lane
    for (; s + kCombineWarps < nsplit; s += 2 * kCombineWarps) {
      const float l0 = pl[s];
      const float l1 = pl[s + kCombineWarps];
      float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
      if (active) {
        v0 = *reinterpret_cast<const float4*>(po + static_cast<size_t>(s) * D);
        v1 = *reinterpret_cast<const float4*>(po + static_cast<size_t>(s + kCombineWarps) * D);
      }
      const float w0 = (l0 == -INFINITY) ? 0.f : expf(l0 - m);
      const float w1 = (l1 == -INFINITY) ? 0.f : expf(l1 - m);
      den += w0 + w1;
      acc.x += w0 * v0.x + w1 * v1.x;
      acc.y += w0 * v0.y + w1 * v1.y;
      acc.z += w0 * v0.z + w1 * v1.z;
      acc.w += w0 * v0.w + w1 * v1.w;
    }
    if (s < nsplit) {
      const float l0 = pl[s];
      const float w0 = (l0 == -INFINITY) ? 0.f : expf(l0 - m);
      den += w0;
      if (active) {
        const float4 v0 = *reinterpret_cast<const float4*>(po + static_cast<size_t>(s) * D);
        acc.x += w0 * v0.x;
        acc.y += w0 * v0.y;
        acc.z += w0 * v0.z;
        acc.w += w0 * v0.w;
      }
    }
  }
  s_acc[warp][lane] = acc;
  if (lane == 0) s_den[warp] = den;
  __syncthreads();
  if (warp != 0) return;
  float tot = 0.f;
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) {
    tot += s_den[w];
    const float4 a = s_acc[w][lane];
    sum.x += a.x;
    sum.y += a.y;
    sum.z += a.z;
    sum.w += a.w;
  }
  const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
  if (col < D) {
    const size_t o = static_cast<size_t>(row) * D + col;
    if (OUT_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(out) + o) =
          make_float4(sum.x * inv, sum.y * inv, sum.z * inv, sum.w * inv);
    } else {
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(out) + o;
      *reinterpret_cast<__nv_bfloat162*>(ob) = __floats2bfloat162_rn(sum.x * inv, sum.y * inv);
      *reinterpret_cast<__nv_bfloat162*>(ob + 2) = __floats2bfloat162_rn(sum.z * inv, sum.w * inv);
    }
  }
  if (lane == 0 && blockIdx.y == 0 && lse_out != nullptr)
    lse_out[row] = (tot > 0.f) ? m + logf(tot) : -INFINITY;
}

}  // namespace wmtp

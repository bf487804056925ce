// Log-sum-exp merge of split-KV partial attention results.
//
// Not on the pages: the standard identity behind split-KV ("flash-decoding")
// decode attention.  With m = max_s lse_s and w_s = e^(lse_s - m):
//   o = sum_s w_s o_s / sum_s w_s,   lse = m + ln sum_s w_s.
// Splits with lse = -inf (no attended keys) get weight 0; a row whose splits
// are all empty yields o = 0, lse = -inf.
//
// Layout of the work: CTA = (row, 128-column block).  Each of the 8 warps
// takes every 8th split, up to 12 of them per round with every load of the
// round (the split's lse and its 512 contiguous bytes of o: a lane owns 4
// consecutive columns) in flight at once, and keeps a running maximum of its
// own splits' lse.  The warps' (maximum, weight sum, weighted sum) meet in
// shared memory, so a row with up to 96 splits costs one memory round trip
// after the wait for the partials.
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
constexpr int kCombineBatch = 12;  // splits whose loads a warp issues together

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <bool OUT_F32>
__global__ void __launch_bounds__(kCombineThreads, 2)
    splitkv_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                           int nsplit, int D, void* __restrict__ out, float* __restrict__ lse_out) {
  __shared__ float4 s_acc[kCombineWarps][32];
  __shared__ float s_den[kCombineWarps];
  __shared__ float s_max[kCombineWarps];
  grid_dependency_wait();

  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int col = blockIdx.y * kCombineCols + lane * 4;
  const bool active = col < D;
  const float* pl = part_lse + static_cast<size_t>(row) * nsplit;
  const float* po = part_o + static_cast<size_t>(row) * nsplit * D + col;

  // this warp's splits w, w + 8, ...: a running maximum m of their lse and,
  // in units of e^m, the weight sum and the weighted sum of their o
  float m = -INFINITY;
  float den = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = warp; s0 < nsplit; s0 += kCombineWarps * kCombineBatch) {
    float4 v[kCombineBatch];
    float l[kCombineBatch];
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) {
      const int s = s0 + i * kCombineWarps;
      l[i] = s < nsplit ? pl[s] : -INFINITY;
      v[i] = (s < nsplit && active) ? *reinterpret_cast<const float4*>(po + static_cast<size_t>(s) * D)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mr = m;
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) mr = fmaxf(mr, l[i]);
    if (mr == -INFINITY) continue;  // every split so far empty
    const float c = (m == -INFINITY) ? 0.f : expf(m - mr);
    den *= c;
    acc.x *= c;
    acc.y *= c;
    acc.z *= c;
    acc.w *= c;
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) {
      const float w = (l[i] == -INFINITY) ? 0.f : expf(l[i] - mr);
      den += w;
      acc.x += w * v[i].x;
      acc.y += w * v[i].y;
      acc.z += w * v[i].z;
      acc.w += w * v[i].w;
    }
    m = mr;
  }
  s_acc[warp][lane] = acc;
  if (lane == 0) {
    s_den[warp] = den;
    s_max[warp] = m;
  }
  __syncthreads();
  if (warp != 0) return;
  float mt = -INFINITY;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) mt = fmaxf(mt, s_max[w]);
  float tot = 0.f;
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mt != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
      const float c = (s_max[w] == -INFINITY) ? 0.f : expf(s_max[w] - mt);
      tot += c * s_den[w];
      const float4 a = s_acc[w][lane];
      sum.x += c * a.x;
      sum.y += c * a.y;
      sum.z += c * a.z;
      sum.w += c * a.w;
    }
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
    lse_out[row] = (tot > 0.f) ? mt + logf(tot) : -INFINITY;
}

}  // namespace wmtp

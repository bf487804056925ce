// Log-sum-exp merge of split-KV partial attention results.
//
// Not on the pages: the standard identity behind split-KV ("flash-decoding")
// decode attention.  With m = max_s lse_s and w_s = e^(lse_s - m):
//   o = sum_s w_s o_s / sum_s w_s,   lse = m + ln sum_s w_s.
// Splits with lse = -inf (no attended keys) get weight 0; a row whose splits
// are all empty yields o = 0, lse = -inf.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace wmtp {

constexpr int kCombineThreads = 64;

// One CTA per output row; each thread owns 4 consecutive columns (float4).
template <bool OUT_F32>
__global__ void __launch_bounds__(kCombineThreads)
    splitkv_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                           int nsplit, int D, void* __restrict__ out, float* __restrict__ lse_out) {
  const int row = blockIdx.x;
  const float* pl = part_lse + static_cast<size_t>(row) * nsplit;
  float m = -INFINITY;
  for (int s = 0; s < nsplit; ++s) m = fmaxf(m, pl[s]);
  const int d = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (m != -INFINITY) {
    const float* po = part_o + static_cast<size_t>(row) * nsplit * D + d;
    for (int s = 0; s < nsplit; ++s) {
      const float ls = pl[s];
      if (ls == -INFINITY) continue;
      const float w = expf(ls - m);
      den += w;
      if (d < D) {
        const float4 v = *reinterpret_cast<const float4*>(po + static_cast<size_t>(s) * D);
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
      }
    }
  }
  const float inv = (den > 0.f) ? 1.f / den : 0.f;
  if (d < D) {
    const size_t o = static_cast<size_t>(row) * D + d;
    if (OUT_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(out) + o) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    } else {
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(out) + o;
      __nv_bfloat162 v01 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      __nv_bfloat162 v23 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      *reinterpret_cast<__nv_bfloat162*>(ob) = v01;
      *reinterpret_cast<__nv_bfloat162*>(ob + 2) = v23;
    }
  }
  if (threadIdx.x == 0 && lse_out != nullptr)
    lse_out[row] = (den > 0.f) ? m + logf(den) : -INFINITY;
}

}  // namespace wmtp

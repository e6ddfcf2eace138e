// merge_lse.cuh -- combination of S partial attention results by their
// log-sum-exp.  Each part s of a row attended a disjoint key set K_s and
// holds o_s (normalised over K_s) and lse_s = log sum_{j in K_s} e^{s_j};
// over the union, lse = log sum_s e^{lse_s} and o = sum_s e^{lse_s - lse} o_s.
// This is the correct version of the per-page sum in the paged_attention
// method of the "Real-time inference optimisation" page (llmapi-app.pages.dev),
// and the same algebra as the online-softmax update in that page's "Flash
// Attention optimisation" section.
//
// One warp per row; lanes cover D with vector loads; HBM-bound (reads S*D*4 +
// S*4 bytes and writes D*2 + 4 bytes per row).
#pragma once

#include "frt_device.cuh"

namespace frt {

constexpr int kMergeWarps = 8;

template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32)
merge_lse_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int S,
                 long long rows, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  constexpr int kPer = D / 32;   // elements per lane (2 or 4)
  const long long row = (long long)blockIdx.x * kMergeWarps + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  griddep_wait();   // the parts may come from the kernel before this one
  griddep_launch_dependents();
  if (row >= rows) return;
  constexpr float kLog2e = 1.4426950408889634f;

  float m = -INFINITY;
  for (int s = 0; s < S; ++s) m = fmaxf(m, lse_parts[(size_t)s * rows + row]);
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float ls = lse_parts[(size_t)s * rows + row];
      if (ls == -INFINITY) continue;        // empty part: weight exactly 0
      const float w = fast_exp2((ls - m) * kLog2e);
      wsum += w;
      const float* src = o_parts + ((size_t)s * rows + row) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] += w * v.x; acc[1] += w * v.y; acc[2] += w * v.z; acc[3] += w * v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] += w * v.x; acc[1] += w * v.y;
      }
    }
  }
  const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = o + (size_t)row * D + lane * kPer;
#pragma unroll
  for (int i = 0; i < kPer; i += 2) {
    *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
  }
  if (lse != nullptr && lane == 0)
    lse[row] = (wsum > 0.f) ? m + logf(wsum) : -INFINITY;
}

}  // namespace frt

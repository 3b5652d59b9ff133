// merge.cuh — combine attention results over disjoint blocks of keys into the
// result over their union.
//
// Each block s holds, per query row, its normalised output O_s (fp32) and its
// natural-log LSE_s (-inf for a row that saw no key of the block). Since
// exp(LSE_s) is block s's softmax denominator, with M = max_s LSE_s and
// w_s = exp(LSE_s - M):
//   O = sum_s w_s O_s / sum_s w_s,   LSE = M + ln sum_s w_s.
// This is the online-softmax rescale of the "Flash Attention" glossary page
// (second paragraph: partial results accumulated with the numerically stable
// online softmax) applied to whole partial results computed in parallel, as
// splitting the keys over several CTAs, or over several devices (same page,
// fourth paragraph: ring attention), needs.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100.cuh"

namespace fa {

constexpr int kMergeThreads = 256;

// One warp per row; lane l holds columns l*PER .. l*PER+PER-1. Reads
// n_part * D * 4 bytes and writes D * 2 (+4) bytes per row: HBM-bound.
template <int D>
__global__ void __launch_bounds__(kMergeThreads)
lse_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, int n_part, int64_t rows,
                 __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  constexpr int PER = D / 32;  // 2, 4 or 8 floats per lane
  static_assert(PER == 2 || PER == 4 || PER == 8, "head dim");
  constexpr float kLog2e = 1.4426950408889634f;
  const int lane = static_cast<int>(threadIdx.x & 31u);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kMergeThreads / 32);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (kMergeThreads / 32) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    float m = -INFINITY;
    for (int s = lane; s < n_part; s += 32) m = fmaxf(m, __ldg(lse_part + static_cast<int64_t>(s) * rows + r));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float wsum = 0.f;
    if (m != -INFINITY) {
#pragma unroll 4
      for (int s = 0; s < n_part; ++s) {
        const int64_t pr = static_cast<int64_t>(s) * rows + r;
        const float w = exp2f((__ldg(lse_part + pr) - m) * kLog2e);  // 0 for an empty block
        const float* src = o_part + pr * D + lane * PER;
        float val[PER];
        if constexpr (PER == 2) {
          const float2 t = __ldg(reinterpret_cast<const float2*>(src));
          val[0] = t.x; val[1] = t.y;
        } else {
#pragma unroll
          for (int i = 0; i < PER; i += 4) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(src + i));
            val[i] = t.x; val[i + 1] = t.y; val[i + 2] = t.z; val[i + 3] = t.w;
          }
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, val[i], acc[i]);
        wsum += w;
      }
    }
    const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
    uint32_t packed[PER / 2];
#pragma unroll
    for (int i = 0; i < PER / 2; ++i) packed[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    __nv_bfloat16* dst = o + r * D + lane * PER;
    if constexpr (PER == 2) {
      *reinterpret_cast<uint32_t*>(dst) = packed[0];
    } else if constexpr (PER == 4) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    if (lse != nullptr && lane == 0) lse[r] = m == -INFINITY ? -INFINITY : m + logf(wsum);
  }
}

}  // namespace fa

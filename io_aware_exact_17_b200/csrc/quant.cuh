// quant.cuh — Hadamard rotate + per-tensor e4m3 quantisation for the FP8 path.
//
// "FlashAttention-3 (PT)", section "Inovações técnicas", subsection 3 ("Baixa
// precisão (FP8)"): before attention, Q and K are multiplied by a random
// orthogonal (Hadamard) matrix, which spreads outlier coordinates over all
// coordinates; then they are quantised to FP8; the product Q Kᵀ is unchanged by
// the rotation. Here the rotation is x' = x D H_d / sqrt(d) along the head
// dimension (D = optional diagonal of +-1 signs, H_d the Sylvester Hadamard
// matrix), applied as log2(d) butterfly stages in registers and warp shuffles,
// never as a matrix. One scale per tensor: descale = amax|x'| / 448, codes =
// RNE-satfinite e4m3(x' * 448 / amax).
//
// Two streaming passes over the bf16 input, both HBM/L2-bound:
//   pass 1: rotate, reduce |x'| to one block max, atomicMax into a scratch word;
//   pass 2: rotate again, scale, convert, store 8 codes (8 bytes) per thread.
// A tensor of up to ~60 MB stays in the 126 MB L2 between the passes, so the
// second read mostly hits L2.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100.cuh"

namespace fa {

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;  // independent 16-byte loads in flight per thread

template <int D>
struct QuantCfg {
  static constexpr int L = D / 8;               // threads per row, 8 elements (16 B) each
  static constexpr int RPW = 32 / L;            // rows per warp per step
  static constexpr int ROWS_PER_STEP = RPW * kQuantUnroll;
  static_assert(D == 64 || D == 128 || D == 256, "head dim");
};

__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// In place: v holds elements [8*lr, 8*lr+8) of one row; after the call it holds
// the same elements of (v * signs) H_D / sqrt(D). Every lane of the warp must call.
template <int D>
__device__ __forceinline__ void hadamard_rotate(float (&v)[8], int lr, const float* signs) {
  if (signs != nullptr) {
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(signs + 8 * lr));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(signs + 8 * lr + 4));
    v[0] *= s0.x; v[1] *= s0.y; v[2] *= s0.z; v[3] *= s0.w;
    v[4] *= s1.x; v[5] *= s1.y; v[6] *= s1.z; v[7] *= s1.w;
  }
  // Butterflies over index bits 0..2 (inside the thread).
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if ((e & h) == 0) {
        const float a = v[e], b = v[e + h];
        v[e] = a + b;
        v[e + h] = a - b;
      }
    }
  }
  // Butterflies over index bits 3.. (across the L lanes of the row).
#pragma unroll
  for (int m = 1; m < D / 8; m <<= 1) {
    const bool upper = (lr & m) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, v[e], m);
      v[e] = upper ? other - v[e] : v[e] + other;
    }
  }
  constexpr float inv_sqrt_d = D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] *= inv_sqrt_d;
}

// Pass 1: amax of the (rotated) tensor into *amax_bits (a non-negative float's
// bit pattern orders like an unsigned integer, so atomicMax on the bits works).
template <int D, bool ROT>
__global__ void __launch_bounds__(kQuantThreads)
quant_amax_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, const float* __restrict__ signs,
                  unsigned int* amax_bits) {
  using C = QuantCfg<D>;
  const int lane = threadIdx.x & 31;
  const int lr = lane % C::L, sub = lane / C::L;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kQuantThreads) >> 5;
  float m = 0.f;
  for (int64_t w = warp_g; w * C::ROWS_PER_STEP < rows; w += nwarps) {
    float v[kQuantUnroll][8];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t row = w * C::ROWS_PER_STEP + u * C::RPW + sub;
      if (row < rows) {
        load_bf16x8(x + row * D + 8 * lr, v[u]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      if (ROT) hadamard_rotate<D>(v[u], lr, signs);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[u][e]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float warp_max[kQuantThreads / 32];
  if (lane == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = warp_max[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) b = fmaxf(b, warp_max[i]);
    atomicMax(amax_bits, __float_as_uint(b));
  }
}

// Pass 2: codes = e4m3(x' * 448 / amax); block 0 also writes descale = amax / 448
// (1 when the tensor is all zeros).
template <int D, bool ROT>
__global__ void __launch_bounds__(kQuantThreads)
quant_apply_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out, int64_t rows,
                   const float* __restrict__ signs, const unsigned int* amax_bits, float* descale_out) {
  using C = QuantCfg<D>;
  const float amax = __uint_as_float(*amax_bits);
  const float scale = amax > 0.f ? 448.0f / amax : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *descale_out = amax > 0.f ? amax / 448.0f : 1.0f;
  const int lane = threadIdx.x & 31;
  const int lr = lane % C::L, sub = lane / C::L;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kQuantThreads) >> 5;
  for (int64_t w = warp_g; w * C::ROWS_PER_STEP < rows; w += nwarps) {
    float v[kQuantUnroll][8];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t row = w * C::ROWS_PER_STEP + u * C::RPW + sub;
      if (row < rows) {
        load_bf16x8(x + row * D + 8 * lr, v[u]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      if (ROT) hadamard_rotate<D>(v[u], lr, signs);
      const int64_t row = w * C::ROWS_PER_STEP + u * C::RPW + sub;
      uint32_t lo = static_cast<uint32_t>(pack_e4m3x2(v[u][0] * scale, v[u][1] * scale)) |
                    (static_cast<uint32_t>(pack_e4m3x2(v[u][2] * scale, v[u][3] * scale)) << 16);
      uint32_t hi = static_cast<uint32_t>(pack_e4m3x2(v[u][4] * scale, v[u][5] * scale)) |
                    (static_cast<uint32_t>(pack_e4m3x2(v[u][6] * scale, v[u][7] * scale)) << 16);
      if (row < rows) *reinterpret_cast<uint2*>(out + row * D + 8 * lr) = make_uint2(lo, hi);
    }
  }
}

}  // namespace fa

// quant_t.cuh — V's e4m3 codes with one scale per tensor, written transposed.
//
// "FlashAttention-3 (PT)", section "Inovações técnicas", subsection 3: the FP8
// path quantises its operands to 8-bit floating point with a scale; the pages
// rotate only Q and K and say nothing of V's layout. Reading used here: V is
// quantised without rotation, with one scale per tensor (amax over the tensor,
// descale = amax / 448, codes e4m3(fl(v * (448 / amax))) rounded to nearest even
// and saturated, the same arithmetic as the unrotated quantiser), and its codes
// are laid out [BH][d][N], so that an e4m3 product P V reads V with the keys
// along the contiguous dimension.
//
// Two launches on the caller's stream, both HBM-bound:
//   quant_t_amax_kernel: max |v| over the tensor, four 16-byte loads per thread
//     and loop step, each block's maximum folded into one word with atomicMax
//     on the bit pattern (non-negative floats order like their bits);
//   quant_t_kernel<D>: one CTA per 64 positions of a head: the tile's D x 64
//     codes go through shared memory (row stride 65 bytes, so the transposing
//     byte stores of a warp fall in distinct banks) and leave as D rows of up to
//     64 contiguous codes.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100.cuh"

namespace fa {

__global__ void __launch_bounds__(256) quant_t_amax_kernel(const uint4* __restrict__ x, int64_t n16,
                                                           unsigned int* amax_word) {
  float m = 0.f;
  // four independent 16-byte loads in flight per thread and step
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < n16; i0 += 4 * stride) {
    uint4 u[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int64_t i = i0 + t * stride;
      u[t] = i < n16 ? x[i] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t w[4] = {u[t].x, u[t].y, u[t].z, u[t].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // one atomic per block: the word's atomics are serialised at its L2 slice
  __shared__ float warp_max[8];
  if ((threadIdx.x & 31u) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = warp_max[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) b = fmaxf(b, warp_max[w]);
    atomicMax(amax_word, __float_as_uint(b));
  }
}

constexpr int kQuantTPos = 64;               // positions per CTA
constexpr int kQuantTStride = kQuantTPos + 1;  // shared-memory row stride (bytes)

template <int D>
__global__ void __launch_bounds__(256) quant_t_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out,
                                                      int N, const unsigned int* amax_word, float* descale_out) {
  __shared__ uint8_t sT[D * kQuantTStride];
  const float amax = __uint_as_float(*amax_word);
  const float sc = amax > 0.f ? 448.0f / amax : 1.0f;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *descale_out = amax > 0.f ? amax / 448.0f : 1.0f;
  const int bh = static_cast<int>(blockIdx.y);
  const int n0 = static_cast<int>(blockIdx.x) * kQuantTPos;
  const int valid = min(kQuantTPos, N - n0);
  const __nv_bfloat16* xh = x + (static_cast<size_t>(bh) * N + n0) * D;
  // 16-byte chunks of the tile: chunk k is row k / (D / 8), columns 8 (k % (D / 8)) ..
  constexpr int CPR = D / 8;
  constexpr int PER = kQuantTPos * CPR / 256;  // chunks per thread: 2, 4 or 8, all loaded before any is used
  uint4 u[PER];
#pragma unroll
  for (int t = 0; t < PER; ++t) {
    const int k = static_cast<int>(threadIdx.x) + 256 * t;
    const int row = k / CPR, c8 = (k % CPR) * 8;
    u[t] = row < valid ? *reinterpret_cast<const uint4*>(xh + static_cast<size_t>(row) * D + c8)
                       : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int t = 0; t < PER; ++t) {
    const int k = static_cast<int>(threadIdx.x) + 256 * t;
    const int row = k / CPR, c8 = (k % CPR) * 8;
    const uint32_t w[4] = {u[t].x, u[t].y, u[t].z, u[t].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      const uint16_t q = pack_e4m3x2(f.x * sc, f.y * sc);
      sT[(c8 + 2 * e) * kQuantTStride + row] = static_cast<uint8_t>(q & 0xffu);
      sT[(c8 + 2 * e + 1) * kQuantTStride + row] = static_cast<uint8_t>(q >> 8);
    }
  }
  __syncthreads();
  // D rows of `valid` codes: row c goes to out[bh][c][n0 ..]. Four codes per
  // lane and 16 lanes per row when the rows start 4-byte aligned and the tile is
  // whole, else one code per lane.
  uint8_t* oh = out + static_cast<size_t>(bh) * D * N + n0;
  const int warp = static_cast<int>(threadIdx.x >> 5), lane = static_cast<int>(threadIdx.x & 31u);
  if ((N & 3) == 0 && valid == kQuantTPos) {
#pragma unroll 1
    for (int c = 2 * warp + (lane >> 4); c < D; c += 16) {
      const int j = 4 * (lane & 15);
      const uint8_t* s = sT + c * kQuantTStride + j;
      const uint32_t v = static_cast<uint32_t>(s[0]) | (static_cast<uint32_t>(s[1]) << 8) |
                         (static_cast<uint32_t>(s[2]) << 16) | (static_cast<uint32_t>(s[3]) << 24);
      *reinterpret_cast<uint32_t*>(oh + static_cast<size_t>(c) * N + j) = v;
    }
  } else {
#pragma unroll 1
    for (int c = warp; c < D; c += 8)
      for (int j = lane; j < valid; j += 32) oh[static_cast<size_t>(c) * N + j] = sT[c * kQuantTStride + j];
  }
}

}  // namespace fa

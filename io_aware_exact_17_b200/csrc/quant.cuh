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
//   pass 2: rotate again, scale, convert, store the codes.
// A tensor of up to ~60 MB stays in the 126 MB L2 between the passes, so the
// second read mostly hits L2. quant_fused_kernel runs both passes in one
// cooperative launch, for up to 8 tensors at once (each with its own scale);
// quant_amax_kernel + quant_apply_kernel are the two-launch form (used where
// the scratch is the library's own static array). quant_block_kernel (end of
// the file) takes one scale per 128-row block of a head, in one pass.
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

namespace fa {

// ---------------------------------------------------------------------------
// One-launch variant: both passes in one cooperative kernel with a grid-wide
// barrier between them (all blocks are co-resident, which the cooperative
// launch guarantees), 32 elements per thread (fewer cross-lane butterfly
// stages), and the second pass re-reading the tensor while it is still in L2.
// The butterfly stages run in the same order (index bits 0, 1, 2, ...) with
// the same operands as hadamard_rotate, so the codes are bit-identical to the
// two-kernel path.
// ---------------------------------------------------------------------------
constexpr int kFusedThreads = 256;

template <int D>
struct FusedCfg {
  static constexpr int E = 32;          // elements per thread (four 16-byte chunks)
  static constexpr int L = D / E;       // threads per row
  static constexpr int RPW = 32 / L;    // rows per warp per step
  static_assert(D == 64 || D == 128 || D == 256, "head dim");
};

// Thread lr of a row holds the four 16-byte chunks lr, lr+L, lr+2L, lr+3L (8
// elements each) of the row: v[8*q + i] is element 8*(lr + L*q) + i. A warp's
// load instruction q then covers L consecutive chunks of each of its rows.
template <int D>
__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* row, int lr, float (&v)[32]) {
  constexpr int L = D / 32;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + lr + L * q);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// In place: (v * signs) H_D / sqrt(D) for the elements this thread holds (the
// layout of load_bf16x32). Butterflies run over index bits 0, 1, 2 (inside a
// chunk), then the log2(L) bits of the chunk's lane (warp shuffles), then the two
// bits of q (inside the thread): the same stage order as hadamard_rotate.
// Every lane of the warp must call.
template <int D>
__device__ __forceinline__ void hadamard_rotate32(float (&v)[32], int lr, const float* signs) {
  constexpr int L = D / 32;
  // Stages over index bits 1 and up pair neighbouring elements (v[2i], v[2i+1])
  // with another such pair, so they run as packed f32x2 operations: the same
  // two IEEE additions (or subtractions, multiplications) per instruction, hence
  // the same results as the scalar form.
  uint64_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = f2_pack(v[2 * i], v[2 * i + 1]);
  if (signs != nullptr) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(signs + 8 * (lr + L * q)));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(signs + 8 * (lr + L * q) + 4));
      w[4 * q + 0] = f2_mul(w[4 * q + 0], f2_pack(s0.x, s0.y));
      w[4 * q + 1] = f2_mul(w[4 * q + 1], f2_pack(s0.z, s0.w));
      w[4 * q + 2] = f2_mul(w[4 * q + 2], f2_pack(s1.x, s1.y));
      w[4 * q + 3] = f2_mul(w[4 * q + 3], f2_pack(s1.z, s1.w));
    }
  }
  // index bit 0: inside each pair (scalar)
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float a, b;
    f2_unpack(w[i], a, b);
    w[i] = f2_pack(a + b, a - b);
  }
  // index bits 1, 2: pair i with pair i + h/2 inside each 8-element chunk
#pragma unroll
  for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        const uint64_t a = w[i], b = w[i + h];
        w[i] = f2_add(a, b);
        w[i + h] = f2_sub(a, b);
      }
    }
  }
  // index bits 3 .. 2+log2(L): across the L lanes of the row. Lower lane:
  // v + other; upper lane: other - v; both as one fma with +-1 (exact: the same
  // single rounding as the add or subtract).
#pragma unroll
  for (int m = 1; m < L; m <<= 1) {
    const float sg = (lr & m) != 0 ? -1.0f : 1.0f;
    const uint64_t sgn = f2_pack(sg, sg);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float a, b;
      f2_unpack(w[i], a, b);
      const float oa = __shfl_xor_sync(0xffffffffu, a, m);
      const float ob = __shfl_xor_sync(0xffffffffu, b, m);
      w[i] = f2_fma(w[i], sgn, f2_pack(oa, ob));
    }
  }
  // the two bits of q: pair i with pair i + 4 and i + 8
#pragma unroll
  for (int h = 4; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        const uint64_t a = w[i], b = w[i + h];
        w[i] = f2_add(a, b);
        w[i + h] = f2_sub(a, b);
      }
    }
  }
  constexpr float inv_sqrt_d = D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
  const uint64_t isd = f2_pack(inv_sqrt_d, inv_sqrt_d);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    w[i] = f2_mul(w[i], isd);
    f2_unpack(w[i], v[2 * i], v[2 * i + 1]);
  }
}

// Up to kQuantBatch tensors of one shape, rotated and quantised in one launch,
// each with its own scale.
constexpr int kQuantBatch = 8;
struct QuantBatch {
  const __nv_bfloat16* x[kQuantBatch];
  uint8_t* out[kQuantBatch];
  int n;
};

// ws[0 .. n-1]: amax bits of each tensor, ws[n]: arrival counter of the grid
// barrier; all zero at launch. descale_out[i]: tensor i's descale.
template <int D, bool ROT>
__global__ void __launch_bounds__(kFusedThreads, 3)
quant_fused_kernel(const QuantBatch b, int64_t rows, const float* __restrict__ signs, unsigned int* ws,
                   float* descale_out) {
  DevStatus* st = &g_fa_status;
  using C = FusedCfg<D>;
  const int lane = threadIdx.x & 31;
  const int lr = lane % C::L, sub = lane / C::L;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * kFusedThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kFusedThreads) >> 5;
  __shared__ float warp_max[kFusedThreads / 32];
  __shared__ unsigned int amax_sh[kQuantBatch];
  // pass 1: amax of each rotated tensor
#pragma unroll 1
  for (int t = 0; t < b.n; ++t) {
    const __nv_bfloat16* x = b.x[t];
    float m = 0.f;
    for (int64_t w = warp_g; w * C::RPW < rows; w += nwarps) {
      const int64_t row = w * C::RPW + sub;
      float v[32];
      if (row < rows) {
        load_bf16x32<D>(x + row * D, lr, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
      }
      if (ROT) hadamard_rotate32<D>(v, lr, signs);
#pragma unroll
      for (int e = 0; e < 32; e += 2) m = fmax3(m, fabsf(v[e]), fabsf(v[e + 1]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      float bm = warp_max[0];
#pragma unroll
      for (int i = 1; i < kFusedThreads / 32; ++i) bm = fmaxf(bm, warp_max[i]);
      atomicMax(&ws[t], __float_as_uint(bm));
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    // Grid-wide barrier: every block is resident (cooperative launch). The wait
    // is bounded; if it runs out the status word records it and the block goes on.
    __threadfence();
    atomicAdd(&ws[b.n], 1u);
    const unsigned long long t0 = globaltimer_ns();
    unsigned int arrived;
    for (;;) {
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(arrived) : "l"(ws + b.n) : "memory");
      if (arrived >= gridDim.x) break;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        if (atomicCAS(&st->code, 0u, 5u) == 0u) {
          st->site = 60;
          st->block = blockIdx.x;
        }
        break;
      }
      __nanosleep(64);
    }
    for (int t = 0; t < b.n; ++t) {
      unsigned int a;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(a) : "l"(ws + t) : "memory");
      amax_sh[t] = a;
    }
  }
  __syncthreads();
  // pass 2: quantise (each tensor is re-read, mostly from L2)
#pragma unroll 1
  for (int t = 0; t < b.n; ++t) {
    const __nv_bfloat16* x = b.x[t];
    uint8_t* out = b.out[t];
    const float amax = __uint_as_float(amax_sh[t]);
    const float scale = amax > 0.f ? 448.0f / amax : 1.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) descale_out[t] = amax > 0.f ? amax / 448.0f : 1.0f;
    for (int64_t w = warp_g; w * C::RPW < rows; w += nwarps) {
      const int64_t row = w * C::RPW + sub;
      float v[32];
      if (row < rows) {
        load_bf16x32<D>(x + row * D, lr, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
      }
      if (ROT) hadamard_rotate32<D>(v, lr, signs);
      uint32_t q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        q[i] = static_cast<uint32_t>(pack_e4m3x2(v[4 * i] * scale, v[4 * i + 1] * scale)) |
               (static_cast<uint32_t>(pack_e4m3x2(v[4 * i + 2] * scale, v[4 * i + 3] * scale)) << 16);
      if (row < rows) {
        // chunk c of the row (8 codes, 8 bytes) goes to out[row*D + 8c]
        uint2* dst = reinterpret_cast<uint2*>(out + row * D);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) dst[lr + C::L * qq] = make_uint2(q[2 * qq], q[2 * qq + 1]);
      }
    }
  }
}

}  // namespace fa

namespace fa {

// ---------------------------------------------------------------------------
// Per-block scales: one CTA per block of 128 consecutive rows of a head. The
// block's rotated values stay in registers between its amax and its codes, so
// the input is read once, with no second pass and no grid-wide barrier (every
// scale depends on one CTA's data only). The rotation is hadamard_rotate32's.
// ---------------------------------------------------------------------------
constexpr int kBlockRows = 128;
constexpr int kBlockThreads = 256;

template <int D, bool ROT>
__global__ void __launch_bounds__(kBlockThreads)
quant_block_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ out, int N, int nb,
                   const float* __restrict__ signs, float* __restrict__ descales) {
  using C = FusedCfg<D>;
  constexpr int WARPS = kBlockThreads / 32;
  constexpr int STEPS = kBlockRows / (WARPS * C::RPW);  // rows of a warp / rows per warp-step
  static_assert(STEPS * WARPS * C::RPW == kBlockRows, "block rows");
  const int bh = blockIdx.x / nb, blk = blockIdx.x % nb;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lr = lane % C::L, sub = lane / C::L;
  const int row0 = blk * kBlockRows;
  const __nv_bfloat16* xh = x + static_cast<int64_t>(bh) * N * D;
  uint8_t* oh = out + static_cast<int64_t>(bh) * N * D;
  float v[STEPS][32];
  float m = 0.f;
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int row = row0 + (s * WARPS + warp) * C::RPW + sub;
    if (row < N) {
      load_bf16x32<D>(xh + static_cast<int64_t>(row) * D, lr, v[s]);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[s][e] = 0.f;
    }
  }
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    if (ROT) hadamard_rotate32<D>(v[s], lr, signs);
#pragma unroll
    for (int e = 0; e < 32; e += 2) m = fmax3(m, fabsf(v[s][e]), fabsf(v[s][e + 1]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float warp_max[WARPS];
  if (lane == 0) warp_max[warp] = m;
  __syncthreads();
  float amax = warp_max[0];
#pragma unroll
  for (int i = 1; i < WARPS; ++i) amax = fmaxf(amax, warp_max[i]);
  const float scale = amax > 0.f ? 448.0f / amax : 1.0f;
  if (threadIdx.x == 0) descales[blockIdx.x] = amax > 0.f ? amax / 448.0f : 1.0f;
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int row = row0 + (s * WARPS + warp) * C::RPW + sub;
    uint32_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      q[i] = static_cast<uint32_t>(pack_e4m3x2(v[s][4 * i] * scale, v[s][4 * i + 1] * scale)) |
             (static_cast<uint32_t>(pack_e4m3x2(v[s][4 * i + 2] * scale, v[s][4 * i + 3] * scale)) << 16);
    if (row < N) {
      uint2* dst = reinterpret_cast<uint2*>(oh + static_cast<int64_t>(row) * D);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) dst[lr + C::L * qq] = make_uint2(q[2 * qq], q[2 * qq + 1]);
    }
  }
}

}  // namespace fa

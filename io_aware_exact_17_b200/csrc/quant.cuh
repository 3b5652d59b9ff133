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
// Tensors of up to ~100 MB stay in the 126 MB L2 between the passes, so the
// second read mostly hits L2. quant_tma_kernel runs both passes in one
// cooperative launch, for up to 8 tensors at once (each with its own scale),
// with the input staged through shared memory by TMA; quant_amax_kernel +
// quant_apply_kernel are the two-launch form (used where the scratch is the
// library's own static array). quant_block_tma_kernel (end of the file) takes
// one scale per 128-row block of a head, in one pass.
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

// Up to kQuantBatch tensors of one shape, rotated and quantised in one launch,
// each with its own scale.
constexpr int kQuantBatch = 8;
struct QuantBatch {
  const __nv_bfloat16* x[kQuantBatch];
  uint8_t* out[kQuantBatch];
  int n;
};

// ---------------------------------------------------------------------------
// Per-tensor scales in one cooperative launch, with the input staged through
// shared memory by TMA (quant_tma_kernel).
//
// One CTA per SM. A producer warp streams blocks of RB rows of the tensors
// through a ring of stages (TMA, 128-byte swizzle), far enough ahead to keep
// HBM busy; 8 consumer warps take one stage at a time, each thread a whole row
// (d <= 128) or half a row (d = 256), so the butterfly stages of the rotation
// stay inside the thread (one cross-lane stage at d = 256) and a warp's sign
// loads are broadcasts. Pass 1 reduces |x'| per tensor; a bounded grid barrier
// publishes the amax words; pass 2 streams the same blocks again, in reverse
// order so that the most recently read ones, still in L2, come first, and
// writes the codes. The producer runs on into pass 2 while the consumers wait
// at the barrier.
//
// The butterflies run over index bits 0, 1, ... in increasing order with the
// same operations as hadamard_rotate, so the codes are bit-identical to the
// two-launch kernels'. Pass 1 takes the max before the
// 1/sqrt(d) factor and multiplies it once: fp32 rounding is monotonic, so
// max_i fl(|v_i| c) = fl(c max_i |v_i|).
// ---------------------------------------------------------------------------
// descale_out[0 .. n-1] = v (the descales of empty tensors).
__global__ void fill_f32_kernel(float* out, int n, float v) {
  if (static_cast<int>(threadIdx.x) < n) out[threadIdx.x] = v;
}

constexpr int kTmaQuantConsumers = 256;
constexpr int kTmaQuantStages = 3;

template <int D>
struct TmaQuantCfg {
  static constexpr int E = D < 128 ? D : 128;            // elements per thread
  static constexpr int W = E / 2;                        // packed pairs per thread
  static constexpr int TPR = D / E;                      // threads per row
  static constexpr int RB = kTmaQuantConsumers / TPR;    // rows per stage
  static constexpr int BOX_ROWS = RB < 256 ? RB : 256;   // TMA box height (at most 256)
  static constexpr int COLS = D / 64;                    // 128-byte columns per row
  static constexpr int STAGE = RB * D * 2;               // bytes per stage
  static constexpr int CONSUMER_WARPS = kTmaQuantConsumers / 32;
  static constexpr int THREADS = kTmaQuantConsumers + 32;  // + the producer warp
  static constexpr int SMEM = 1024 + kTmaQuantStages * STAGE;
  static_assert(D == 64 || D == 128 || D == 256, "head dim");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct QuantMaps {
  CUtensorMap x[kQuantBatch];  // tensor t as [rows][D] bf16, box (64, BOX_ROWS), 128-byte swizzle
  uint8_t* out[kQuantBatch];
  int n;
};

// In place: the thread's E consecutive elements e0 .. e0+E-1 of a row (w[i] =
// elements e0+2i, e0+2i+1) become the same elements of (x * signs) H_D,
// without the 1/sqrt(D) factor. At d = 256 the two threads of a row (lanes 8
// apart, part p = e0 / 128 = bit 3 of the lane) must call together.
template <int D, bool ROT>
__device__ __forceinline__ void rotate_part(uint64_t (&w)[TmaQuantCfg<D>::W], int p, const float* sgn) {
  constexpr int E = TmaQuantCfg<D>::E, W = TmaQuantCfg<D>::W;
  if (!ROT) return;
  if (sgn != nullptr) {
#pragma unroll
    for (int i = 0; i < W; i += 2) {
      const float4 s4 = *reinterpret_cast<const float4*>(sgn + E * p + 2 * i);
      w[i] = f2_mul(w[i], f2_pack(s4.x, s4.y));
      w[i + 1] = f2_mul(w[i + 1], f2_pack(s4.z, s4.w));
    }
  }
  // index bit 0: inside each pair
#pragma unroll
  for (int i = 0; i < W; ++i) {
    float a, b;
    f2_unpack(w[i], a, b);
    w[i] = f2_pack(a + b, a - b);
  }
  // index bits 1 .. log2(E) - 1: pair i with pair i + h
#pragma unroll
  for (int h = 1; h < W; h <<= 1) {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      if ((i & h) == 0) {
        const uint64_t a = w[i], b = w[i + h];
        w[i] = f2_add(a, b);
        w[i + h] = f2_sub(a, b);
      }
    }
  }
  // index bits log2(E) ..: across the TPR lanes of the row (lower part: v +
  // other, upper part: other - v, each one fma with +-1, i.e. one rounding)
#pragma unroll
  for (int m = 1; m < D / E; m <<= 1) {
    const float sg = (p & m) != 0 ? -1.0f : 1.0f;
    const uint64_t sgn2 = f2_pack(sg, sg);
#pragma unroll
    for (int i = 0; i < W; ++i) {
      float a, b;
      f2_unpack(w[i], a, b);
      const float oa = __shfl_xor_sync(0xffffffffu, a, 8 * m);
      const float ob = __shfl_xor_sync(0xffffffffu, b, 8 * m);
      w[i] = f2_fma(w[i], sgn2, f2_pack(oa, ob));
    }
  }
}

// Consumer side shared by the TMA-staged quantisers: the thread's row within a
// stage and its part of the row (E elements: p = 0 unless d = 256), and the
// reads of that part. Lane bits 0-2: row (low bits), then (d = 256) the part,
// higher bits: row (high bits). The 8 lanes of a shared-memory phase (one
// 16-byte load each) read the same chunk j of one column of 8 consecutive
// rows, whose swizzled positions j ^ (row & 7) are 8 different bank groups.
template <int D>
struct TmaQuantLane {
  using C = TmaQuantCfg<D>;
  static constexpr int LT = C::TPR == 1 ? 0 : 1;  // log2(TPR)
  int p, rr;
  __device__ __forceinline__ TmaQuantLane(int warp, int lane)
      : p((lane >> 3) & (C::TPR - 1)), rr(warp * (32 / C::TPR) + (lane & 7) + 8 * (lane >> (3 + LT))) {}
  __device__ __forceinline__ void load(const uint8_t* stage_base, uint64_t (&w)[C::W]) const {
#pragma unroll
    for (int cc = 0; cc < C::E / 64; ++cc) {
      const uint8_t* base = stage_base + (p * (C::E / 64) + cc) * (C::RB * 128) + rr * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 u = *reinterpret_cast<const uint4*>(base + ((j ^ (rr & 7)) << 4));
        uint64_t* o = &w[32 * cc + 4 * j];
        o[0] = f2_pack(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u));
        o[1] = f2_pack(__uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
        o[2] = f2_pack(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xFFFF0000u));
        o[3] = f2_pack(__uint_as_float(u.w << 16), __uint_as_float(u.w & 0xFFFF0000u));
      }
    }
  }
};

// max |v| over the thread's values
template <int W>
__device__ __forceinline__ float absmax_part(const uint64_t (&w)[W]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < W; ++i) {
    float a, b;
    f2_unpack(w[i], a, b);
    m = fmax3(m, fabsf(a), fabsf(b));
  }
  return m;
}

// Codes of the thread's E values: e4m3(v [/ sqrt(D)] * sc), stored to dst (E
// bytes, 16-byte aligned).
template <int D, bool ROT>
__device__ __forceinline__ void store_codes_part(const uint64_t (&w)[TmaQuantCfg<D>::W], float sc, uint8_t* dst) {
  constexpr int E = TmaQuantCfg<D>::E;
  constexpr float inv_sqrt_d = D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
  const uint64_t isd = f2_pack(inv_sqrt_d, inv_sqrt_d), sc2 = f2_pack(sc, sc);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < E / 16; ++c) {  // 16 codes per store
    uint32_t q[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float a0, b0, a1, b1;
      f2_unpack(f2_mul(ROT ? f2_mul(w[8 * c + 2 * k], isd) : w[8 * c + 2 * k], sc2), a0, b0);
      f2_unpack(f2_mul(ROT ? f2_mul(w[8 * c + 2 * k + 1], isd) : w[8 * c + 2 * k + 1], sc2), a1, b1);
      q[k] = static_cast<uint32_t>(pack_e4m3x2(a0, b0)) | (static_cast<uint32_t>(pack_e4m3x2(a1, b1)) << 16);
    }
    d4[c] = make_uint4(q[0], q[1], q[2], q[3]);
  }
}

// ws[0 .. n-1]: amax bits of each tensor, ws[n]: arrival counter of the grid
// barrier (one round per tensor); all zero at launch. descale_out[t]: tensor
// t's descale. The tensors are taken one after the other (pass 1, barrier,
// pass 2 of tensor 0, then of tensor 1, ...), so that pass 2 re-reads a tensor
// while it is still in L2 even when all of them together are larger.
template <int D, bool ROT>
__global__ void __launch_bounds__(TmaQuantCfg<D>::THREADS, 1)
quant_tma_kernel(const __grid_constant__ QuantMaps qm, int rows, const float* __restrict__ signs, unsigned int* ws,
                 float* descale_out) {
  using C = TmaQuantCfg<D>;
  constexpr float inv_sqrt_d = D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kTmaQuantStages], empty[kTmaQuantStages];
  __shared__ __align__(16) float sgn[D];
  __shared__ unsigned int amax_cta;
  __shared__ float amax_t;
  __shared__ volatile int abort_flag;
  DevStatus* st = &g_fa_status;
  const int tid = static_cast<int>(threadIdx.x), warp = tid >> 5, lane = tid & 31;
  const int nblk = (rows + C::RB - 1) / C::RB;  // row blocks per tensor
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int per = c < nblk ? (nblk - 1 - c) / G + 1 : 0;  // this CTA's blocks per tensor
  // Stream position s = 2 per t + i: tensor t, pass 1 for i < per (block
  // c + i G), pass 2 for i >= per (the same blocks in reverse).
  auto block_of = [&](int i) { return c + (i < per ? i : 2 * per - 1 - i) * G; };
  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < kTmaQuantStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::CONSUMER_WARPS);
    }
    amax_cta = 0u;
    fence_mbar_init();
  }
  if (ROT && tid < D) sgn[tid] = signs != nullptr ? signs[tid] : 1.0f;
  __syncthreads();

  if (warp == C::CONSUMER_WARPS) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      for (int t = 0; t < qm.n; ++t) tma_prefetch_desc(&qm.x[t]);
      bool ok = true;
      int s = 0;
      for (; s < 2 * per * qm.n && ok; ++s) {
        const int t = s / (2 * per), b = block_of(s % (2 * per));
        const int stage = s % kTmaQuantStages, round = s / kTmaQuantStages;
        if (round > 0) ok = mbar_wait(&empty[stage], (round - 1) & 1, &abort_flag, st, 61);
        if (!ok) break;
        uint8_t* dst = smem + stage * C::STAGE;
        mbar_arrive_expect_tx(&full[stage], C::STAGE);
#pragma unroll
        for (int col = 0; col < C::COLS; ++col)
#pragma unroll
          for (int r0 = 0; r0 < C::RB; r0 += C::BOX_ROWS)
            tma_load_2d(dst + col * (C::RB * 128) + r0 * 128, &qm.x[t], &full[stage], col * 64, b * C::RB + r0);
      }
      // every issued load lands before the CTA can exit
      for (int q = s - kTmaQuantStages; q < s; ++q)
        if (q >= 0) {
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[q % kTmaQuantStages], (q / kTmaQuantStages) & 1))
            if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  const TmaQuantLane<D> ln(warp, lane);
  const float* sg = (ROT && signs != nullptr) ? sgn : nullptr;
  // The stage is handed back to the producer, whose next TMA write to it goes
  // through the async proxy: this thread's shared-memory reads of it are
  // ordered before that write by a proxy fence ahead of the warp's arrival.
  auto release_stage = [&](int stage) {
    fence_proxy_async_shared();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  };
  bool ok = true;
  int s = 0;
  for (int t = 0; t < qm.n; ++t) {
    // pass 1: amax of the rotated tensor
    float m = 0.f;
    for (int i = 0; i < per && ok; ++i, ++s) {
      const int stage = s % kTmaQuantStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[stage], (s / kTmaQuantStages) & 1, &abort_flag, st, 62));
      if (!ok) break;
      uint64_t w[C::W];
      ln.load(smem + stage * C::STAGE, w);
      release_stage(stage);
      rotate_part<D, ROT>(w, ln.p, sg);
      m = fmaxf(m, absmax_part(w));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) atomicMax(&amax_cta, __float_as_uint(m));
    named_barrier_sync(1, kTmaQuantConsumers);
    if (tid == 0) {
      const float cm = __uint_as_float(amax_cta);
      amax_cta = 0u;  // for the next tensor (every consumer has passed its atomicMax)
      atomicMax(&ws[t], __float_as_uint(ROT ? cm * inv_sqrt_d : cm));
      // Grid-wide barrier, round t: every CTA is resident (cooperative launch).
      // The wait is bounded; if it runs out the status word records it and the
      // CTA goes on.
      __threadfence();
      atomicAdd(&ws[qm.n], 1u);
      const unsigned int target = static_cast<unsigned int>(G) * static_cast<unsigned int>(t + 1);
      const unsigned long long t0 = globaltimer_ns();
      unsigned int arrived;
      for (;;) {
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(arrived) : "l"(ws + qm.n) : "memory");
        if (arrived >= target) break;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          if (atomicCAS(&st->code, 0u, 5u) == 0u) {
            st->site = 60;
            st->block = blockIdx.x;
          }
          break;
        }
        __nanosleep(64);
      }
      unsigned int a;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(a) : "l"(ws + t) : "memory");
      amax_t = __uint_as_float(a);
      if (blockIdx.x == 0) descale_out[t] = __uint_as_float(a) > 0.f ? __uint_as_float(a) / 448.0f : 1.0f;
    }
    named_barrier_sync(1, kTmaQuantConsumers);
    const float amax = amax_t;
    const float sc = amax > 0.f ? 448.0f / amax : 1.0f;
    // pass 2: the codes, the same blocks in reverse order
    for (int i = per; i < 2 * per && ok; ++i, ++s) {
      const int stage = s % kTmaQuantStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[stage], (s / kTmaQuantStages) & 1, &abort_flag, st, 63));
      if (!ok) break;
      uint64_t w[C::W];
      ln.load(smem + stage * C::STAGE, w);
      release_stage(stage);
      rotate_part<D, ROT>(w, ln.p, sg);
      const int row = block_of(i) * C::RB + ln.rr;
      if (row < rows) store_codes_part<D, ROT>(w, sc, qm.out[t] + static_cast<int64_t>(row) * D + C::E * ln.p);
    }
    // amax_t is read again only after the next round's first named barrier
  }
}

// ---------------------------------------------------------------------------
// Per-block scales, staged by TMA (quant_block_tma_kernel): one pass, no grid
// barrier, since every scale depends on one block of 128 rows of one head. The
// stages are RB rows of one head (2-D tiles of a [BH][N][D] map, rows past N
// zero-filled); the 128 * TPR threads of each 128-row block reduce its amax
// through shared memory and a named barrier of their own, then write its codes
// and descale. Same rotation and rounding as quant_tma_kernel.
// ---------------------------------------------------------------------------
template <int D, bool ROT>
__global__ void __launch_bounds__(TmaQuantCfg<D>::THREADS, 1)
quant_block_tma_kernel(const __grid_constant__ CUtensorMap tmx, uint8_t* __restrict__ out, int BH, int N,
                       const float* __restrict__ signs, float* __restrict__ descales) {
  using C = TmaQuantCfg<D>;
  constexpr int BLK = 128;                         // rows per scale block
  constexpr int NBPS = C::RB / BLK;                // blocks per stage
  constexpr int WPB = C::CONSUMER_WARPS / NBPS;    // warps per block
  static_assert(C::RB % BLK == 0, "stage rows");
  constexpr float inv_sqrt_d = D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kTmaQuantStages], empty[kTmaQuantStages];
  __shared__ __align__(16) float sgn[D];
  __shared__ float red[2][C::CONSUMER_WARPS];  // per-warp maxima, double-buffered by step
  __shared__ volatile int abort_flag;
  DevStatus* st = &g_fa_status;
  const int tid = static_cast<int>(threadIdx.x), warp = tid >> 5, lane = tid & 31;
  const int nsph = (N + C::RB - 1) / C::RB;  // stages per head
  const int nb = (N + BLK - 1) / BLK;         // scale blocks per head
  const long long units = static_cast<long long>(BH) * nsph;
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int K = c < units ? static_cast<int>((units - 1 - c) / G + 1) : 0;  // this CTA's stages
  // step i: unit u = c + i G, head u / nsph, stage u % nsph
  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < kTmaQuantStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::CONSUMER_WARPS);
    }
    fence_mbar_init();
  }
  if (ROT && tid < D) sgn[tid] = signs != nullptr ? signs[tid] : 1.0f;
  __syncthreads();

  if (warp == C::CONSUMER_WARPS) {
    if (lane == 0) {
      tma_prefetch_desc(&tmx);
      bool ok = true;
      int i = 0;
      for (; i < K && ok; ++i) {
        const long long u = c + static_cast<long long>(i) * G;
        const int bh = static_cast<int>(u / nsph), sr = static_cast<int>(u % nsph) * C::RB;
        const int stage = i % kTmaQuantStages, round = i / kTmaQuantStages;
        if (round > 0) ok = mbar_wait(&empty[stage], (round - 1) & 1, &abort_flag, st, 64);
        if (!ok) break;
        uint8_t* dst = smem + stage * C::STAGE;
        mbar_arrive_expect_tx(&full[stage], C::STAGE);
#pragma unroll
        for (int col = 0; col < C::COLS; ++col)
#pragma unroll
          for (int r0 = 0; r0 < C::RB; r0 += C::BOX_ROWS)
            tma_load_3d(dst + col * (C::RB * 128) + r0 * 128, &tmx, &full[stage], col * 64, sr + r0, bh);
      }
      for (int q = i - kTmaQuantStages; q < i; ++q)
        if (q >= 0) {
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[q % kTmaQuantStages], (q / kTmaQuantStages) & 1))
            if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
    }
    return;
  }

  const TmaQuantLane<D> ln(warp, lane);
  const float* sg = (ROT && signs != nullptr) ? sgn : nullptr;
  const int blk = ln.rr / BLK;  // this thread's block within a stage
  for (int i = 0; i < K; ++i) {
    const int stage = i % kTmaQuantStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], (i / kTmaQuantStages) & 1, &abort_flag, st, 65))) break;
    uint64_t w[C::W];
    ln.load(smem + stage * C::STAGE, w);
    fence_proxy_async_shared();  // reads ordered before the producer's next TMA write of the stage
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    rotate_part<D, ROT>(w, ln.p, sg);
    float m = absmax_part(w);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[i & 1][warp] = m;
    named_barrier_sync(2 + blk, WPB * 32);
    float amax = red[i & 1][blk * WPB];
#pragma unroll
    for (int k = 1; k < WPB; ++k) amax = fmaxf(amax, red[i & 1][blk * WPB + k]);
    if (ROT) amax *= inv_sqrt_d;
    const long long u = c + static_cast<long long>(i) * G;
    const int bh = static_cast<int>(u / nsph), r0 = static_cast<int>(u % nsph) * C::RB + blk * BLK;
    if (r0 < N) {  // a block with rows in this head
      if (ln.rr % BLK == 0 && ln.p == 0) descales[static_cast<long long>(bh) * nb + r0 / BLK] =
          amax > 0.f ? amax / 448.0f : 1.0f;
      const int row = r0 + ln.rr % BLK;
      if (row < N)
        store_codes_part<D, ROT>(w, amax > 0.f ? 448.0f / amax : 1.0f,
                                 out + (static_cast<long long>(bh) * N + row) * D + C::E * ln.p);
    }
  }
}

}  // namespace fa

namespace fa {

}  // namespace fa

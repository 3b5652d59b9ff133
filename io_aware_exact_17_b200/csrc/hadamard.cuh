// hadamard.cuh — the Hadamard rotation of 128-row bf16 tiles on the tensor core,
// and the e4m3 codes of the rotated rows: shared by the quantisers (quant.cuh)
// and by the attention kernel that rotates and quantises its own query tiles
// (attn_fwd.cuh), so that both produce the same codes bit for bit.
//
// "FlashAttention-3 (PT)", section "Inovações técnicas", subsection 3: Q and K
// are multiplied by a random orthogonal Hadamard matrix before quantisation.
// Here x' = x D H_d / sqrt(d) (D: diagonal of +-1 signs, H_d: Sylvester
// Hadamard). Sylvester's construction gives H_d = H_{d/64} (x) H_64, so
//   x D H_d = [x_0 D_0 H_64, ..., x_{n-1} D_{n-1} H_64] (H_{d/64} (x) I_64),
// with x_b, D_b the b-th 64-wide block of x and of the signs. A tile X (128
// rows x d, bf16, in the 128-byte-swizzle layout TMA writes: column blocks of
// 64 elements, 16 KB apart) is multiplied block by block by the operands D_b
// H_64 built in shared memory (entries +-1, exact in bf16), with tcgen05.mma
// into fp32 tensor-memory columns [64 b, 64 b + 64): the products are exact and
// the sums fp32. The remaining log2(d/64) stages (index bits 6, 7) are fp32
// butterflies on the way out of tensor memory, one rounding each. The split
// keeps the tensor-core work per tile at 128 x 64 x d multiply-adds instead
// of 128 x d x d. Without rotation the operand is the identity and no stage
// runs, so X comes back exactly. The 1/sqrt(d) factor is applied by the
// caller, after the amax.
#pragma once
#include <cstdint>
#include "sm100.cuh"

namespace fa {

template <int D>
struct HadCfg {
  static constexpr int BM = 128;                // rows per tile (tensor-memory lanes)
  static constexpr int NB = 64;                 // width of one Hadamard block (H_64)
  static constexpr int NBLK = D / NB;           // blocks per row: 1, 2 or 4
  static constexpr int HBLK = NB * NB * 2;      // bytes of one signed Hadamard block
  static constexpr int HMAT = NBLK * HBLK;      // bytes of the operand
  static constexpr float INV_SQRT_D = D == 64 ? 0.125f : (D == 128 ? 0.08838834764831845f : 0.0625f);
  static_assert(D == 64 || D == 128 || D == 256, "head dim");
};

// The B operand of the rotation at hm (1024-byte aligned), K-major in the
// 128-byte-swizzle layout: element (n, k) of block b is s_{b NB + k} H[k][n]
// with H[k][n] = (-1)^popcount(k & n), so that column n of the product of row
// x_r is (x_r D H) restricted to block b; without ROT, the identity. The whole
// CTA calls it; 16 bytes (8 consecutive k of one n) per store. A sign is -1
// where signs[i] < 0 (signs may be null: all +1).
template <int D, bool ROT>
__device__ __forceinline__ void build_rotation_operand(uint8_t* hm, const float* __restrict__ signs) {
  using C = HadCfg<D>;
  constexpr int NB = C::NB, UPR = NB / 8;  // 16-byte units per row n
  constexpr int UNITS = C::NBLK * NB * UPR;
  // A thread's units share k0 = 8 (tid % UPR) when blockDim.x is a multiple of
  // UPR (every launch here): its sign loads go out together, before any use.
  const int my_k0 = 8 * (static_cast<int>(threadIdx.x) % UPR);
  float sg[C::NBLK][8];
  if (ROT) {
#pragma unroll
    for (int b = 0; b < C::NBLK; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) sg[b][e] = signs != nullptr ? __ldg(signs + b * NB + my_k0 + e) : 1.0f;
  }
  for (int u = static_cast<int>(threadIdx.x); u < UNITS; u += static_cast<int>(blockDim.x)) {
    const int blk = u / (NB * UPR), n = (u / UPR) % NB, k0 = (u % UPR) * 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float v[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = k0 + e + h;
        if (ROT) {
          float s = 1.0f;
          if (k0 == my_k0) {
#pragma unroll
            for (int b = 0; b < C::NBLK; ++b)
              if (b == blk) s = sg[b][e + h];
          } else if (signs != nullptr) {
            s = __ldg(signs + blk * NB + k);
          }
          v[h] = (((__popc(k & n) & 1) != 0) != (s < 0.f)) ? -1.0f : 1.0f;
        } else {
          v[h] = k == n ? 1.0f : 0.0f;
        }
      }
      w[e / 2] = pack_bf16x2(v[0], v[1]);
    }
    const int chunk = k0 / 64, c16 = (k0 % 64) / 8;
    *reinterpret_cast<uint4*>(hm + blk * C::HBLK + chunk * (NB * 128) + n * 128 + ((c16 ^ (n & 7)) << 4)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// X (128 x D bf16 at shared address a) times the operands at shared address
// hm, block b into tensor-memory columns d_tmem + 64 b .. + 63 (fp32). One
// thread.
template <int D>
__device__ __forceinline__ void issue_rotation(uint32_t d_tmem, uint32_t a, uint32_t hm) {
  using C = HadCfg<D>;
  constexpr uint32_t idesc = idesc_make(1u, C::BM, C::NB, false);
#pragma unroll
  for (int blk = 0; blk < C::NBLK; ++blk)
#pragma unroll
    for (int kk = 0; kk < C::NB / 16; ++kk) {
      const int ka = (blk * C::NB + kk * 16) * 2, kb = kk * 32;  // bytes along a row of X, of the operand
      const uint64_t adesc = sdesc_sw128(a + (ka / 128) * (C::BM * 128) + ka % 128, 0, 1024);
      const uint64_t bdesc = sdesc_sw128(hm + blk * C::HBLK + (kb / 128) * (C::NB * 128) + kb % 128, 0, 1024);
      mma_bf16_ss(d_tmem + blk * C::NB, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
    }
}

__device__ __forceinline__ float absmax32(const uint32_t* v, float m) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) m = fmax3(m, fabsf(__uint_as_float(v[j])), fabsf(__uint_as_float(v[j + 1])));
  return m;
}

// 32-column chunks per product block read per tensor-memory round trip: both
// (all of the row, 64 or 128 registers) at d <= 128, one at d = 256.
template <int D>
constexpr int kRowChunks = D <= 128 ? 2 : 1;

// Loads 32-column chunks c0 .. c0 + NC - 1 (of 0, 1) of each of the thread's
// NBLK product blocks (columns 64 b + 32 c .. + 31) with one wait, and applies
// the stages of index bits 6, 7, ... in that order (with ROT): blocks b and
// b + h become v_b + v_{b+h} and v_b - v_{b+h}, one fp32 rounding each.
// Afterwards v[cc][b] holds output columns 64 b + 32 (c0 + cc) .. + 31 of the row.
template <int D, bool ROT, int NC>
__device__ __forceinline__ void row_chunks(uint32_t tb, int c0, uint32_t (&v)[NC][D / 64][32]) {
  constexpr int NBLK = D / 64;
#pragma unroll
  for (int cc = 0; cc < NC; ++cc)
#pragma unroll
    for (int b = 0; b < NBLK; ++b) tmem_ld32(tb + 64 * b + 32 * (c0 + cc), v[cc][b]);
#pragma unroll
  for (int cc = 0; cc < NC; ++cc)
#pragma unroll
    for (int b = 0; b < NBLK; ++b) tmem_wait_ld_dep32(v[cc][b]);  // the first waits for all; each ties its registers
  if constexpr (ROT && NBLK > 1) {
#pragma unroll
    for (int cc = 0; cc < NC; ++cc)
#pragma unroll
      for (int h = 1; h < NBLK; h <<= 1)
#pragma unroll
        for (int b = 0; b < NBLK; ++b)
          if ((b & h) == 0)
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const uint64_t x = f2_pack(__uint_as_float(v[cc][b][j]), __uint_as_float(v[cc][b][j + 1]));
              const uint64_t y = f2_pack(__uint_as_float(v[cc][b + h][j]), __uint_as_float(v[cc][b + h][j + 1]));
              float s0, s1, d0, d1;
              f2_unpack(f2_add(x, y), s0, s1);
              f2_unpack(f2_sub(x, y), d0, d1);
              v[cc][b][j] = __float_as_uint(s0);
              v[cc][b][j + 1] = __float_as_uint(s1);
              v[cc][b + h][j] = __float_as_uint(d0);
              v[cc][b + h][j + 1] = __float_as_uint(d1);
            }
  }
}

// max |x'| over the thread's row of a product in tensor memory (tb: the warp's
// lane quarter and the product's first column), before the 1/sqrt(d) factor.
// Every lane of the warp must call (tcgen05.ld is warp-wide).
template <int D, bool ROT>
__device__ __forceinline__ float row_absmax(uint32_t tb) {
  constexpr int NC = kRowChunks<D>;
  float m = 0.f;
#pragma unroll 1
  for (int c0 = 0; c0 < 2; c0 += NC) {
    uint32_t v[NC][D / 64][32];
    row_chunks<D, ROT, NC>(tb, c0, v);
#pragma unroll
    for (int cc = 0; cc < NC; ++cc)
#pragma unroll
      for (int b = 0; b < D / 64; ++b) m = absmax32(v[cc][b], m);
  }
  return m;
}

// The codes of 32 values: e4m3(fl(fl(v * 1/sqrt(d)) * sc)) with ROT, else
// e4m3(fl(v * sc)); round to nearest even, saturating. c0 holds values 0-15
// (value 0 in its lowest byte), c1 values 16-31.
template <int D, bool ROT>
__device__ __forceinline__ void codes32(const uint32_t* v, float sc, uint4& c0, uint4& c1) {
  const uint64_t isd = f2_pack(HadCfg<D>::INV_SQRT_D, HadCfg<D>::INV_SQRT_D), sc2 = f2_pack(sc, sc);
  uint32_t q[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint64_t x0 = f2_pack(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]));
    const uint64_t x1 = f2_pack(__uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
    float a0, b0, a1, b1;
    f2_unpack(f2_mul(ROT ? f2_mul(x0, isd) : x0, sc2), a0, b0);
    f2_unpack(f2_mul(ROT ? f2_mul(x1, isd) : x1, sc2), a1, b1);
    q[k] = static_cast<uint32_t>(pack_e4m3x2(a0, b0)) | (static_cast<uint32_t>(pack_e4m3x2(a1, b1)) << 16);
  }
  c0 = make_uint4(q[0], q[1], q[2], q[3]);
  c1 = make_uint4(q[4], q[5], q[6], q[7]);
}

// The codes of the thread's row, handed out 16 at a time: put(j, codes of
// elements 16j .. 16j+15). Every lane of the warp must call.
template <int D, bool ROT, typename Put>
__device__ __forceinline__ void row_codes(uint32_t tb, float sc, Put&& put) {
  constexpr int NC = kRowChunks<D>;
#pragma unroll 1
  for (int c0 = 0; c0 < 2; c0 += NC) {
    uint32_t v[NC][D / 64][32];
    row_chunks<D, ROT, NC>(tb, c0, v);
#pragma unroll
    for (int cc = 0; cc < NC; ++cc)
#pragma unroll
      for (int b = 0; b < D / 64; ++b) {
        uint4 q0, q1;
        codes32<D, ROT>(v[cc][b], sc, q0, q1);
        put(4 * b + 2 * (c0 + cc), q0);
        put(4 * b + 2 * (c0 + cc) + 1, q1);
      }
  }
}

}  // namespace fa

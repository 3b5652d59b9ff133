// attn_fwd.cuh — fused, tiled exact-attention forward for sm_100a.
//
// Computes, per (batch, head) and query row i,
//   O_i = sum_j softmax_j(scale * q_i . k_j) v_j   over visible keys j,
//   LSE_i = ln sum_j exp(scale * q_i . k_j),
// with the N x N score matrix never leaving the SM: "Flash Attention" glossary
// page, second paragraph (tiling in on-chip memory plus the online, numerically
// stable softmax); "FlashAttention-3 (PT)", section "FlashAttention e
// FlashAttention-2" (tiling and fusing matmul + softmax + matmul in one kernel).
//
// Blackwell design (the pages' Hopper design is prior art):
//  * one CTA = NQ query tiles of 128 rows of one (batch, head); NQ = 2 for
//    d <= 128 so that the softmax of one tile overlaps the tensor-core work of
//    the other (the pages' "ping-pong", section "Inovações técnicas", 1);
//  * warp roles (section "Inovações técnicas", 1, producer/consumer warps):
//      warps 0..4*NQ-1 : softmax, one thread per query row, one warpgroup per tile;
//      warp 4*NQ       : tcgen05.mma issuer (one elected thread), TMEM owner;
//      warp 4*NQ+1     : TMA producer (Q once; K_j, V_j through a ring of
//                        shared-memory slots, prefetched ahead: section 2);
//  * S_t = Q_t K_jᵀ accumulates in TMEM (128 fp32 columns); softmax reads it,
//    writes P_t = exp2(..) as bf16 over the same columns, and the MMA warp
//    issues O_t += P_t V_j with P_t taken straight from TMEM;
//  * online softmax in base 2 with the scale folded into one FMA; the running
//    reference max is moved only when a row's max grows by more than 2^8, so
//    the O rescale (a TMEM read-modify-write) is rare. The final O / l and the
//    LSE use the same reference, so the result is exact, not approximated.
//  * the QK product can take e4m3 Q and K (the FP8 path with Hadamard-rotated
//    inputs: section "Inovações técnicas", 3); P and V stay bf16.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100.cuh"

namespace fa {

__device__ DevStatus g_fa_status;  // first device-side error of any launch

template <int D, int NQ, bool QK_FP8>
struct FwdCfg {
  static constexpr int BM = 128;  // query rows per tile (TMEM lanes)
  static constexpr int BN = 128;  // keys per K/V tile
  static constexpr int EQK = QK_FP8 ? 1 : 2;
  static constexpr int QK_CHUNKS = D * EQK / 128;  // 128-byte swizzle columns per Q/K row
  static constexpr int V_CHUNKS = D * 2 / 128;
  static constexpr int Q_TILE = BM * D * EQK;
  static constexpr int K_TILE = BN * D * EQK;
  static constexpr int V_TILE = BN * D * 2;
  static constexpr int SLOT = V_TILE;  // a ring slot holds one K or one V tile
  static constexpr int RING_BUDGET = 200 * 1024 - NQ * Q_TILE;
  static constexpr int NSLOT = (RING_BUDGET / SLOT) > 6 ? 6 : (RING_BUDGET / SLOT);
  static constexpr int SMEM_BYTES = 1024 + NQ * Q_TILE + NSLOT * SLOT;
  static constexpr int MMA_WARP = 4 * NQ;
  static constexpr int TMA_WARP = 4 * NQ + 1;
  static constexpr int THREADS = (4 * NQ + 2) * 32;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL(int t) { return static_cast<uint32_t>(t) * 128u; }
  static constexpr uint32_t O_COL(int t) { return static_cast<uint32_t>(NQ) * 128u + static_cast<uint32_t>(t * D); }
  static_assert(D == 64 || D == 128 || D == 256, "head dim");
  static_assert(QK_CHUNKS >= 1, "an e4m3 row must fill a 128-byte swizzle row");
  static_assert(NSLOT >= 2, "ring needs two slots");
  static_assert(NQ * 128 + NQ * D <= 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(SMEM_BYTES > 114 * 1024, "one CTA per SM (TMEM is allocated whole)");
};

struct FwdParams {
  __nv_bfloat16* o;          // [BH][N][D]
  float* lse;                // [BH][N], may be null
  const float* descale_qk;   // e4m3 path: {dq, dk}; else null
  int N;
  int n_qb;                  // query blocks (NQ*128 rows) per head
  float scale_log2;          // scale * log2(e)
};

// Bounded wait used only while tearing down after an abort: ignores the abort
// flag and records nothing.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 255u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

template <int D, int NQ, bool CAUSAL, bool QK_FP8>
__global__ void __launch_bounds__(FwdCfg<D, NQ, QK_FP8>::THREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D, NQ, QK_FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                      // NQ tiles
  uint8_t* sRing = smem + NQ * C::Q_TILE;  // NSLOT slots

  __shared__ __align__(8) uint64_t bar_full[C::NSLOT], bar_empty[C::NSLOT];
  __shared__ __align__(8) uint64_t bar_q, bar_drain, bar_s[NQ], bar_p[NQ], bar_o[NQ];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const uint32_t warp = warp_id(), lane = lane_id();

  // Work item: head bh, query block qb (heaviest causal blocks of a head first).
  const int bh = blockIdx.x / p.n_qb;
  int qb = blockIdx.x % p.n_qb;
  if (CAUSAL) qb = p.n_qb - 1 - qb;
  const int q0 = qb * NQ * C::BM;
  const int kv_end = CAUSAL ? min(p.N, q0 + NQ * C::BM) : p.N;
  const int n_kv = (kv_end + C::BN - 1) / C::BN;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_q, 1);
    mbar_init(&bar_drain, 1);
    for (int t = 0; t < NQ; ++t) {
      mbar_init(&bar_s[t], 1);
      mbar_init(&bar_p[t], 128);
      mbar_init(&bar_o[t], 1);
    }
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(&tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  DevStatus* st = &g_fa_status;

  if (warp == C::TMA_WARP) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar_q, NQ * C::Q_TILE);
      for (int t = 0; t < NQ; ++t)
        for (int c = 0; c < C::QK_CHUNKS; ++c)
          tma_load_3d(sQ + t * C::Q_TILE + c * (C::BM * 128), &tmQ, &bar_q, c * (128 / C::EQK),
                      q0 + t * C::BM, bh);
      int pos = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int kind = 0; kind < 2 && ok; ++kind, ++pos) {
          const int slot = pos % C::NSLOT;
          const int round = pos / C::NSLOT;
          if (round > 0) ok = mbar_wait(&bar_empty[slot], (round - 1) & 1, &abort_flag, st, 10);
          if (!ok) break;
          uint8_t* dst = sRing + slot * C::SLOT;
          if (kind == 0) {
            mbar_arrive_expect_tx(&bar_full[slot], C::K_TILE);
            for (int c = 0; c < C::QK_CHUNKS; ++c)
              tma_load_3d(dst + c * (C::BN * 128), &tmK, &bar_full[slot], c * (128 / C::EQK), j * C::BN, bh);
          } else {
            mbar_arrive_expect_tx(&bar_full[slot], C::V_TILE);
            for (int c = 0; c < C::V_CHUNKS; ++c)
              tma_load_3d(dst + c * (C::BN * 128), &tmV, &bar_full[slot], c * 64, j * C::BN, bh);
          }
        }
      }
      // Let every load this thread issued land before the CTA can exit.
      mbar_drain(&bar_q, 0);
      for (int q = pos - C::NSLOT; q < pos; ++q)
        if (q >= 0) mbar_drain(&bar_full[q % C::NSLOT], (q / C::NSLOT) & 1);
    }
  } else if (warp == C::MMA_WARP) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_make(QK_FP8 ? 0u : 1u, 128, C::BN, false);
      constexpr uint32_t idesc_pv = idesc_make(1u, 128, D, true);
      const uint32_t ring = smem_u32(sRing);
      const uint32_t qaddr = smem_u32(sQ);
      bool ok = mbar_wait(&bar_q, 0, &abort_flag, st, 20);
      for (int j = 0; j <= n_kv && ok; ++j) {
        const int kpos = 2 * j, vpos = 2 * j - 1;
        const int kslot = kpos % C::NSLOT, vslot = (vpos + C::NSLOT) % C::NSLOT;
        if (j < n_kv) ok = mbar_wait(&bar_full[kslot], (kpos / C::NSLOT) & 1, &abort_flag, st, 21);
        if (ok && j > 0) ok = mbar_wait(&bar_full[vslot], (vpos / C::NSLOT) & 1, &abort_flag, st, 22);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < NQ && ok; ++t) {
          if (j > 0) {
            ok = mbar_wait(&bar_p[t], (j - 1) & 1, &abort_flag, st, 23);
            if (!ok) break;
            tc_fence_after();
            // O_t += P_t V_{j-1}: A = P_t from TMEM (bf16 pairs), B = V tile (MN-major).
            const uint32_t vaddr = ring + vslot * C::SLOT;
#pragma unroll
            for (int kk = 0; kk < C::BN / 16; ++kk) {
              const uint64_t bdesc = sdesc_sw128(vaddr + kk * 16 * 128, C::BN * 128, 1024);
              mma_bf16_ts(tbase + C::O_COL(t), tbase + C::S_COL(t) + kk * 8, bdesc, idesc_pv,
                          (j > 1 || kk > 0) ? 1u : 0u);
            }
            if (j == n_kv) mma_commit(&bar_o[t]);
          }
          if (j < n_kv) {
            // S_t = Q_t K_jᵀ, both K-major, 32 bytes of the reduction dim per MMA.
            const uint32_t kaddr = ring + kslot * C::SLOT;
            const uint32_t qt = qaddr + t * C::Q_TILE;
#pragma unroll
            for (int kk = 0; kk < D * C::EQK / 32; ++kk) {
              const int kb = kk * 32, chunk = kb / 128, within = kb % 128;
              const uint64_t adesc = sdesc_sw128(qt + chunk * (C::BM * 128) + within, 0, 1024);
              const uint64_t bdesc = sdesc_sw128(kaddr + chunk * (C::BN * 128) + within, 0, 1024);
              if constexpr (QK_FP8)
                mma_e4m3_ss(tbase + C::S_COL(t), adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
              else
                mma_bf16_ss(tbase + C::S_COL(t), adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar_s[t]);
          }
        }
        if (!ok) break;
        if (j > 0) mma_commit(&bar_empty[vslot]);
        if (j < n_kv) mma_commit(&bar_empty[kslot]);
      }
      // Drain: TMEM is freed below only after every issued MMA has finished.
      mma_commit(&bar_drain);
      mbar_drain(&bar_drain, 0);
    }
  } else {
    // ------------------------------------------------------------- softmax --
    const int t = static_cast<int>(warp >> 2);
    const uint32_t lane_base = (warp & 3u) * 32u;
    const int r = static_cast<int>(lane_base + lane);
    const int qrow = q0 + t * C::BM + r;
    const uint32_t tS = tbase + (lane_base << 16) + C::S_COL(t);
    const uint32_t tO = tbase + (lane_base << 16) + C::O_COL(t);
    float s_log2 = p.scale_log2;
    if constexpr (QK_FP8) s_log2 *= __ldg(p.descale_qk) * __ldg(p.descale_qk + 1);
    const int kmax = CAUSAL ? min(qrow, p.N - 1) : p.N - 1;  // last visible key of this row
    float m_ref = -INFINITY;  // reference max, scaled log2 units
    float l_exact = 0.f;      // sum of the fp32 weights: gives the LSE
    float l_round = 0.f;      // sum of the bf16-rounded weights P uses: normalises O
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[t], j & 1, &abort_flag, st, 30 + t));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tS + 0, &s[0]);
      tmem_ld32(tS + 32, &s[32]);
      tmem_ld32(tS + 64, &s[64]);
      tmem_ld32(tS + 96, &s[96]);
      tmem_wait_ld();
      const int kbase = j * C::BN;
      if (kbase + C::BN - 1 > kmax) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (kbase + c > kmax) s[c] = __float_as_uint(-INFINITY);
      }
      // Row max: four independent chains of 3-input max.
      float a0 = fmaxf(__uint_as_float(s[0]), __uint_as_float(s[1]));
      float a1 = fmaxf(__uint_as_float(s[2]), __uint_as_float(s[3]));
      float a2 = fmaxf(__uint_as_float(s[4]), __uint_as_float(s[5]));
      float a3 = fmaxf(__uint_as_float(s[6]), __uint_as_float(s[7]));
#pragma unroll
      for (int c = 8; c < 128; c += 8) {
        a0 = fmax3(a0, __uint_as_float(s[c + 0]), __uint_as_float(s[c + 1]));
        a1 = fmax3(a1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        a2 = fmax3(a2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
        a3 = fmax3(a3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
      }
      const float mx_s = fmax3(a0, a1, fmaxf(a2, a3)) * s_log2;
      const bool grow = mx_s > m_ref + 8.0f;
      const float m_new = grow ? mx_s : m_ref;
      const float alpha = ex2_approx(m_ref - m_new);  // 1 when unchanged, 0 on the first tile
      m_ref = m_new;
      // p = 2^(x*s - m): one packed FMA per pair, then the SFU exp2; P packs to bf16.
      const uint64_t s2 = f2_pack(s_log2, s_log2);
      const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
      uint64_t acc_e[2] = {0ull, 0ull}, acc_r[2] = {0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        float t0, t1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), s2, nm2), t0, t1);
        const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
        const uint32_t pk = pack_bf16x2(p0, p1);
        const int a = (c >> 1) & 1;
        acc_e[a] = f2_add(acc_e[a], f2_pack(p0, p1));
        acc_r[a] = f2_add(acc_r[a], f2_pack(__uint_as_float(pk << 16), __uint_as_float(pk & 0xFFFF0000u)));
        s[c >> 1] = pk;
      }
      tmem_st32(tS + 0, &s[0]);
      tmem_st32(tS + 32, &s[32]);
      float e0, e1, e2, e3, r0, r1, r2, r3;
      f2_unpack(acc_e[0], e0, e1);
      f2_unpack(acc_e[1], e2, e3);
      f2_unpack(acc_r[0], r0, r1);
      f2_unpack(acc_r[1], r2, r3);
      l_exact = l_exact * alpha + ((e0 + e1) + (e2 + e3));
      l_round = l_round * alpha + ((r0 + r1) + (r2 + r3));
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // Rescale this warp's O rows in TMEM. The PV product of tile j-1 has
        // completed: the commit that signalled S_t for tile j also covers it, and
        // PV of tile j is issued only after this warpgroup arrives below.
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + c0, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(tO + c0, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p[t]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar_o[t], 0, &abort_flag, st, 40 + t));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_round;
      const bool in_range = qrow < p.N;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + (in_range ? qrow : 0)) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        tmem_ld32(tO + c0, ov);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (in_range && p.lse != nullptr)
        p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m_ref + __log2f(l_exact)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace fa

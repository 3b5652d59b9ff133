// attn_fwd_db.cuh — the square attention forward for d = 128 with 64-key steps
// and S double-buffered in tensor memory (attn_fwd_db_kernel).
//
// Same result and the same online softmax as attn_fwd_kernel (attn_fwd.cuh):
// exact attention per (batch, head) and query row, O = softmax(scale q kᵀ) V and
// the LSE, with the N x N scores kept on chip ("Flash Attention" glossary page,
// second paragraph; "FlashAttention-3 (PT)", section "FlashAttention e
// FlashAttention-2"). What differs is the schedule:
//
//  * a key step is 64 keys, so one query tile's S is 64 TMEM columns and each
//    of the two query tiles of a CTA has two S buffers: S_t(j) lands in buffer
//    j & 1 while the softmax warpgroup works on S_t(j-1) in the other one. The
//    MMA warp keeps S two steps ahead of P V: at step it it issues
//    O_t += P_t(it-2) V_(it-2) and then S_t(it) into the buffer that P_t(it-2)
//    occupied (the tensor core runs one thread's MMAs in order). The softmax
//    of a tile therefore never waits for its own product to come back; it waits
//    only for the S that was computed while it worked on the previous one;
//  * TMEM: S_0 (2 x 64 columns), S_1 (2 x 64), O_0 (128), O_1 (128) = 512;
//  * P_t(j) is signalled on a barrier of its own S buffer (bar_p[t][j & 1]):
//    the softmax may finish P_t(j+1) before the MMA warp has taken P_t(j), so
//    one barrier for both would run two phases ahead of its waiter;
//  * a rescale of O (the reference max grew by more than 2^8) needs O's product
//    of the previous step to be complete: that is the commit of S_t(j+1) (issued
//    after it), or for a tile's last step a commit issued right after its last
//    but one P V (bar_pvq).
// Square launches only (Nq = Nk, no key split, no decode layout); bf16 or e4m3
// Q and K (one scale per tensor or per 128-row block; QROT: bf16 Q rotated and
// quantised per 128-row tile in the kernel, as in attn_fwd_kernel); P and V bf16.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "attn_fwd.cuh"

namespace fa {

template <bool QK_FP8, bool QROT = false>
struct DbCfg {
  static constexpr int D = 128;
  static constexpr int NQ = 2;
  static constexpr int BM = 128;  // query rows per tile (TMEM lanes)
  static constexpr int BN = 64;   // keys per step
  static constexpr int EQK = QK_FP8 ? 1 : 2;
  static constexpr int QK_CHUNKS = D * EQK / 128;  // 128-byte swizzle columns per Q/K row
  static constexpr int V_CHUNKS = D * 2 / 128;
  // Q as loaded: bf16 under QROT (converted in place), else the MMA's type
  static constexpr int Q_LOAD_CHUNKS = QROT ? D * 2 / 128 : QK_CHUNKS;
  static constexpr int Q_LOAD_ELEMS = QROT ? 64 : 128 / EQK;
  static constexpr int Q_TILE = BM * D * (QROT ? 2 : EQK);
  static constexpr int K_TILE = BN * D * EQK;
  static_assert(!QROT || QK_FP8, "Q is quantised in the kernel for e4m3 only");
  static constexpr int V_TILE = BN * D * 2;
  static constexpr int SLOT = V_TILE;  // a ring slot holds one K or one V tile
  static constexpr int RING_BUDGET = 200 * 1024 - NQ * Q_TILE;
  static constexpr int NSLOT = (RING_BUDGET / SLOT) > 12 ? 12 : (RING_BUDGET / SLOT);
  static constexpr int SMEM_BYTES = 1024 + NQ * Q_TILE + NSLOT * SLOT;
  static constexpr int SOFTMAX_WARPS = 8;
  static constexpr int MMA_WARP = 8;
  static constexpr int TMA_WARP = 9;
  static constexpr int THREADS = 384;
  static constexpr int REG_LAUNCH = 168;
  static constexpr int REG_SOFTMAX = FA_REG_SOFTMAX;
  static constexpr int REG_OTHER = FA_REG_OTHER;
  static_assert(8 * 32 * REG_SOFTMAX + 128 * REG_OTHER <= THREADS * REG_LAUNCH, "register split");
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL(int t, int b) { return static_cast<uint32_t>(t * 128 + b * 64); }
  static constexpr uint32_t O_COL(int t) { return 256u + static_cast<uint32_t>(t) * 128u; }
  static_assert(NSLOT >= 8, "the ring holds K and V of four steps");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// One 64-key row of S (TMEM at tS) through the exponentials, as softmax_row
// for 128 keys: the second 32-column load is in flight during the first
// chunk's exps; P is packed into s[0 .. 31]. FULL: no key of the step is masked
// (the normalising sum is then the fp32 sum, else the sum of the bf16-rounded
// weights P holds).
template <bool FULL>
__device__ __forceinline__ void softmax_row64(uint32_t tS, uint32_t* s, float s_log2, float m_ref, int kbase,
                                              int kmax, float& sum_e, float& sum_r) {
  const uint64_t s2 = f2_pack(s_log2, s_log2);
  const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
  uint64_t acc_e[2] = {0ull, 0ull}, acc_r[2] = {0ull, 0ull};
  float mx[4];  // unused: no running max
  tmem_ld32(tS + 0, &s[0]);
  tmem_wait_ld_dep32(&s[0]);
  tmem_ld32(tS + 32, &s[32]);
  if (!FULL) mask_chunk32(&s[0], kbase, kmax);
  exp_chunk32<false, !FULL>(&s[0], &s[0], s2, nm2, acc_e, acc_r, mx);
  tmem_wait_ld_dep32(&s[32]);
  if (!FULL) mask_chunk32(&s[32], kbase + 32, kmax);
  exp_chunk32<false, !FULL>(&s[32], &s[16], s2, nm2, acc_e, acc_r, mx);
  float e0, e1, e2, e3, r0, r1, r2, r3;
  f2_unpack(acc_e[0], e0, e1);
  f2_unpack(acc_e[1], e2, e3);
  f2_unpack(acc_r[0], r0, r1);
  f2_unpack(acc_r[1], r2, r3);
  sum_e = (e0 + e1) + (e2 + e3);
  sum_r = FULL ? sum_e : (r0 + r1) + (r2 + r3);
}

__device__ __forceinline__ void softmax_row64_dispatch(uint32_t tS, uint32_t* s, float s_log2, float m_ref,
                                                       int kbase, int kmax, bool masked, float& se, float& sr) {
  // `masked` is warp-uniform: both paths issue tcgen05.ld
  if (masked)
    softmax_row64<false>(tS, s, s_log2, m_ref, kbase, kmax, se, sr);
  else
    softmax_row64<true>(tS, s, s_log2, m_ref, kbase, kmax, se, sr);
}

// Raw-score max of a 64-key row of S.
__device__ __forceinline__ float row_max64(uint32_t tS, uint32_t* s, int kbase, int kmax, bool masked) {
  float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    tmem_ld32(tS + 32 * ch, &s[32 * ch]);
    tmem_wait_ld_dep32(&s[32 * ch]);
    if (masked) mask_chunk32(&s[32 * ch], kbase + 32 * ch, kmax);
#pragma unroll
    for (int c = 0; c < 32; c += 8) {
      a[0] = fmax3(a[0], __uint_as_float(s[32 * ch + c + 0]), __uint_as_float(s[32 * ch + c + 1]));
      a[1] = fmax3(a[1], __uint_as_float(s[32 * ch + c + 2]), __uint_as_float(s[32 * ch + c + 3]));
      a[2] = fmax3(a[2], __uint_as_float(s[32 * ch + c + 4]), __uint_as_float(s[32 * ch + c + 5]));
      a[3] = fmax3(a[3], __uint_as_float(s[32 * ch + c + 6]), __uint_as_float(s[32 * ch + c + 7]));
    }
  }
  return fmax3(a[0], a[1], fmaxf(a[2], a[3]));
}

template <bool CAUSAL, bool QK_FP8, bool QROT = false>
__global__ void __launch_bounds__(DbCfg<QK_FP8, QROT>::THREADS, 1)
attn_fwd_db_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = DbCfg<QK_FP8, QROT>;
  constexpr int D = C::D, NQ = C::NQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                      // NQ tiles
  uint8_t* sRing = smem + NQ * C::Q_TILE;  // NSLOT slots

  __shared__ __align__(8) uint64_t bar_full[C::NSLOT], bar_empty[C::NSLOT];
  // bar_s[t][b]: S_t landed in buffer b; bar_pvq[t]: the tile's last but one
  // P V has completed; bar_qfree: the item's S MMAs (readers of sQ) are done
  __shared__ __align__(8) uint64_t bar_q, bar_qfree, bar_drain, bar_s[NQ][2], bar_p[NQ][2], bar_o[NQ], bar_pvq[NQ];
  // QROT: query tile t is in e4m3 (its warpgroup has converted it)
  __shared__ __align__(8) uint64_t bar_qready[NQ];
  __shared__ float qrot_red[NQ][4];  // per-warp maxima of each tile
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const uint32_t warp = warp_id(), lane = lane_id();

  // Work items as in attn_fwd_kernel: NQ query tiles of one head; CTA c takes
  // items c, c + gridDim.x, ... (snake order for causal launches).
  auto next_item = [&](int r) {
    const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return r * g + ((p.snake && (r & 1)) ? g - 1 - c : c);
  };
  auto item_at = [&](int it) {
    FwdItem w;
    w.sp = 0;
    w.bh = p.snake ? it % p.BH : it / p.n_qb;
    int qb = p.snake ? it / p.BH : it % p.n_qb;
    if (CAUSAL) qb = p.n_qb - 1 - qb;
    w.q0 = qb * NQ * C::BM;
    w.kt0 = 0;
    auto n_kv_of = [&](int t) {  // 64-key steps of query tile t
      const int row0 = w.q0 + t * C::BM;
      if (row0 >= p.Nq) return 0;
      const int end = CAUSAL ? min(p.Nk, min(p.Nq, row0 + C::BM) + p.causal_off) : p.Nk;
      return (end + C::BN - 1) / C::BN;
    };
    w.n_kv0 = n_kv_of(0);
    w.n_kv1 = n_kv_of(1);
    w.n_kv = max(w.n_kv0, w.n_kv1);
    return w;
  };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_q, 1);
    mbar_init(&bar_qfree, 1);
    mbar_init(&bar_drain, 1);
    for (int t = 0; t < NQ; ++t) {
      mbar_init(&bar_s[t][0], 1);
      mbar_init(&bar_s[t][1], 1);
      mbar_init(&bar_p[t][0], 4);  // one arrival per softmax warp of the tile
      mbar_init(&bar_p[t][1], 4);
      mbar_init(&bar_o[t], 1);
      mbar_init(&bar_pvq[t], 1);
      mbar_init(&bar_qready[t], 4);
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

  if (warp >= C::SOFTMAX_WARPS) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::REG_OTHER));
    if (warp == C::TMA_WARP && lane == 0) {
      // ---------------------------------------------------------- producer --
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int pos = 0, iter = 0;
      bool ok = true;
      for (int it = next_item(0); it < p.n_items && ok; it = next_item(iter + 1), ++iter) {
        const FwdItem w = item_at(it);
        if (iter > 0) ok = mbar_wait(&bar_qfree, (iter - 1) & 1, &abort_flag, st, 111);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar_q, NQ * C::Q_TILE);
        for (int t = 0; t < NQ; ++t)
          for (int c = 0; c < C::Q_LOAD_CHUNKS; ++c)
            tma_load_3d(sQ + t * C::Q_TILE + c * (C::BM * 128), &tmQ, &bar_q, c * C::Q_LOAD_ELEMS, w.q0 + t * C::BM,
                        w.bh);
        for (int j = 0; j < w.n_kv && ok; ++j) {
          for (int kind = 0; kind < 2 && ok; ++kind, ++pos) {
            const int slot = pos % C::NSLOT, round = pos / C::NSLOT;
            if (round > 0) ok = mbar_wait(&bar_empty[slot], (round - 1) & 1, &abort_flag, st, 110);
            if (!ok) break;
            uint8_t* dst = sRing + slot * C::SLOT;
            if (kind == 0) {
              mbar_arrive_expect_tx(&bar_full[slot], C::K_TILE);
              for (int c = 0; c < C::QK_CHUNKS; ++c)
                tma_load_3d(dst + c * (C::BN * 128), &tmK, &bar_full[slot], c * (128 / C::EQK), j * C::BN, w.bh);
            } else {
              mbar_arrive_expect_tx(&bar_full[slot], C::V_TILE);
              for (int c = 0; c < C::V_CHUNKS; ++c)
                tma_load_3d(dst + c * (C::BN * 128), &tmV, &bar_full[slot], c * 64, j * C::BN, w.bh);
            }
          }
        }
      }
      // every load this thread issued lands before the CTA can exit
      if (iter > 0) mbar_drain(&bar_q, (iter - 1) & 1);
      for (int q = pos - C::NSLOT; q < pos; ++q)
        if (q >= 0) mbar_drain(&bar_full[q % C::NSLOT], (q / C::NSLOT) & 1);
    } else if (warp == C::MMA_WARP && lane == 0) {
      // -------------------------------------------------------- MMA issuer --
      constexpr uint32_t idesc_qk = idesc_make(QK_FP8 ? 0u : 1u, 128, C::BN, false);
      constexpr uint32_t idesc_pv = idesc_make(1u, 128, D, true);
      const uint32_t ring = smem_u32(sRing);
      const uint32_t qaddr = smem_u32(sQ);
      int pos = 0, iter = 0;
      uint32_t pc[2][2] = {{0u, 0u}, {0u, 0u}};  // P-barrier phases waited, per query tile and buffer
      bool ok = true;
      for (int it = next_item(0); it < p.n_items && ok; it = next_item(iter + 1), ++iter) {
        const FwdItem w = item_at(it);
        const int nk = w.n_kv;
        auto n_kv_at = [&](int t) { return t == 0 ? w.n_kv0 : w.n_kv1; };
        if constexpr (!QROT) ok = mbar_wait(&bar_q, iter & 1, &abort_flag, st, 120);
        // Step s: P V of step s-2 (for each tile), then S of step s.
        for (int s = 0; s < nk + 2 && ok; ++s) {
          const int kpos = pos + 2 * s, vpos = pos + 2 * (s - 2) + 1;
          const int kslot = kpos % C::NSLOT, vslot = ((vpos % C::NSLOT) + C::NSLOT) % C::NSLOT;
          if (s < nk) ok = mbar_wait(&bar_full[kslot], (kpos / C::NSLOT) & 1, &abort_flag, st, 121);
          if (ok && s >= 2) ok = mbar_wait(&bar_full[vslot], (vpos / C::NSLOT) & 1, &abort_flag, st, 122);
          if (!ok) break;
          tc_fence_after();
          for (int t = 0; t < NQ && ok; ++t) {
            const int n_t = n_kv_at(t);
            const int jv = s - 2;  // the step whose P V runs now
            if (jv >= 0 && jv < n_t) {
              uint32_t& cnt = t == 0 ? (jv & 1 ? pc[0][1] : pc[0][0]) : (jv & 1 ? pc[1][1] : pc[1][0]);
              const uint32_t ph = cnt & 1u;
              ++cnt;
              ok = mbar_wait(&bar_p[t][jv & 1], ph, &abort_flag, st, 123 + t, kMmaWaitSleepNs);
              if (!ok) break;
              tc_fence_after();
              // O_t += P_t(jv) V_jv: A = P (bf16 pairs over S buffer jv & 1), B = V (MN-major)
              const uint32_t vaddr = ring + vslot * C::SLOT;
#pragma unroll
              for (int kk = 0; kk < C::BN / 16; ++kk) {
                const uint64_t bdesc = sdesc_sw128(vaddr + kk * 16 * 128, C::BN * 128, 1024);
                mma_bf16_ts(tbase + C::O_COL(t), tbase + C::S_COL(t, jv & 1) + kk * 8, bdesc, idesc_pv,
                            (jv > 0 || kk > 0) ? 1u : 0u);
              }
              if (jv == n_t - 2) mma_commit(&bar_pvq[t]);
              if (jv == n_t - 1) mma_commit(&bar_o[t]);
            }
            if (s < n_t) {
              if constexpr (QROT) {
                if (s == 0) {  // this tile's Q, converted to e4m3 by its warpgroup
                  ok = mbar_wait(&bar_qready[t], iter & 1, &abort_flag, st, 126 + t);
                  if (!ok) break;
                  tc_fence_after();
                }
              }
              // S_t(s) = Q_t K_sᵀ into buffer s & 1 (after the P V above, which read it)
              const uint32_t kaddr = ring + kslot * C::SLOT;
              const uint32_t qt = qaddr + t * C::Q_TILE;
#pragma unroll
              for (int kk = 0; kk < D * C::EQK / 32; ++kk) {
                const int kb = kk * 32, chunk = kb / 128, within = kb % 128;
                const uint64_t adesc = sdesc_sw128(qt + chunk * (C::BM * 128) + within, 0, 1024);
                const uint64_t bdesc = sdesc_sw128(kaddr + chunk * (C::BN * 128) + within, 0, 1024);
                if constexpr (QK_FP8)
                  mma_e4m3_ss(tbase + C::S_COL(t, s & 1), adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                else
                  mma_bf16_ss(tbase + C::S_COL(t, s & 1), adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
              }
              mma_commit(&bar_s[t][s & 1]);
            }
          }
          if (!ok) break;
          if (s == nk - 1) mma_commit(&bar_qfree);  // the item's last S MMAs read sQ
          if (s >= 2 && s - 2 < nk) mma_commit(&bar_empty[vslot]);
          if (s < nk) mma_commit(&bar_empty[kslot]);
        }
        if (!ok) break;
        if (nk == 0) mma_commit(&bar_qfree);
        pos += 2 * nk;
      }
      // Drain: TMEM is freed below only after every issued MMA has finished.
      mma_commit(&bar_drain);
      mbar_drain(&bar_drain, 0);
    }
  } else {
    // ----------------------------------------------------------- softmax --
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(C::REG_SOFTMAX));
    const int t = static_cast<int>(warp >> 2);
    uint32_t sc0 = 0u, sc1 = 0u;  // phases of bar_s[t][0], bar_s[t][1] waited
    uint32_t oc = 0, qc = 0;    // phases of bar_o[t], bar_pvq[t] waited
    bool ok = true;
    for (int round = 0, it = next_item(0); it < p.n_items && ok; it = next_item(++round)) {
      const FwdItem w = item_at(it);
      const int bh = w.bh, q0 = w.q0;
      const uint32_t lane_base = (warp & 3u) * 32u;
      const int r = static_cast<int>(lane_base + lane);
      const int qrow = q0 + t * C::BM + r;
      const uint32_t row_addr = tbase + (lane_base << 16);
      const uint32_t tO = row_addr + C::O_COL(t);
      float s_q = p.scale_log2;
      const float* dkb = nullptr;
      if constexpr (QROT) {
        // this warpgroup's Q tile, bf16 from the TMA, to e4m3 in place
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_q, round & 1, &abort_flag, st, 140));
        if (!ok) break;
        const float dq = qrot_tile(sQ + t * C::Q_TILE, r, p.qrot_rotate ? p.qrot_signs : nullptr,
                                   p.qrot_rotate != 0, qrot_red[t], warp & 3u, lane, 2 + t);
        fence_proxy_async_shared();  // the tensor core reads the codes through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_qready[t]);
        if (p.dq_out != nullptr && r == 0 && q0 + t * C::BM < p.Nq)
          p.dq_out[static_cast<size_t>(bh) * p.nbq + (q0 + t * C::BM) / C::BM] = dq;
        s_q *= dq;
        dkb = p.dk_block + static_cast<size_t>(bh) * p.nbk;
      } else if constexpr (QK_FP8) {
        if (p.dq_block != nullptr) {
          if (q0 + t * C::BM < p.Nq)
            s_q *= __ldg(p.dq_block + static_cast<size_t>(bh) * p.nbq + (q0 + t * C::BM) / C::BM);
          dkb = p.dk_block + static_cast<size_t>(bh) * p.nbk;
        } else {
          s_q *= __ldg(p.descale_qk) * __ldg(p.descale_qk + 1);
        }
      }
      const int kmax = CAUSAL ? min(qrow + p.causal_off, p.Nk - 1) : p.Nk - 1;  // last visible key
      float m_ref = -INFINITY, l_exact = 0.f, l_round = 0.f;
      const int n_t = t == 0 ? w.n_kv0 : w.n_kv1;
      // per-block key descales: one per 128 keys, i.e. per two steps
      float dk_cur = (QK_FP8 && dkb != nullptr && n_t > 0) ? __ldg(dkb) : 1.0f;
      for (int j = 0; j < n_t; ++j) {
        const int b = j & 1;
        const float s_log2 = s_q * dk_cur;
        if (QK_FP8 && dkb != nullptr && (j & 1) && j + 1 < n_t) dk_cur = __ldg(dkb + (j + 1) / 2);
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[t][b], (b ? sc1 : sc0) & 1u, &abort_flag, st, 130 + t));
        if (b) ++sc1; else ++sc0;
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = row_addr + C::S_COL(t, b);
        uint32_t s[64];
        const int kbase = j * C::BN;
        const bool masked = __any_sync(0xffffffffu, kbase + C::BN - 1 > kmax);  // warp-uniform
        float sum_e, sum_r, alpha = 1.0f;
        if (j == 0) {
          m_ref = row_max64(tS, s, kbase, kmax, masked) * s_log2;
          softmax_row64_dispatch(tS, s, s_log2, m_ref, kbase, kmax, masked, sum_e, sum_r);
        } else {
          softmax_row64_dispatch(tS, s, s_log2, m_ref, kbase, kmax, masked, sum_e, sum_r);
          if (__any_sync(0xffffffffu, sum_e > 256.0f)) {
            const float mx_s = row_max64(tS, s, kbase, kmax, masked) * s_log2;
            const bool grow = mx_s > m_ref + 8.0f;
            const float m_new = grow ? mx_s : m_ref;
            alpha = ex2_approx(m_ref - m_new);
            m_ref = m_new;
            softmax_row64_dispatch(tS, s, s_log2, m_ref, kbase, kmax, masked, sum_e, sum_r);
            if (__any_sync(0xffffffffu, grow)) {
              // O's product of step j-1 must be complete before O is rescaled:
              // the commit of S_t(j+1) follows it, and for the last step the
              // commit after the last but one P V does.
              if (j + 1 < n_t) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[t][b ^ 1], (b ? sc0 : sc1) & 1u, &abort_flag, st,
                                                       132 + t));
              } else {
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_pvq[t], qc & 1u, &abort_flag, st, 134 + t));
              }
              if (!ok) break;
              tc_fence_after();
#pragma unroll 1
              for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(tO + c0, ov);
                tmem_wait_ld_dep32(ov);
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                tmem_st32(tO + c0, ov);
              }
            }
          }
        }
        tmem_st32(tS, &s[0]);  // P: 32 columns of bf16 pairs over this S buffer
        l_exact = l_exact * alpha + sum_e;
        l_round = l_round * alpha + sum_r;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p[t][b]);
      }
      if (n_t >= 2 && ok) {  // keep bar_pvq's phase in step (the wait is immediate here)
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_pvq[t], qc & 1u, &abort_flag, st, 136 + t));
      }
      if (n_t >= 2) ++qc;
      if (ok && n_t > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar_o[t], oc & 1u, &abort_flag, st, 138 + t));
      if (n_t > 0) ++oc;
      const bool in_range = qrow < p.Nq;
      if (ok && n_t > 0) {
        tc_fence_after();
        const float inv_l = 1.0f / l_round;
        __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.Nq + (in_range ? qrow : 0)) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + c0, ov);
          tmem_wait_ld_dep32(ov);
          uint32_t q[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            q[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
          if (in_range) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(q[4 * i], q[4 * i + 1], q[4 * i + 2], q[4 * i + 3]);
          }
        }
        if (in_range && p.lse != nullptr)
          p.lse[static_cast<size_t>(bh) * p.Nq + qrow] = (m_ref + __log2f(l_exact)) * 0.69314718055994530942f;
      }
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

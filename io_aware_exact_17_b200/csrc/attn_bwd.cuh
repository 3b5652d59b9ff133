// attn_bwd.cuh — backward pass of exact attention for sm_100a: the gradients
// dQ, dK, dV of a loss through O = softmax(scale Q Kᵀ) V, given dO, the forward
// output O and its per-row LSE.
//
// The pages name training with the method ("FlashAttention-3 (PT)", opening
// paragraph and section "Desempenho e importância") but give no backward
// algorithm. This computes the chain rule through the plain definition, with
// the probabilities recomputed on chip from Q, K and the LSE, so that no N x N
// matrix reaches memory (the IO-aware principle of the "Flash Attention"
// glossary page, second paragraph):
//   P = exp(scale Q Kᵀ - LSE), dV = Pᵀ dO, dP = dO Vᵀ, D_i = dO_i · O_i,
//   dS = P ∘ (dP - D), dQ = scale dS K, dK = scale dSᵀ Q.
// (D_i = Σ_j P_ij dP_ij because O_i = Σ_j P_ij v_j.)
//
// Blackwell design:
//  * one CTA per (batch·head, tile of 128 keys). Its K_j and V_j stay in
//    shared memory, and dK_j and dV_j accumulate in TMEM over the query tiles
//    (causal: from the diagonal tile on, heaviest key tiles launched first);
//  * per query tile i (128 rows): TMA brings Q_i, dO_i and the tile's LSE and D
//    through a ring of stages; Sᵀ = K_j Q_iᵀ and dPᵀ = V_j dO_iᵀ land in TMEM
//    with keys on the lanes, each with its own barrier;
//  * two softmax warpgroups, 64 queries each, form P from Sᵀ (while dPᵀ is
//    still being computed), then dS = P (dP - D). They write P and dSᵀ back
//    over Sᵀ as bf16 pairs, the TMEM A operands of dV += Pᵀ dO_i and
//    dK += dSᵀ Q_i, and dSᵀ to shared memory in the 128-byte-swizzle layout,
//    read MN-major as the A operand of dQ_i = dS K_j;
//  * dQ_i is issued first and lands in the dP columns. The softmax warps read it
//    out (the next dPᵀ waits only for that), stage it in shared memory and add
//    it into an fp32 workspace with TMA reduce-adds, 32 x 32 tiles, while the
//    tensor core runs dV, dK and the next Sᵀ;
//  * a prologue kernel forms D_i and -LSE in log2 units, padded per head to
//    whole tiles (-inf and 0, so that padded queries get P = 0). An epilogue
//    kernel scales dQ and rounds it to bf16.
// TMEM holds Sᵀ (128 columns), dPᵀ / dQ (128), dV (d) and dK (d): d <= 128.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100.cuh"

namespace fa {

template <int D>
struct BwdCfg {
  static constexpr int BK = 128;                 // keys per CTA (TMEM lanes)
  static constexpr int BQ = 128;                 // queries per step
  static constexpr int TILE = 128 * D * 2;       // one 128 x D bf16 tile
  static constexpr int CHUNK = 128 * 128;        // one 128-byte swizzle column of a 128-row tile
  static constexpr int DS_TILE = BK * BQ * 2;    // dSᵀ, 128 keys x 128 queries bf16
  static constexpr int NST = D == 128 ? 2 : 3;   // Q_i / dO_i stages
  static constexpr int STAGE = 2 * TILE;
  static constexpr int LD_BYTES = 2 * BQ * 4;    // per stage: the step's -LSE log2(e), then its D
  // Dynamic shared memory, 1024-byte aligned (the swizzled tiles need it; the
  // kernel checks): K_j, V_j, dSᵀ, the Q_i / dO_i stages, their LSE / D, barriers.
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_DS = 2 * TILE;
  static constexpr int OFF_STAGE = OFF_DS + DS_TILE;
  static constexpr int OFF_LD = OFF_STAGE + NST * STAGE;
  static constexpr int OFF_BAR = OFF_LD + NST * LD_BYTES;
  static constexpr int N_BARS = 1 + 2 * NST + 8;
  static constexpr int SMEM_BYTES = OFF_BAR + 8 * N_BARS + 16;  // + TMEM address and abort flag
  static constexpr int THREADS = 384;            // 8 softmax warps, MMA warp, TMA warp, 2 idle
  static constexpr int MMA_WARP = 8;
  static constexpr int TMA_WARP = 9;
  // TMEM columns. S region: Sᵀ; then P (bf16 pairs, columns 0-63) and dSᵀ
  // (bf16 pairs, columns 64-127). dP region: dPᵀ, then dQ_i (D columns).
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t DP_COL = 128;
  static constexpr uint32_t DV_COL = 256;
  static constexpr uint32_t DK_COL = 256 + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct BwdParams {
  __nv_bfloat16* dk;        // [BH][N][D]
  __nv_bfloat16* dv;        // [BH][N][D]
  const float* nlse2;       // [BH][Npad]: -LSE * log2(e), -inf past N
  const float* dvec;        // [BH][Npad]: D_i = dO_i · O_i, 0 past N
  int BH, N, Npad, n_t;     // n_t = Npad / 128 tiles per head
  float scale, scale_log2;  // scale, scale * log2(e)
};

// Element-wise add of a shared-memory tile into global memory through a tensor
// map (the TMA's reduction; out-of-range elements of the box are not written),
// tracked by this thread's bulk async-group.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* smem_src, int x, int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// The same with an L2 eviction-priority policy for the destination lines.
__device__ __forceinline__ void tma_reduce_add_3d_hint(const CUtensorMap* map, const void* smem_src, int x, int y,
                                                       int z, uint64_t policy) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4}], [%1], %5;" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}
// 3-D tiled load for this CTA alone, with an L2 eviction-priority policy.
__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// Untiled bulk copy global -> this CTA's shared memory (both addresses 16-byte
// aligned, bytes a multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmdK,
                    const __grid_constant__ CUtensorMap tmdV, const BwdParams p) {
  (void)tmdK;  // dK and dV by per-row stores here (the d = 128 kernel stages them)
  (void)tmdV;
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    // the 128-byte-swizzle tiles need 1024-byte alignment: refuse, loudly
    if (threadIdx.x == 0 && atomicCAS(&g_fa_status.code, 0u, 3u /*FA_ERR_ALIGNMENT*/) == 0u) {
      g_fa_status.site = 70;
      g_fa_status.block = blockIdx.x;
    }
    return;
  }
  uint8_t* sK = smem_raw;
  uint8_t* sV = smem_raw + C::OFF_V;
  uint8_t* sdS = smem_raw + C::OFF_DS;
  uint8_t* sStage = smem_raw + C::OFF_STAGE;  // stage s: Q_i then dO_i
  const float* sLD = reinterpret_cast<const float*>(smem_raw + C::OFF_LD);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + C::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_full = bars + 1;
  uint64_t* bar_empty = bars + 1 + C::NST;
  uint64_t* bar_S = bars + 1 + 2 * C::NST;  // Sᵀ_i in TMEM
  uint64_t* bar_dP = bar_S + 1;             // dPᵀ_i in TMEM
  uint64_t* bar_sread = bar_S + 2;          // every softmax warp has read Sᵀ_i
  uint64_t* bar_p = bar_S + 3;              // P_i, dSᵀ_i written (TMEM and shared memory)
  uint64_t* bar_dq = bar_S + 4;             // dQ_i in TMEM
  uint64_t* bar_dqfree = bar_S + 5;         // dQ_i read out
  uint64_t* bar_done = bar_S + 6;           // dK, dV complete
  uint64_t* bar_drain = bar_S + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::N_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const uint32_t warp = warp_id(), lane = lane_id();
  // causal: key tile 0 (the most query tiles) first
  const int kt = static_cast<int>(blockIdx.x) / p.BH;
  const int bh = static_cast<int>(blockIdx.x) % p.BH;
  // Query tile of step i. Causal: from the diagonal tile on. Non-causal: all
  // tiles, starting at the CTA's own key tile, so that the CTAs of one head
  // that run at the same time add into different dQ rows.
  const int qt0 = CAUSAL ? kt : 0;
  const int n_steps = p.n_t - qt0;
  auto q_tile = [&](int i) { return CAUSAL ? kt + i : (kt + i) % p.n_t; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar_kv, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(bar_S, 1);
    mbar_init(bar_dP, 1);
    mbar_init(bar_sread, 8);  // one arrival per softmax warp
    mbar_init(bar_p, 8);
    mbar_init(bar_dq, 1);
    mbar_init(bar_dqfree, 8);
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  DevStatus* st = &g_fa_status;
  if (threadIdx.x == 0) launch_dependents();  // the dQ conversion may be scheduled (it waits for this grid)

  if (warp == C::TMA_WARP && lane == 0) {
    // ------------------------------------------------------------ producer --
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmdO);
    mbar_arrive_expect_tx(bar_kv, 2 * C::TILE);
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sK + c * C::CHUNK, &tmK, bar_kv, c * 64, kt * C::BK, bh);
      tma_load_3d(sV + c * C::CHUNK, &tmV, bar_kv, c * 64, kt * C::BK, bh);
    }
    grid_dependency_wait();  // the prologue's -LSE, D (and zeroed dQ accumulator) from here on
    const float* nlse2h = p.nlse2 + static_cast<size_t>(bh) * p.Npad;
    const float* dvh = p.dvec + static_cast<size_t>(bh) * p.Npad;
    bool ok = true;
    int issued = 0;
    for (int i = 0; i < n_steps && ok; ++i) {
      const int slot = i % C::NST, round = i / C::NST;
      if (round > 0) ok = mbar_wait(&bar_empty[slot], (round - 1) & 1, abort_flag, st, 50);
      if (!ok) break;
      uint8_t* dst = sStage + slot * C::STAGE;
      uint8_t* ld = smem_raw + C::OFF_LD + slot * C::LD_BYTES;
      const int q0 = q_tile(i) * C::BQ;
      mbar_arrive_expect_tx(&bar_full[slot], 2 * C::TILE + C::LD_BYTES);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(dst + c * C::CHUNK, &tmQ, &bar_full[slot], c * 64, q0, bh);
        tma_load_3d(dst + C::TILE + c * C::CHUNK, &tmdO, &bar_full[slot], c * 64, q0, bh);
      }
      bulk_load(ld, nlse2h + q0, C::BQ * 4, &bar_full[slot]);
      bulk_load(ld + C::BQ * 4, dvh + q0, C::BQ * 4, &bar_full[slot]);
      ++issued;
    }
    // every load this thread issued lands before the CTA can exit
    mbar_drain(bar_kv, 0);
    for (int i = issued - C::NST; i < issued; ++i)
      if (i >= 0) mbar_drain(&bar_full[i % C::NST], (i / C::NST) & 1);
  } else if (warp == C::MMA_WARP && lane == 0) {
    // ---------------------------------------------------------- MMA issuer --
    constexpr uint32_t idesc_kq = idesc_make(1u, 128, 128, false);            // A, B K-major
    constexpr uint32_t idesc_bmn = idesc_make(1u, 128, D, true);              // B MN-major
    constexpr uint32_t idesc_dq = idesc_make(1u, 128, D, true) | (1u << 15);  // A and B MN-major
    const uint32_t kaddr = smem_u32(sK), vaddr = smem_u32(sV), dsaddr = smem_u32(sdS);
    const uint32_t stage0 = smem_u32(sStage);
    // D_tmem = A Bᵀ over d: A a 128-row K-major tile (keys), B one (queries)
    auto issue_rows = [&](uint32_t dcol, uint32_t a, uint32_t b) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int kb = kk * 32, chunk = kb / 128, within = kb % 128;
        mma_bf16_ss(tbase + dcol, sdesc_sw128(a + chunk * C::CHUNK + within, 0, 1024),
                    sdesc_sw128(b + chunk * C::CHUNK + within, 0, 1024), idesc_kq, kk > 0 ? 1u : 0u);
      }
    };
    bool ok = mbar_wait(bar_kv, 0, abort_flag, st, 51);
    if (ok) ok = mbar_wait(&bar_full[0], 0, abort_flag, st, 52);
    if (ok) {
      tc_fence_after();
      issue_rows(C::S_COL, kaddr, stage0);
      mma_commit(bar_S);
      issue_rows(C::DP_COL, vaddr, stage0 + C::TILE);
      mma_commit(bar_dP);
    }
    for (int i = 0; i < n_steps && ok; ++i) {
      const int slot = i % C::NST;
      const uint32_t qaddr = stage0 + slot * C::STAGE, doaddr = qaddr + C::TILE;
      ok = mbar_wait(bar_p, i & 1, abort_flag, st, 53, 0u);
      if (!ok) break;
      tc_fence_after();
      // dQ_i = dS K_j into the dP columns (read by the softmax warps while the
      // products below run): A = dSᵀ read MN-major, B = K_j MN-major; 16 keys per MMA
#pragma unroll
      for (int kk = 0; kk < C::BK / 16; ++kk)
        mma_bf16_ss(tbase + C::DP_COL, sdesc_sw128(dsaddr + kk * 16 * 128, C::CHUNK, 1024),
                    sdesc_sw128(kaddr + kk * 16 * 128, C::CHUNK, 1024), idesc_dq, kk > 0 ? 1u : 0u);
      mma_commit(bar_dq);
      // dV += Pᵀ dO_i and dK += dSᵀ Q_i: A from TMEM (bf16 pairs, keys on lanes),
      // B = dO_i / Q_i MN-major; 16 queries per MMA
#pragma unroll
      for (int kk = 0; kk < C::BQ / 16; ++kk)
        mma_bf16_ts(tbase + C::DV_COL, tbase + C::S_COL + kk * 8, sdesc_sw128(doaddr + kk * 16 * 128, C::CHUNK, 1024),
                    idesc_bmn, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < C::BQ / 16; ++kk)
        mma_bf16_ts(tbase + C::DK_COL, tbase + C::S_COL + 64 + kk * 8,
                    sdesc_sw128(qaddr + kk * 16 * 128, C::CHUNK, 1024), idesc_bmn, (i > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&bar_empty[slot]);  // Q_i, dO_i and their LSE / D read
      if (i + 1 < n_steps) {
        const int ns = (i + 1) % C::NST;
        const uint32_t nq = stage0 + ns * C::STAGE;
        ok = mbar_wait(&bar_full[ns], ((i + 1) / C::NST) & 1, abort_flag, st, 54);
        if (!ok) break;
        tc_fence_after();
        issue_rows(C::S_COL, kaddr, nq);  // after dV_i and dK_i, which read P and dS from these columns
        mma_commit(bar_S);
        ok = mbar_wait(bar_dqfree, i & 1, abort_flag, st, 55, 0u);
        if (!ok) break;
        tc_fence_after();
        issue_rows(C::DP_COL, vaddr, nq + C::TILE);
        mma_commit(bar_dP);
      }
    }
    if (ok) mma_commit(bar_done);
    // TMEM is freed below only after every issued MMA has finished
    mma_commit(bar_drain);
    mbar_drain(bar_drain, 0);
  } else if (warp < 8) {
    // ------------------------------------------------------------- softmax --
    grid_dependency_wait();  // they reduce into the accumulator the prologue zeroed
    const int g = static_cast<int>(warp >> 2);  // query columns 64g .. 64g + 63
    const uint32_t lane_base = (warp & 3u) * 32u;
    const int r = static_cast<int>(lane_base + lane);  // key row (Sᵀ lane); query row for dQ
    const int kr = kt * C::BK + r;
    const uint32_t row_addr = tbase + (lane_base << 16);
    const uint32_t ds_row = smem_u32(sdS) + g * C::CHUNK + r * 128;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    // This warp's 4 KB of the dSᵀ tile (key rows 32 (warp & 3) .., column half g)
    // doubles as its staging area for dQ: the dQ MMA that read dSᵀ has completed
    // when dQ is read out, and the warp writes its dSᵀ rows again only after its
    // staged dQ has been read by the TMA (below).
    uint8_t* stage_dq = sdS + g * C::CHUNK + (warp & 3u) * 4096;
    // dQ_i rows (queries on lanes) added into the fp32 accumulator: TMEM ->
    // registers (then the columns are free for the next dPᵀ) -> shared memory,
    // 32 rows x 32 columns at a time in the 128-byte-swizzle layout -> one TMA
    // reduce-add per tile by lane 0 (rows past N are clipped by the map).
    auto dq_out = [&](int i) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(bar_dq, i & 1, abort_flag, st, 62))) return false;
      tc_fence_after();
      constexpr int NC = D / 64;  // 32-column chunks of this warpgroup's D / 2 columns
      uint32_t v[NC][32];
#pragma unroll
      for (int c = 0; c < NC; ++c) tmem_ld32(row_addr + C::DP_COL + g * (D / 2) + 32 * c, v[c]);
#pragma unroll
      for (int c = 0; c < NC; ++c) tmem_wait_ld_dep32(v[c]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dqfree);
      const uint32_t row_st = smem_u32(stage_dq) + lane * 128;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        if (c > 0) {
          if (lane == 0) bulk_wait_read_all();  // the previous tile has left the staging area
          __syncwarp();
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          st_shared_v4(row_st + ((static_cast<uint32_t>(u) ^ (lane & 7u)) << 4), v[c][4 * u], v[c][4 * u + 1],
                       v[c][4 * u + 2], v[c][4 * u + 3]);
        fence_proxy_async_shared();
        __syncwarp();
        const int y = q_tile(i) * C::BQ + static_cast<int>(lane_base);  // first query row of the tile
        if (lane == 0 && y < p.N) {  // rows past N are padding (and are clipped by the map)
          tma_reduce_add_3d(&tmdQ, stage_dq, g * (D / 2) + 32 * c, y, bh);
          bulk_commit();
        }
      }
      if (lane == 0) bulk_wait_read_all();  // before this warp writes its dSᵀ rows again
      __syncwarp();
      return true;
    };
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      if (i > 0 && !(ok = dq_out(i - 1))) break;
      const float* lse_s = sLD + (i % C::NST) * (C::LD_BYTES / 4) + 64 * g;  // this warpgroup's 64 queries
      const float* d_s = lse_s + C::BQ;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_S, i & 1, abort_flag, st, 60));
      if (!ok) break;
      tc_fence_after();
      // P = exp2(scale log2(e) s - LSE log2(e)) for this key row and 64 queries
      float pv[64];
      uint32_t sv2[2][32];
      tmem_ld32(row_addr + C::S_COL + 64 * g, sv2[0]);
      tmem_wait_ld_dep32(sv2[0]);
      tmem_ld32(row_addr + C::S_COL + 64 * g + 32, sv2[1]);  // in flight during chunk 0's exps
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t* sv = sv2[c];
        if (c == 1) tmem_wait_ld_dep32(sv);
        const float4* l4 = reinterpret_cast<const float4*>(lse_s + 32 * c);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 l = l4[u];  // -LSE log2(e) of four queries
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * u + 0]), __uint_as_float(sv[4 * u + 1])), sl2x2,
                           f2_pack(l.x, l.y)), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * u + 2]), __uint_as_float(sv[4 * u + 3])), sl2x2,
                           f2_pack(l.z, l.w)), x2, x3);
          pv[32 * c + 4 * u + 0] = ex2_approx(x0);
          pv[32 * c + 4 * u + 1] = ex2_approx(x1);
          pv[32 * c + 4 * u + 2] = ex2_approx(x2);
          pv[32 * c + 4 * u + 3] = ex2_approx(x3);
        }
      }
      // this warp's reads of Sᵀ are done (P and dS overwrite those columns below)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_sread);
      if (kr >= p.N) {
#pragma unroll
        for (int e = 0; e < 64; ++e) pv[e] = 0.f;
      }
      if (CAUSAL && i == 0) {
        // diagonal tile: query q0 + 64g + e sees key kr iff 64g + e >= r
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (64 * g + e < r) pv[e] = 0.f;
      }
      // dS = P (dP - D), rounded to bf16: into row r of dSᵀ in shared memory
      // (swizzled 16-byte units) and kept as pairs for TMEM
      ok = __all_sync(0xffffffffu, mbar_wait(bar_dP, i & 1, abort_flag, st, 64));
      if (!ok) break;
      tc_fence_after();
      uint32_t dsp[32];
      uint32_t dv2[2][32];
      tmem_ld32(row_addr + C::DP_COL + 64 * g, dv2[0]);
      tmem_wait_ld_dep32(dv2[0]);
      tmem_ld32(row_addr + C::DP_COL + 64 * g + 32, dv2[1]);  // in flight during chunk 0
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t* dv = dv2[c];
        if (c == 1) tmem_wait_ld_dep32(dv);
        const float4* d4 = reinterpret_cast<const float4*>(d_s + 32 * c);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 dd = d4[u];
          const float* pp = &pv[32 * c + 4 * u];
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack(pp[0], pp[1]),
                           f2_sub(f2_pack(__uint_as_float(dv[4 * u + 0]), __uint_as_float(dv[4 * u + 1])),
                                  f2_pack(dd.x, dd.y))), a0, a1);
          f2_unpack(f2_mul(f2_pack(pp[2], pp[3]),
                           f2_sub(f2_pack(__uint_as_float(dv[4 * u + 2]), __uint_as_float(dv[4 * u + 3])),
                                  f2_pack(dd.z, dd.w))), a2, a3);
          dsp[16 * c + 2 * u] = pack_bf16x2(a0, a1);
          dsp[16 * c + 2 * u + 1] = pack_bf16x2(a2, a3);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t unit = static_cast<uint32_t>(4 * c + u) ^ static_cast<uint32_t>(r & 7);
          st_shared_v4(ds_row + unit * 16, dsp[16 * c + 4 * u], dsp[16 * c + 4 * u + 1], dsp[16 * c + 4 * u + 2],
                       dsp[16 * c + 4 * u + 3]);
        }
      }
      uint32_t pp[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) pp[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
      // P and dSᵀ as bf16 pairs over Sᵀ, once every softmax warp has read its Sᵀ columns
      ok = __all_sync(0xffffffffu, mbar_wait(bar_sread, i & 1, abort_flag, st, 61));
      if (!ok) break;
      tc_fence_after();
      tmem_st32(row_addr + C::S_COL + 32 * g, pp);
      tmem_st32(row_addr + C::S_COL + 64 + 32 * g, dsp);
      tmem_wait_st();
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p);
    }
    if (ok && n_steps > 0) ok = dq_out(n_steps - 1);
    // ------------------------------------------------------------ epilogue --
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort_flag, st, 63));
    if (ok) {
      tc_fence_after();
      const size_t orow = (static_cast<size_t>(bh) * p.N + (kr < p.N ? kr : 0)) * D;
#pragma unroll
      for (int c0 = g * (D / 2); c0 < (g + 1) * (D / 2); c0 += 32) {
        uint32_t v[32], k[32];
        tmem_ld32(row_addr + C::DV_COL + c0, v);
        tmem_ld32(row_addr + C::DK_COL + c0, k);
        tmem_wait_ld_dep32(v);
        tmem_wait_ld_dep32(k);
        uint32_t pv2[16], pk2[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pv2[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
          pk2[e] = pack_bf16x2(__uint_as_float(k[2 * e]) * p.scale, __uint_as_float(k[2 * e + 1]) * p.scale);
        }
        if (kr < p.N) {
          uint4* dv4 = reinterpret_cast<uint4*>(p.dv + orow + c0);
          uint4* dk4 = reinterpret_cast<uint4*>(p.dk + orow + c0);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            dv4[u] = make_uint4(pv2[4 * u], pv2[4 * u + 1], pv2[4 * u + 2], pv2[4 * u + 3]);
            dk4[u] = make_uint4(pk2[4 * u], pk2[4 * u + 1], pk2[4 * u + 2], pk2[4 * u + 3]);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // the dQ reductions have completed before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// The same backward pass at d = 128 with the two softmax warpgroups ping-
// ponging (attn_bwd_pp_kernel): each step's 128 queries are two halves of 64,
// with their own Sᵀ, dPᵀ / dQᵀ columns and barriers, so that warpgroup h works
// on its half's P and dS while the tensor core runs the other half's products:
//   TMEM: Sᵀ_0 | Sᵀ_1 (64 columns each; then P_h and dSᵀ_h as bf16 pairs, 32
//         columns each) | dPᵀ_0 / dQᵀ_0 | dPᵀ_1 / dQᵀ_1 (64 each) | dV | dK.
// Per half h of step i the issuer waits for P_h, dS_h and runs
//   dQᵀ_h = K_jᵀ dSᵀ_h (A = K_j, B = dSᵀ_h from shared memory, both MN-major;
//   M = 128 = d on the lanes, N = 64 queries), dV += P_hᵀ dO_h, dK += dSᵀ_h Q_h
// (A from TMEM, K = 64 queries), then the next step's Sᵀ_h and, once the
// warpgroup has read dQᵀ_h out, dPᵀ_h (N = 64). dQ comes out transposed: lane
// = one of d's 128 indices, 64 queries along the columns; a warp's 32 lanes
// write one 128-byte row of a 32 x 32 staging tile per query, so the staging
// is conflict-free, and the TMA reduce-adds it into the fp32 accumulator as in
// attn_bwd_kernel.
// ---------------------------------------------------------------------------
struct BwdPpCfg {
  static constexpr int D = 128;
  static constexpr int BK = 128, BQ = 128, BH2 = 64;  // keys per CTA, queries per step, per half
  static constexpr int TILE = 128 * D * 2;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int DS_TILE = BK * BQ * 2;  // dSᵀ: half h in column chunk h
  static constexpr int NST = 2;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int LD_BYTES = 2 * BQ * 4;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_DS = 2 * TILE;
  static constexpr int OFF_STAGE = OFF_DS + DS_TILE;
  static constexpr int OFF_LD = OFF_STAGE + NST * STAGE;
  static constexpr int OFF_BAR = OFF_LD + NST * LD_BYTES;
  static constexpr int N_BARS = 1 + 2 * NST + 2 * 5 + 2 + 2;
  static constexpr int SMEM_BYTES = OFF_BAR + 8 * N_BARS + 16;
  static constexpr int THREADS = 384;
  static constexpr int MMA_WARP = 8;
  static constexpr int TMA_WARP = 9;
  static constexpr uint32_t S_COL(int h) { return 64u * static_cast<uint32_t>(h); }
  static constexpr uint32_t DP_COL(int h) { return 128u + 64u * static_cast<uint32_t>(h); }
  static constexpr uint32_t DV_COL = 256;
  static constexpr uint32_t DK_COL = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmdK,
                       const __grid_constant__ CUtensorMap tmdV, const BwdParams p) {
  using C = BwdPpCfg;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    // the 128-byte-swizzle tiles need 1024-byte alignment: refuse, loudly
    if (threadIdx.x == 0 && atomicCAS(&g_fa_status.code, 0u, 3u /*FA_ERR_ALIGNMENT*/) == 0u) {
      g_fa_status.site = 70;
      g_fa_status.block = blockIdx.x;
    }
    return;
  }
  uint8_t* sK = smem_raw;
  uint8_t* sV = smem_raw + C::OFF_V;
  uint8_t* sdS = smem_raw + C::OFF_DS;
  uint8_t* sStage = smem_raw + C::OFF_STAGE;  // stage s: Q_i then dO_i
  const float* sLD = reinterpret_cast<const float*>(smem_raw + C::OFF_LD);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + C::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_full = bars + 1;
  uint64_t* bar_empty = bars + 1 + C::NST;
  uint64_t* hb = bars + 1 + 2 * C::NST;  // per half h: hb[5 h + 0 .. 4]
  auto bar_S = [&](int h) { return hb + 5 * h; };       // Sᵀ_h in TMEM
  auto bar_dP = [&](int h) { return hb + 5 * h + 1; };  // dPᵀ_h in TMEM
  auto bar_p = [&](int h) { return hb + 5 * h + 2; };   // P_h, dSᵀ_h written (TMEM and shared memory)
  auto bar_dq = [&](int h) { return hb + 5 * h + 3; };  // dQᵀ_h in TMEM
  auto bar_dqfree = [&](int h) { return hb + 5 * h + 4; };  // dQᵀ_h read out
  uint64_t* bar_done = hb + 10;                         // dK, dV complete
  uint64_t* bar_drain = hb + 11;
  auto bar_epi = [&](int h) { return hb + 12 + h; };    // warpgroup h's dK, dV rows staged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::N_BARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int kt = static_cast<int>(blockIdx.x) / p.BH;  // causal: key tile 0 (the most query tiles) first
  const int bh = static_cast<int>(blockIdx.x) % p.BH;
  // Query tile of step i, as in attn_bwd_kernel.
  const int qt0 = CAUSAL ? kt : 0;
  const int n_steps = p.n_t - qt0;
  auto q_tile = [&](int i) { return CAUSAL ? kt + i : (kt + i) % p.n_t; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar_kv, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar_S(h), 1);
      mbar_init(bar_dP(h), 1);
      mbar_init(bar_p(h), 4);  // one arrival per warp of the half's warpgroup
      mbar_init(bar_dq(h), 1);
      mbar_init(bar_dqfree(h), 4);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_epi(0), 4);
    mbar_init(bar_epi(1), 4);
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  DevStatus* st = &g_fa_status;
  if (threadIdx.x == 0) launch_dependents();  // the dQ conversion may be scheduled (it waits for this grid)

  if (warp == C::TMA_WARP && lane == 0) {
    // ------------------------------------------------------------ producer --
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmdO);
    // K_j and V_j are read by this CTA alone: let them leave L2 first, so that
    // the heads' Q, dO and the dQ accumulator stay
    const uint64_t pol_once = l2_policy_evict_first();
    mbar_arrive_expect_tx(bar_kv, 2 * C::TILE);
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d_hint(sK + c * C::CHUNK, &tmK, bar_kv, c * 64, kt * C::BK, bh, pol_once);
      tma_load_3d_hint(sV + c * C::CHUNK, &tmV, bar_kv, c * 64, kt * C::BK, bh, pol_once);
    }
    grid_dependency_wait();  // the prologue's -LSE, D (and zeroed dQ accumulator) from here on
    const float* nlse2h = p.nlse2 + static_cast<size_t>(bh) * p.Npad;
    const float* dvh = p.dvec + static_cast<size_t>(bh) * p.Npad;
    bool ok = true;
    int issued = 0;
    for (int i = 0; i < n_steps && ok; ++i) {
      const int slot = i % C::NST, round = i / C::NST;
      if (round > 0) ok = mbar_wait(&bar_empty[slot], (round - 1) & 1, abort_flag, st, 50);
      if (!ok) break;
      uint8_t* dst = sStage + slot * C::STAGE;
      uint8_t* ld = smem_raw + C::OFF_LD + slot * C::LD_BYTES;
      const int q0 = q_tile(i) * C::BQ;
      mbar_arrive_expect_tx(&bar_full[slot], 2 * C::TILE + C::LD_BYTES);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(dst + c * C::CHUNK, &tmQ, &bar_full[slot], c * 64, q0, bh);
        tma_load_3d(dst + C::TILE + c * C::CHUNK, &tmdO, &bar_full[slot], c * 64, q0, bh);
      }
      bulk_load(ld, nlse2h + q0, C::BQ * 4, &bar_full[slot]);
      bulk_load(ld + C::BQ * 4, dvh + q0, C::BQ * 4, &bar_full[slot]);
      ++issued;
    }
    // every load this thread issued lands before the CTA can exit
    mbar_drain(bar_kv, 0);
    for (int i = issued - C::NST; i < issued; ++i)
      if (i >= 0) mbar_drain(&bar_full[i % C::NST], (i / C::NST) & 1);
  } else if (warp == C::MMA_WARP && lane == 0) {
    // ---------------------------------------------------------- MMA issuer --
    constexpr uint32_t idesc_half = idesc_make(1u, 128, C::BH2, false);          // Sᵀ_h, dPᵀ_h: K-major A, B
    constexpr uint32_t idesc_dqt = idesc_make(1u, 128, C::BH2, true) | (1u << 15);  // dQᵀ_h: A, B MN-major
    constexpr uint32_t idesc_bmn = idesc_make(1u, 128, D, true);                 // dV, dK: B MN-major
    const uint32_t kaddr = smem_u32(sK), vaddr = smem_u32(sV), dsaddr = smem_u32(sdS);
    const uint32_t stage0 = smem_u32(sStage);
    // D_tmem = A Bᵀ over d: A a 128-row K-major tile (keys), B 64 rows (queries) of one
    auto issue_half = [&](uint32_t dcol, uint32_t a, uint32_t b) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int kb = kk * 32, chunk = kb / 128, within = kb % 128;
        mma_bf16_ss(tbase + dcol, sdesc_sw128(a + chunk * C::CHUNK + within, 0, 1024),
                    sdesc_sw128(b + chunk * C::CHUNK + within, 0, 1024), idesc_half, kk > 0 ? 1u : 0u);
      }
    };
    // The issuer polls its barriers and issues whatever is ready, the urgent
    // products first: the tensor core runs them in issue order, and a half's
    // dQᵀ gates that warpgroup's next step, so it goes out as soon as the
    // half's P and dS are written, ahead of work that has slack (the next Sᵀ
    // and dPᵀ, needed only after the warpgroup has added dQ). Per half h:
    //   qk[h]: steps whose dQᵀ_h, dV, dK (needs P_h(step)) are issued;
    //   sn[h]: steps whose Sᵀ_h is issued (needs dV, dK of the step before,
    //          which read P_h and dSᵀ_h from those columns, and the stage);
    //   dn[h]: steps whose dPᵀ_h is issued (needs Sᵀ_h and dQᵀ_h of the step
    //          before read out).
    bool ok = mbar_wait(bar_kv, 0, abort_flag, st, 51);
    int qk[2] = {0, 0}, sn[2] = {0, 0}, dn[2] = {0, 0};
    unsigned long long idle_since = globaltimer_ns();
    while (ok && (qk[0] < n_steps || qk[1] < n_steps)) {
      bool progress = false;
      for (int h = 0; h < 2; ++h) {
        const int i = qk[h];
        if (i < n_steps && i < dn[h] && mbar_try_wait(bar_p(h), i & 1)) {
          tc_fence_after();
          const int slot = i % C::NST;
          const uint32_t qaddr = stage0 + slot * C::STAGE, doaddr = qaddr + C::TILE;
          // dQᵀ_h = K_jᵀ dSᵀ_h into the dPᵀ_h columns; 16 keys per MMA
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk)
            mma_bf16_ss(tbase + C::DP_COL(h), sdesc_sw128(kaddr + kk * 16 * 128, C::CHUNK, 1024),
                        sdesc_sw128(dsaddr + h * C::CHUNK + kk * 16 * 128, C::CHUNK, 1024), idesc_dqt,
                        kk > 0 ? 1u : 0u);
          mma_commit(bar_dq(h));
          // dV += P_hᵀ dO_h and dK += dSᵀ_h Q_h: A from TMEM (bf16 pairs, keys on
          // lanes), B = rows 64 h .. of dO_i / Q_i, MN-major; 16 queries per MMA
#pragma unroll
          for (int kk = 0; kk < C::BH2 / 16; ++kk)
            mma_bf16_ts(tbase + C::DV_COL, tbase + C::S_COL(h) + kk * 8,
                        sdesc_sw128(doaddr + (h * C::BH2 + kk * 16) * 128, C::CHUNK, 1024), idesc_bmn,
                        (qk[0] + qk[1] > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < C::BH2 / 16; ++kk)
            mma_bf16_ts(tbase + C::DK_COL, tbase + C::S_COL(h) + 32 + kk * 8,
                        sdesc_sw128(qaddr + (h * C::BH2 + kk * 16) * 128, C::CHUNK, 1024), idesc_bmn,
                        (qk[0] + qk[1] > 0 || kk > 0) ? 1u : 0u);
          ++qk[h];
          // Q_i, dO_i and their LSE / D are read once both halves' products are
          if (qk[1 - h] > i) mma_commit(&bar_empty[slot]);
          progress = true;
        }
      }
      for (int h = 0; h < 2; ++h) {
        const int i = sn[h];  // Sᵀ_h of step i
        if (i < n_steps && qk[h] >= i && mbar_try_wait(&bar_full[i % C::NST], (i / C::NST) & 1)) {
          tc_fence_after();
          issue_half(C::S_COL(h), kaddr, stage0 + (i % C::NST) * C::STAGE + h * C::BH2 * 128);
          mma_commit(bar_S(h));
          ++sn[h];
          progress = true;
        }
      }
      for (int h = 0; h < 2; ++h) {
        const int i = dn[h];  // dPᵀ_h of step i
        if (i < n_steps && sn[h] > i && (i == 0 || mbar_try_wait(bar_dqfree(h), (i - 1) & 1))) {
          tc_fence_after();
          issue_half(C::DP_COL(h), vaddr, stage0 + (i % C::NST) * C::STAGE + C::TILE + h * C::BH2 * 128);
          mma_commit(bar_dP(h));
          ++dn[h];
          progress = true;
        }
      }
      // bounded: a wait that cannot end (a lost arrival) gives up like mbar_wait
      if (progress) {
        idle_since = globaltimer_ns();
      } else if (*abort_flag) {
        ok = false;
      } else if (globaltimer_ns() - idle_since > kWaitLimitNs) {
        *abort_flag = 1;
        if (atomicCAS(&st->code, 0u, 5u /*FA_ERR_TIMEOUT*/) == 0u) {
          st->site = 53;
          st->block = blockIdx.x;
        }
        ok = false;
      }
    }
    if (ok) mma_commit(bar_done);
    // TMEM is freed below only after every issued MMA has finished
    mma_commit(bar_drain);
    mbar_drain(bar_drain, 0);
  } else if (warp < 8) {
    // ------------------------------------------------------------- softmax --
    grid_dependency_wait();  // they reduce into the accumulator the prologue zeroed
    const int h = static_cast<int>(warp >> 2);  // this warpgroup's half: queries 64 h .. 64 h + 63 of a step
    const uint32_t lane_base = (warp & 3u) * 32u;
    const int r = static_cast<int>(lane_base + lane);  // key row (Sᵀ lane); d index for dQᵀ
    const int kr = kt * C::BK + r;
    const uint32_t row_addr = tbase + (lane_base << 16);
    const uint32_t ds_row = smem_u32(sdS) + h * C::CHUNK + r * 128;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    // This warp's 4 KB of dSᵀ_h (key rows 32 (warp & 3) ..) doubles as its dQ
    // staging area: the dQᵀ_h MMA that read dSᵀ_h has completed when dQᵀ_h is
    // read out, and the warp writes its dSᵀ rows again only after its staged dQ
    // has been read by the TMA (below).
    uint8_t* stage_dq = sdS + h * C::CHUNK + (warp & 3u) * 4096;
    // the accumulator is reduced into by every key tile of the head: keep it in L2
    const uint64_t pol_acc = l2_policy_evict_last();
    // dQᵀ_h (d = this lane's row, 64 queries) added into the fp32 accumulator:
    // TMEM -> registers (then the columns are free for the next dPᵀ_h) ->
    // shared memory, 32 queries x 32 d at a time (query = row, this lane's d =
    // column, 128-byte swizzle) -> one TMA reduce-add per tile by lane 0.
    auto dq_out = [&](int i) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(bar_dq(h), i & 1, abort_flag, st, 62))) return false;
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(row_addr + C::DP_COL(h), v[0]);
      tmem_ld32(row_addr + C::DP_COL(h) + 32, v[1]);
      tmem_wait_ld_dep32(v[0]);
      tmem_wait_ld_dep32(v[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dqfree(h));
      const uint32_t st0 = smem_u32(stage_dq) + ((lane & 3u) << 2);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (c > 0) {
          if (lane == 0) bulk_wait_read_all();  // the previous tile has left the staging area
          __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j)
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(st0 + j * 128 + ((((lane >> 2) ^ static_cast<uint32_t>(j & 7)))
                                                                           << 4)),
                       "r"(v[c][j])
                       : "memory");
        fence_proxy_async_shared();
        __syncwarp();
        const int y = q_tile(i) * C::BQ + h * C::BH2 + 32 * c;  // first query row of the tile
        if (lane == 0 && y < p.N) {  // rows past N are padding (and are clipped by the map)
          tma_reduce_add_3d_hint(&tmdQ, stage_dq, static_cast<int>(lane_base), y, bh, pol_acc);
          bulk_commit();
        }
      }
      // the last tile's read by the TMA is waited for only before this warp
      // writes its dSᵀ rows again (below), while the exps run
      return true;
    };
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      if (i > 0 && !(ok = dq_out(i - 1))) break;
      const float* lse_s = sLD + (i % C::NST) * (C::LD_BYTES / 4) + C::BH2 * h;  // this half's 64 queries
      const float* d_s = lse_s + C::BQ;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_S(h), i & 1, abort_flag, st, 60));
      if (!ok) break;
      tc_fence_after();
      // P = exp2(scale log2(e) s - LSE log2(e)) for this key row and 64 queries
      float pv[64];
      uint32_t sv2[2][32];
      tmem_ld32(row_addr + C::S_COL(h), sv2[0]);
      tmem_wait_ld_dep32(sv2[0]);
      tmem_ld32(row_addr + C::S_COL(h) + 32, sv2[1]);  // in flight during chunk 0's exps
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t* sv = sv2[c];
        if (c == 1) tmem_wait_ld_dep32(sv);
        const float4* l4 = reinterpret_cast<const float4*>(lse_s + 32 * c);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 l = l4[u];  // -LSE log2(e) of four queries
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * u + 0]), __uint_as_float(sv[4 * u + 1])), sl2x2,
                           f2_pack(l.x, l.y)), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * u + 2]), __uint_as_float(sv[4 * u + 3])), sl2x2,
                           f2_pack(l.z, l.w)), x2, x3);
          pv[32 * c + 4 * u + 0] = ex2_approx(x0);
          pv[32 * c + 4 * u + 1] = ex2_approx(x1);
          pv[32 * c + 4 * u + 2] = ex2_approx(x2);
          pv[32 * c + 4 * u + 3] = ex2_approx(x3);
        }
      }
      if (kr >= p.N) {
#pragma unroll
        for (int e = 0; e < 64; ++e) pv[e] = 0.f;
      }
      if (CAUSAL && i == 0) {
        // diagonal tile: query q0 + 64h + e sees key kr iff 64h + e >= r
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (C::BH2 * h + e < r) pv[e] = 0.f;
      }
      // dS = P (dP - D), rounded to bf16: into row r of dSᵀ_h in shared memory
      // (swizzled 16-byte units) and kept as pairs for TMEM
      ok = __all_sync(0xffffffffu, mbar_wait(bar_dP(h), i & 1, abort_flag, st, 64));
      if (!ok) break;
      tc_fence_after();
      uint32_t dsp[32];
      uint32_t dv2[2][32];
      if (lane == 0) bulk_wait_read_all();  // the staged dQ has left this warp's dSᵀ rows
      __syncwarp();
      tmem_ld32(row_addr + C::DP_COL(h), dv2[0]);
      tmem_wait_ld_dep32(dv2[0]);
      tmem_ld32(row_addr + C::DP_COL(h) + 32, dv2[1]);  // in flight during chunk 0
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t* dv = dv2[c];
        if (c == 1) tmem_wait_ld_dep32(dv);
        const float4* d4 = reinterpret_cast<const float4*>(d_s + 32 * c);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 dd = d4[u];
          const float* pp = &pv[32 * c + 4 * u];
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack(pp[0], pp[1]),
                           f2_sub(f2_pack(__uint_as_float(dv[4 * u + 0]), __uint_as_float(dv[4 * u + 1])),
                                  f2_pack(dd.x, dd.y))), a0, a1);
          f2_unpack(f2_mul(f2_pack(pp[2], pp[3]),
                           f2_sub(f2_pack(__uint_as_float(dv[4 * u + 2]), __uint_as_float(dv[4 * u + 3])),
                                  f2_pack(dd.z, dd.w))), a2, a3);
          dsp[16 * c + 2 * u] = pack_bf16x2(a0, a1);
          dsp[16 * c + 2 * u + 1] = pack_bf16x2(a2, a3);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t unit = static_cast<uint32_t>(4 * c + u) ^ static_cast<uint32_t>(r & 7);
          st_shared_v4(ds_row + unit * 16, dsp[16 * c + 4 * u], dsp[16 * c + 4 * u + 1], dsp[16 * c + 4 * u + 2],
                       dsp[16 * c + 4 * u + 3]);
        }
      }
      uint32_t pp[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) pp[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
      // P_h and dSᵀ_h as bf16 pairs over this thread's own Sᵀ_h row (read above)
      tmem_st32(row_addr + C::S_COL(h), pp);
      tmem_st32(row_addr + C::S_COL(h) + 32, dsp);
      tmem_wait_st();
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p(h));
    }
    if (ok && n_steps > 0) ok = dq_out(n_steps - 1);
    // ------------------------------------------------------------ epilogue --
    // dV and scale dK in bf16 through shared memory: once every MMA has
    // completed (bar_done), the K and V tiles are free, and warpgroup h stages
    // its 64 columns of dV (in sK) and dK (in sV) for all 128 key rows, as
    // 64-column boxes with the 128-byte swizzle (row r's 16-byte chunk c at c ^
    // (r mod 8)); one thread of the warpgroup stores both boxes with the TMA
    // (rows past N clipped).
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort_flag, st, 63));
    if (ok) {
      tc_fence_after();
      uint8_t* dv_row = sK + h * C::CHUNK + r * 128;
      uint8_t* dk_row = sV + h * C::CHUNK + r * 128;
#pragma unroll
      for (int cc = 0; cc < D / 2; cc += 32) {
        const int c0 = h * (D / 2) + cc;
        uint32_t v[32], k[32];
        tmem_ld32(row_addr + C::DV_COL + c0, v);
        tmem_ld32(row_addr + C::DK_COL + c0, k);
        tmem_wait_ld_dep32(v);
        tmem_wait_ld_dep32(k);
        uint32_t pv2[16], pk2[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pv2[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
          pk2[e] = pack_bf16x2(__uint_as_float(k[2 * e]) * p.scale, __uint_as_float(k[2 * e + 1]) * p.scale);
        }
        const int cb = cc / 8;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int off = ((cb + u) ^ (r & 7)) << 4;
          *reinterpret_cast<uint4*>(dv_row + off) = make_uint4(pv2[4 * u], pv2[4 * u + 1], pv2[4 * u + 2], pv2[4 * u + 3]);
          *reinterpret_cast<uint4*>(dk_row + off) = make_uint4(pk2[4 * u], pk2[4 * u + 1], pk2[4 * u + 2], pk2[4 * u + 3]);
        }
      }
      fence_proxy_async_shared();  // the TMA store reads the boxes through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_epi(h));
      if ((warp & 3u) == 0 && lane == 0) {
        if (mbar_wait(bar_epi(h), 0, abort_flag, st, 66 + h)) {
          tma_store_3d(&tmdV, sK + h * C::CHUNK, h * (D / 2), kt * C::BK, bh);
          tma_store_3d(&tmdK, sV + h * C::CHUNK, h * (D / 2), kt * C::BK, bh);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // the dQ reductions and dK, dV stores have completed before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// Prologue: per padded query row, D_i = dO_i · O_i and -LSE_i log2(e) (-inf
// and 0 past N), and zero row i of the dQ accumulator. D / 8 lanes per row,
// 16 bytes of O and of dO each; warps stride over the rows.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            const float* __restrict__ lse, float* nlse2, float* dvec,
                                                            float* dq_acc, int BH, int N, int Npad) {
  launch_dependents();  // the main kernel may set up and load K, V (it waits for this grid before the rest)
  constexpr int LPR = D / 8;     // lanes per row
  constexpr int RPW = 32 / LPR;  // rows per warp per pass
  const long long rows = static_cast<long long>(BH) * Npad;
  const uint32_t lane = lane_id();
  const int sub = static_cast<int>(lane) / LPR, l = static_cast<int>(lane) % LPR;
  const long long stride = static_cast<long long>(gridDim.x) * 8 * RPW;
  for (long long r0 = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * RPW; r0 < rows; r0 += stride) {
    const long long row = r0 + sub;
    const int bh = static_cast<int>(row / Npad), i = static_cast<int>(row % Npad);
    const bool valid = row < rows && i < N;
    float acc = 0.f;
    if (valid) {
      const size_t off = (static_cast<size_t>(bh) * N + i) * D + l * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(o + off);
      const uint4 b = *reinterpret_cast<const uint4*>(dout + off);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[e]));
        const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[e]));
        acc += af.x * bf.x + af.y * bf.y;
      }
      float4* z = reinterpret_cast<float4*>(dq_acc + off);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int s = LPR / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (row < rows && l == 0) {
      nlse2[row] = valid ? lse[static_cast<size_t>(bh) * N + i] * -1.4426950408889634f : -INFINITY;
      dvec[row] = valid ? acc : 0.f;
    }
  }
}

// Epilogue: dQ = scale * accumulator, rounded to bf16. n4 groups of 4 elements.
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float4* __restrict__ acc, uint2* __restrict__ dq,
                                                          long long n4, float scale) {
  grid_dependency_wait();  // the main kernel's reductions are complete
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = acc[i];
    dq[i] = make_uint2(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale));
  }
}

}  // namespace fa

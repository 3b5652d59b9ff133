// quant.cuh — Hadamard rotate + e4m3 quantisation for the FP8 path.
//
// "FlashAttention-3 (PT)", section "Inovações técnicas", subsection 3 ("Baixa
// precisão (FP8)"): before attention, Q and K are multiplied by a random
// orthogonal (Hadamard) matrix, which spreads outlier coordinates over all
// coordinates; then they are quantised to FP8; the product Q Kᵀ is unchanged by
// the rotation. Here the rotation is x' = x D H_d / sqrt(d) along the head
// dimension (D = optional diagonal of +-1 signs, H_d the Sylvester Hadamard
// matrix). Codes = RNE-satfinite e4m3(x' * 448 / amax), descale = amax / 448,
// with amax = max |x'| over the tensor (quant_tensor_kernel) or over each block
// of 128 rows of a head (quant_block_kernel).
//
// The rotation is a dense contraction, so it runs on the tensor core
// (hadamard.cuh): each 128-row tile of x, staged in shared memory by TMA, is
// multiplied by the signed Hadamard matrix with tcgen05.mma into tensor
// memory. The epilogue warps read each row from tensor memory once for the
// amax and once for the codes, so the only per-element arithmetic left on the
// CUDA cores is the max, two multiplies and the convert.
//
// CTA roles (320 threads, one CTA per SM; quant_tensor_kernel adds a sync
// warp): warps 0-7 epilogue (two groups of four; group g takes the tiles of odd
// or even position, each warp the 32 rows of its tensor-memory lane quarter),
// warp 8 lane 0 the TMA producer, warp 9 lane 0 the MMA issuer (warp 9 also
// allocates tensor memory). A ring of
// STAGES shared-memory tiles and NBUF tensor-memory tiles pipelines load,
// product and epilogue. Each epilogue warp writes its 32 rows of codes into a
// staging buffer of its own (swizzled, so that the 32 lanes' 16-byte writes
// hit distinct banks) and stores them with TMA: 32 contiguous rows per store
// (two column halves at d = 256).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "hadamard.cuh"
#include "sm100.cuh"

namespace fa {

// Up to kQuantBatch tensors of one shape, rotated and quantised in one launch,
// each with its own scale.
constexpr int kQuantBatch = 8;
struct QuantBatch {
  const __nv_bfloat16* x[kQuantBatch];
  uint8_t* out[kQuantBatch];
  int n;
};

// descale_out[0 .. n-1] = v (the descales of empty tensors).
__global__ void fill_f32_kernel(float* out, int n, float v) {
  if (static_cast<int>(threadIdx.x) < n) out[threadIdx.x] = v;
}

template <int D>
struct RotQuantCfg : HadCfg<D> {
  using H = HadCfg<D>;
  static constexpr int COLS = D / 64;             // 128-byte columns of a bf16 row
  static constexpr int TILE = H::BM * D * 2;      // bytes of a bf16 tile
  static constexpr int NBUF = 512 / D;            // tiles held in tensor memory
  static constexpr int EPI_WARPS = 8;
  static constexpr int TMA_WARP = 8;
  static constexpr int MMA_WARP = 9;
  static constexpr int THREADS = 320;
  static constexpr int CROW = D < 128 ? D : 128;  // bytes of a row of a code store box
  static constexpr int NBOX = D / CROW;           // code store boxes per row (2 at d = 256)
  static constexpr int CBUF = 32 * D;             // one warp's staging buffer: NBOX boxes of 32 rows
  static constexpr int CODES = EPI_WARPS * CBUF;
  static constexpr int STAGES_FIT = (224 * 1024 - H::HMAT - CODES) / TILE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM = 1024 + H::HMAT + CODES + STAGES * TILE;
  static_assert(STAGES >= 2, "ring needs two stages");
  static_assert(NBUF % 2 == 0, "each tensor-memory tile belongs to one epilogue group");
  static_assert(SMEM <= 227 * 1024 - 1024, "shared memory (with room for the static part)");
};

// The TMA swizzle of the staged codes: 128-byte box rows (d >= 128) or 64-byte ones (d = 64).
template <int D>
constexpr CUtensorMapSwizzle codes_swizzle() {
  return D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
}

struct QuantMaps {
  CUtensorMap x[kQuantBatch];  // tensor t as [rows][D] bf16, box (64, 128), 128-byte swizzle
  CUtensorMap y[kQuantBatch];  // its codes as [rows][D] bytes, box (CROW, 32), codes_swizzle<D>()
  int n;
};

// Shared prologue of both kernels. The producer thread initialises the
// barriers and issues the first loads (positions 0 .. min(STAGES, n_pos) - 1)
// before the CTA builds the rotation operand, so the two overlap; warp 9
// allocates tensor memory. Returns the tensor-memory base.
template <int D, bool ROT, typename Load>
__device__ __forceinline__ uint32_t rot_quant_setup(uint8_t* hm, const float* signs, uint64_t* full, uint64_t* empty,
                                                    uint64_t* tfull, uint64_t* tfree, uint64_t* drain,
                                                    uint32_t* tmem_slot, volatile int* abort_flag, int n_pos,
                                                    Load&& load) {
  using C = RotQuantCfg<D>;
  if (warp_id() == C::TMA_WARP && lane_id() == 0) {
    *abort_flag = 0;
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tfree[i], 4);  // the four warps of the tile's epilogue group
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    for (int s = 0; s < C::STAGES && s < n_pos; ++s) {
      mbar_arrive_expect_tx(&full[s], C::TILE);
      load(s, s, &full[s]);
    }
  }
  build_rotation_operand<D, ROT>(hm, signs);
  fence_proxy_async_shared();  // the tensor core reads the operand through the async proxy
  if (warp_id() == C::MMA_WARP) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tmem_slot;
}

// MMA issuer loop over positions 0 .. n_pos - 1 (stage s % STAGES, tensor
// tile s % NBUF), then a drain: tensor memory is freed only after every issued
// product has completed.
template <int D>
__device__ __forceinline__ void rot_quant_mma_loop(int n_pos, uint32_t ring, uint32_t hm, uint32_t tbase,
                                                   uint64_t* full, uint64_t* empty, uint64_t* tfull,
                                                   uint64_t* tfree, uint64_t* drain, volatile int* abort_flag,
                                                   DevStatus* st, uint32_t site) {
  using C = RotQuantCfg<D>;
  for (int s = 0; s < n_pos; ++s) {
    const int stage = s % C::STAGES, buf = s % C::NBUF;
    if (!mbar_wait(&full[stage], (s / C::STAGES) & 1, abort_flag, st, site, 0)) break;
    if (s >= C::NBUF && !mbar_wait(&tfree[buf], ((s / C::NBUF) - 1) & 1, abort_flag, st, site + 1, 0)) break;
    tc_fence_after();
    issue_rotation<D>(tbase + buf * D, ring + stage * C::TILE, hm);
    mma_commit(&empty[stage]);  // the stage may be refilled once the product has read it
    mma_commit(&tfull[buf]);
  }
  mma_commit(drain);
  mbar_drain(drain, 0);
}

// TMA producer after the prologue: positions STAGES .. n_pos - 1, each into
// the stage its product has released; every issued load lands before the CTA
// can exit.
template <int D, typename Load>
__device__ __forceinline__ void rot_quant_producer(int n_pos, uint64_t* full, uint64_t* empty,
                                                   volatile int* abort_flag, DevStatus* st, uint32_t site,
                                                   Load&& load) {
  using C = RotQuantCfg<D>;
  int s = C::STAGES < n_pos ? C::STAGES : n_pos;
  for (; s < n_pos; ++s) {
    const int stage = s % C::STAGES, round = s / C::STAGES;
    if (!mbar_wait(&empty[stage], (round - 1) & 1, abort_flag, st, site)) break;
    mbar_arrive_expect_tx(&full[stage], C::TILE);
    load(s, stage, &full[stage]);
  }
  for (int q = s - C::STAGES; q < s; ++q)
    if (q >= 0) mbar_drain(&full[q % C::STAGES], (q / C::STAGES) & 1);
}

// The codes of the warp's 32 rows of a product tile (tb: the warp's lane
// quarter and the tile's first column), scale sc: into the warp's staging
// buffer cbuf (row = lane; 16-byte chunk j at its swizzled place in box j / 8),
// then TMA stores by lane 0, store_box(box, x) for each box of 32 rows (x: its
// first column), which clip rows past the tensor's end. The buffer is written
// again only once the previous stores have read it.
template <int D, bool ROT, typename StoreBox>
__device__ __forceinline__ void warp_codes_out(uint32_t tb, float sc, uint8_t* cbuf, int lane, StoreBox&& store_box) {
  using C = RotQuantCfg<D>;
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
  row_codes<D, ROT>(tb, sc, [&](int j, const uint4& v) {
    uint8_t* p = D == 64 ? cbuf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)  // 64-byte swizzle
                         : cbuf + (j >> 3) * (32 * 128) + lane * 128 + (((j & 7) ^ (lane & 7)) << 4);
    *reinterpret_cast<uint4*>(p) = v;
  });
  fence_proxy_async_shared();  // the TMA stores read the buffer through the async proxy
  __syncwarp();
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < C::NBOX; ++h) store_box(cbuf + h * (32 * C::CROW), h * C::CROW);
    bulk_commit();
  }
}

// ---------------------------------------------------------------------------
// One scale per tensor, up to kQuantBatch tensors of `rows` rows, in one
// cooperative launch. Each tensor takes two passes over this CTA's tiles (c,
// c + G, ...): pass 1 reduces the amax, a bounded grid barrier publishes it,
// pass 2 takes the same tiles in reverse order (the last ones read are still
// in L2) and writes the codes. The next tensor's pass 1 starts ahead of this
// tensor's pass 2, so that the HBM reads cover the grid barrier. Positions of a
// CTA with `per` tiles per tensor and a lead of m tiles (0 <= m <= per):
//   phase 0          : pass 1 of tensor 0;
//   phase k (1..n-1) : the first m tiles of pass 1 of tensor k, pass 2 of
//                      tensor k-1, the rest of pass 1 of tensor k;
//   phase n          : pass 2 of tensor n-1.
// The host takes m = per (all of the next pass 1 first) when two tensors fit
// in L2 together, else a short lead, so that pass 2 still finds its tensor in
// L2. Phases are not mixed tile by tile: the ring of STAGES tiles bounds the
// bytes in flight, and an L2 tile between HBM tiles would take a slot from them.
// Epilogue group g takes the positions of parity g. The grid barriers are
// handled by a sync warp (warp 10), so that their global-memory round trips,
// slow while HBM is saturated, stall no epilogue warp: a warp posts its pass-1
// max of tensor t to shared memory (an mbarrier arrival) as soon as it is past
// its pass-1 tiles of t; the sync warp reduces the CTA's max, publishes it,
// arrives at counter t, waits for all G CTAs and posts the tensor's amax; a
// warp waits for that only at its first pass-2 tile of t, which the m pass-1
// tiles opening each phase usually cover, so the loads keep streaming. Max
// before the 1/sqrt(d) factor, multiplied once: fp32 rounding is monotonic, so
// max_i fl(|v_i| c) = fl(c max_i |v_i|).
//
// amax_words[0 .. n-1]: the tensors' amax bits, counters[0 .. n-1]: the CTAs
// arrived at each tensor's barrier; all zero at launch. descale_out[t]: tensor
// t's descale.
// ---------------------------------------------------------------------------
struct QuantPos {
  int t, pass, i;  // tensor, pass (1 or 2), index among the CTA's tiles of the pass
};

// Position s of a CTA with `per` tiles per tensor, n tensors, lead m (schedule above).
__device__ __forceinline__ QuantPos quant_pos(int s, int per, int n, int m) {
  if (s < per) return {0, 1, s};
  s -= per;
  const int k = s / (2 * per) + 1;  // phase
  if (k == n) return {n - 1, 2, s - 2 * per * (n - 1)};
  const int o = s % (2 * per);
  if (o < m) return {k, 1, o};
  if (o < m + per) return {k - 1, 2, o - m};
  return {k, 1, o - per};
}

constexpr int kQuantSyncWarp = 10;  // quant_tensor_kernel: the warp that runs the grid barriers

template <int D, bool ROT>
__global__ void __launch_bounds__(RotQuantCfg<D>::THREADS + 32, 1)
quant_tensor_kernel(const __grid_constant__ QuantMaps qm, int rows, int lead, const float* __restrict__ signs,
                    unsigned int* amax_words, unsigned int* counters, float* descale_out) {
  using C = RotQuantCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* hm = smem;
  uint8_t* codes = smem + C::HMAT;
  uint8_t* ring = smem + C::HMAT + C::CODES;
  __shared__ __align__(8) uint64_t full[C::STAGES], empty[C::STAGES], tfull[C::NBUF], tfree[C::NBUF], drain;
  // bar_max[t]: the 8 epilogue warps have posted their pass-1 maxima of tensor
  // t; bar_amax[t]: the sync warp has posted tensor t's amax
  __shared__ __align__(8) uint64_t bar_max[kQuantBatch], bar_amax[kQuantBatch];
  __shared__ uint32_t tmem_slot;
  __shared__ float warp_max[kQuantBatch][C::EPI_WARPS];
  __shared__ float tensor_amax[kQuantBatch];
  __shared__ volatile int abort_flag;
  DevStatus* st = &g_fa_status;
  const int warp = static_cast<int>(warp_id()), lane = static_cast<int>(lane_id());
  const int ntile = (rows + C::BM - 1) / C::BM;
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int per = c < ntile ? (ntile - 1 - c) / G + 1 : 0;  // this CTA's tiles per tensor
  const int n = qm.n, n_pos = 2 * per * n;
  const int m = lead < per ? lead : per;
  // the tile of pass p's i-th position: c + i G in pass 1, in reverse in pass 2
  auto tile_of = [&](const QuantPos& q) { return c + (q.pass == 1 ? q.i : per - 1 - q.i) * G; };
  // L2 policies (producer thread): a tile read in pass 1 stays in L2 for its
  // pass 2 while the next tensor streams in; the pass-2 read lets it go.
  uint64_t pol_keep = 0, pol_drop = 0;
  if (warp == C::TMA_WARP && lane == 0) {
    pol_keep = l2_policy_evict_last();
    pol_drop = l2_policy_evict_first();
  }
  auto load = [&](int s, int stage, uint64_t* bar) {
    const QuantPos q = quant_pos(s, per, n, m);
    const int r0 = tile_of(q) * C::BM;
    const uint64_t pol = q.pass == 1 ? pol_keep : pol_drop;
#pragma unroll
    for (int col = 0; col < C::COLS; ++col)
      tma_load_2d_hint(ring + stage * C::TILE + col * (C::BM * 128), &qm.x[q.t], bar, col * 64, r0, pol);
  };
  if (warp == kQuantSyncWarp && lane == 0) {
    for (int t = 0; t < kQuantBatch; ++t) {
      mbar_init(&bar_max[t], C::EPI_WARPS);
      mbar_init(&bar_amax[t], 1);
    }
    // made visible to the other threads by the set-up's __syncthreads
  }
  const uint32_t tbase = rot_quant_setup<D, ROT>(hm, signs, full, empty, tfull, tfree, &drain, &tmem_slot,
                                                 &abort_flag, n_pos, load);

  if (warp == C::TMA_WARP) {
    if (lane == 0) rot_quant_producer<D>(n_pos, full, empty, &abort_flag, st, 61, load);
  } else if (warp == C::MMA_WARP) {
    if (lane == 0)
      rot_quant_mma_loop<D>(n_pos, smem_u32(ring), smem_u32(hm), tbase, full, empty, tfull, tfree, &drain,
                            &abort_flag, st, 62);
  } else if (warp == kQuantSyncWarp) {
    // ---------------------------------------------------------- grid barriers --
    if (lane == 0) {
      for (int t = 0; t < n; ++t) {
        // the CTA's max (a failed wait leaves what has been posted)
        mbar_wait(&bar_max[t], 0, &abort_flag, st, 67);
        float cm = 0.f;
#pragma unroll
        for (int w = 0; w < C::EPI_WARPS; ++w) cm = fmaxf(cm, warp_max[t][w]);
        // Fire-and-forget reductions: the arrival is a release, so the max
        // before it is visible to whoever acquires the count it completes.
        const unsigned int bits = __float_as_uint(ROT ? cm * C::INV_SQRT_D : cm);
        asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(amax_words + t), "r"(bits) : "memory");
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(counters + t) : "memory");
        // Every CTA is resident (cooperative launch). The wait is bounded; if it
        // runs out the status word records it and the CTA goes on.
        const unsigned long long t0 = globaltimer_ns();
        unsigned int arrived;
        for (;;) {
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(arrived) : "l"(counters + t) : "memory");
          if (arrived >= static_cast<unsigned int>(G)) break;
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            if (atomicCAS(&st->code, 0u, 5u) == 0u) {
              st->site = 60;
              st->block = blockIdx.x;
            }
            break;
          }
        }
        unsigned int a;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(a) : "l"(amax_words + t) : "memory");
        tensor_amax[t] = __uint_as_float(a);
        mbar_arrive(&bar_amax[t]);  // release: the amax is visible to the waiters
        if (blockIdx.x == 0) descale_out[t] = __uint_as_float(a) > 0.f ? __uint_as_float(a) / 448.0f : 1.0f;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int g = warp >> 2, q = warp & 3;  // group, lane quarter
    uint8_t* cbuf = codes + warp * C::CBUF;
    const uint64_t pol_codes = l2_policy_evict_first();  // the codes are not read again here
    bool ok = true;
    int pub = 0;      // tensors whose pass-1 max this warp has posted
    int known = 0;    // tensors whose amax this warp has taken
    float mx = 0.f;   // this thread's pass-1 max of tensor `pub`
    float sc = 1.0f;  // scale of tensor known - 1
    auto post = [&]() {  // this warp's max of tensor pub
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) {
        warp_max[pub][warp] = mx;
        mbar_arrive(&bar_max[pub]);  // release: the max is visible to the sync warp
      }
      mx = 0.f;
      ++pub;
    };
    auto take = [&]() {  // tensor known's amax, once the sync warp has it
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&bar_amax[known], 0, &abort_flag, st, 68));
      const float amax = tensor_amax[known];
      sc = amax > 0.f ? 448.0f / amax : 1.0f;
      ++known;
    };
    for (int s = g; s < n_pos && ok; s += 2) {
      const QuantPos p = quant_pos(s, per, n, m);
      // past the pass-1 tiles of every tensor before this position's (pass 1),
      // or of this position's tensor too (pass 2)
      while (pub < (p.pass == 1 ? p.t : p.t + 1)) post();
      if (p.pass == 2)
        while (known <= p.t && ok) take();
      if (!ok) break;
      const int buf = s % C::NBUF;
      ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], (s / C::NBUF) & 1, &abort_flag, st, 63));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tbase + (static_cast<uint32_t>(32 * q) << 16) + buf * D;
      if (p.pass == 1) {
        mx = fmaxf(mx, row_absmax<D, ROT>(tb));
      } else {
        const int row0 = tile_of(p) * C::BM + 32 * q;  // the warp's first row
        warp_codes_out<D, ROT>(tb, sc, cbuf, lane,
                               [&](uint8_t* b, int x) { tma_store_2d_hint(&qm.y[p.t], b, x, row0, pol_codes); });
      }
      tc_fence_before();  // the tile's tensor memory may be overwritten
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfree[buf]);
    }
    // every tensor's max is posted (also after a failed wait), so that the sync
    // warp, and through it the other CTAs, are not left waiting
    while (pub < n) post();
    if (lane == 0) bulk_wait_all();  // the code stores have completed before the CTA exits
  }
  // every role is done with tensor memory (the issuer has drained its products)
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------
// One scale per 128-row block of a head, in one pass (every scale depends on
// one tile): persistent CTAs over the tiles (head, block) of a [BH][N][D]
// tensor map, rows past N zero-filled by TMA. The four warps of the tile's
// epilogue group reduce its amax through shared memory and a named barrier of
// their own, then write its codes and descale.
// ---------------------------------------------------------------------------
template <int D, bool ROT>
__global__ void __launch_bounds__(RotQuantCfg<D>::THREADS, 1)
quant_block_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmy, int BH, int N,
                   const float* __restrict__ signs, float* __restrict__ descales) {
  using C = RotQuantCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* hm = smem;
  uint8_t* codes = smem + C::HMAT;
  uint8_t* ring = smem + C::HMAT + C::CODES;
  __shared__ __align__(8) uint64_t full[C::STAGES], empty[C::STAGES], tfull[C::NBUF], tfree[C::NBUF], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ float red[2][2][4];  // [group][tile parity][warp]: per-warp maxima
  __shared__ volatile int abort_flag;
  DevStatus* st = &g_fa_status;
  const int warp = static_cast<int>(warp_id()), lane = static_cast<int>(lane_id());
  const int nt = (N + C::BM - 1) / C::BM;  // tiles (scale blocks) per head
  const long long units = static_cast<long long>(BH) * nt;
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int K = c < units ? static_cast<int>((units - 1 - c) / G + 1) : 0;  // this CTA's tiles
  // position i: unit u = c + i G, head u / nt, block u % nt
  auto load = [&](int i, int stage, uint64_t* bar) {
    const long long u = c + static_cast<long long>(i) * G;
    const int bh = static_cast<int>(u / nt), r0 = static_cast<int>(u % nt) * C::BM;
#pragma unroll
    for (int col = 0; col < C::COLS; ++col)
      tma_load_3d(ring + stage * C::TILE + col * (C::BM * 128), &tmx, bar, col * 64, r0, bh);
  };
  const uint32_t tbase =
      rot_quant_setup<D, ROT>(hm, signs, full, empty, tfull, tfree, &drain, &tmem_slot, &abort_flag, K, load);

  if (warp == C::TMA_WARP) {
    if (lane == 0) rot_quant_producer<D>(K, full, empty, &abort_flag, st, 64, load);
  } else if (warp == C::MMA_WARP) {
    if (lane == 0)
      rot_quant_mma_loop<D>(K, smem_u32(ring), smem_u32(hm), tbase, full, empty, tfull, tfree, &drain,
                            &abort_flag, st, 65);
  } else {
    const int g = warp >> 2, q = warp & 3, r = 32 * q + lane;
    uint8_t* cbuf = codes + warp * C::CBUF;
    for (int i = g; i < K; i += 2) {
      const int buf = i % C::NBUF;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], (i / C::NBUF) & 1, &abort_flag, st, 66));
      const uint32_t tb = tbase + (static_cast<uint32_t>(32 * q) << 16) + buf * D;
      float m = 0.f;
      if (ok) {
        tc_fence_after();
        m = row_absmax<D, ROT>(tb);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int par = (i >> 1) & 1;
      if (lane == 0) red[g][par][q] = m;
      // the group's four warps leave together if any of them gave up waiting
      if (named_barrier_sync_or(2 + g, 128, !ok)) break;
      float amax = fmaxf(fmaxf(red[g][par][0], red[g][par][1]), fmaxf(red[g][par][2], red[g][par][3]));
      if (ROT) amax *= C::INV_SQRT_D;
      const long long u = c + static_cast<long long>(i) * G;
      const int bh = static_cast<int>(u / nt), blk = static_cast<int>(u % nt);
      if (r == 0) descales[static_cast<long long>(bh) * nt + blk] = amax > 0.f ? amax / 448.0f : 1.0f;
      const int row0 = blk * C::BM + 32 * q;  // the warp's first row in the head
      warp_codes_out<D, ROT>(tb, amax > 0.f ? 448.0f / amax : 1.0f, cbuf, lane,
                             [&](uint8_t* b, int x) { tma_store_3d(&tmy, b, x, row0, bh); });
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfree[buf]);
    }
    if (lane == 0) bulk_wait_all();  // the code stores have completed before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace fa

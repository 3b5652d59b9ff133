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
//  * a work item = NQ query tiles of 128 rows of one (batch, head); NQ = 2 for
//    d <= 128 so that the softmax of one tile overlaps the tensor-core work of
//    the other (the pages' "ping-pong", section "Inovações técnicas", 1). CTAs
//    are persistent where the host says so (one per SM, looping over items, the
//    next item's Q load overlapping the current item's tail);
//  * warp roles (section "Inovações técnicas", 1, producer/consumer warps):
//      warps 0..4*NQ-1 : softmax, one thread per query row, one warpgroup per tile;
//      warp 4*NQ       : tcgen05.mma issuer (one elected thread), TMEM owner;
//      warp 4*NQ+1     : TMA producer (Q once; K_j, V_j through a ring of
//                        shared-memory slots, prefetched ahead: section 2);
//      warps 4*NQ+2,3  : idle (they complete the last warpgroup for setmaxnreg);
//  * S_t = Q_t K_jᵀ accumulates in TMEM (128 fp32 columns); softmax reads it
//    in four 32-column chunks, each load overlapping the previous chunk's exps,
//    writes P_t = exp2(..) as bf16 pairs over the first 64 columns, and the MMA
//    warp issues O_t += P_t V_j with P_t taken straight from TMEM;
//  * online softmax in base 2 with the scale folded into one FMA; the reference
//    max is moved only when a row's max grows by more than 8 (log2 units),
//    which a tile weight sum above 2^8 reveals without a per-key running max, so
//    the O rescale (a TMEM read-modify-write) is rare. The final O / l and the
//    LSE use the same reference, so the result is exact, not approximated;
//  * the QK product can take e4m3 Q and K (the FP8 path with Hadamard-rotated
//    inputs: section "Inovações técnicas", 3); P and V stay bf16. Under QROT the
//    kernel rotates and quantises its own bf16 query tiles: the MMA warp
//    multiplies each tile by the signed Hadamard operand (hadamard.cuh) into
//    the tile's S columns, and the tile's softmax warpgroup turns the product
//    into e4m3 codes in place of the bf16 tile.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "hadamard.cuh"
#include "sm100.cuh"

namespace fa {

#ifndef FA_REG_SOFTMAX
#define FA_REG_SOFTMAX 208
#endif
#ifndef FA_REG_OTHER
#define FA_REG_OTHER 88
#endif

// QROT: Q arrives in bf16 and each query tile is rotated (on the tensor core,
// into its S columns) and quantised to e4m3 (one scale per tile, by its softmax
// warpgroup, in place in shared memory) before its first Q Kᵀ; K is e4m3 with
// one scale per 128-key tile.
template <int D, int NQ, bool QK_FP8, bool QROT = false>
struct FwdCfg {
  static constexpr int BM = 128;  // query rows per tile (TMEM lanes)
  static constexpr int BN = 128;  // keys per K/V tile
  static constexpr int EQK = QK_FP8 ? 1 : 2;
  static constexpr int QK_CHUNKS = D * EQK / 128;  // 128-byte swizzle columns per Q/K row (MMA operands)
  static constexpr int V_CHUNKS = D * 2 / 128;
  // Q as loaded: bf16 under QROT (converted in place: the e4m3 tile is the
  // first BM * D bytes of the slot), else the MMA's own element type
  static constexpr int Q_LOAD_CHUNKS = QROT ? D * 2 / 128 : QK_CHUNKS;
  static constexpr int Q_LOAD_ELEMS = QROT ? 64 : 128 / EQK;  // elements per 128-byte column
  static constexpr int Q_TILE = BM * D * (QROT ? 2 : EQK);
  static_assert(!QROT || (QK_FP8 && D == 128), "Q is rotated and quantised in the kernel for e4m3, d = 128");
  static constexpr int K_TILE = BN * D * EQK;
  static constexpr int V_TILE = BN * D * 2;
  static constexpr int SLOT = V_TILE;  // a ring slot holds one K or one V tile
  static constexpr int RING_BUDGET = 200 * 1024 - NQ * Q_TILE;
  static constexpr int NSLOT = (RING_BUDGET / SLOT) > 6 ? 6 : (RING_BUDGET / SLOT);
  static constexpr int ROT_OP = QROT ? HadCfg<D>::HMAT : 0;  // the rotation operand (QROT)
  static constexpr int SMEM_BYTES = 1024 + NQ * Q_TILE + ROT_OP + NSLOT * SLOT;
  // O staging (direct-mode epilogue): OST_COLS columns of a query tile's O as
  // bf16, 64-column boxes of 128 rows with the 128-byte swizzle, written to
  // global memory by TMA stores; D / OST_COLS rounds per tile. For the bf16
  // kernels, where it fits beside the rest, without causal masking
  // (fwd_ostage). (Measured on B200: +4% at N = 512, neutral at N >= 4096 for
  // non-causal bf16; 1-2% slower for causal launches and for the e4m3-QK kernel
  // at B=2, H=16, N=8192, which keep their per-row stores.)
  static constexpr int OST_COLS = D < 128 ? D : 128;
  static constexpr int OST_ROUNDS = D / OST_COLS;
  static constexpr int OST_BOXES = OST_COLS / 64;
  static constexpr bool OST_FITS = !QK_FP8 && SMEM_BYTES + BM * OST_COLS * 2 <= 225 * 1024;
  static constexpr int OST_BYTES = OST_FITS ? BM * OST_COLS * 2 : 0;
  // dynamic shared memory of a launch (direct: O goes through the staging buffer)
  static constexpr int smem_bytes(bool direct) { return SMEM_BYTES + (direct ? OST_BYTES : 0); }
  static constexpr int SOFTMAX_WARPS = 4 * NQ;
  static constexpr int MMA_WARP = SOFTMAX_WARPS;
  static constexpr int TMA_WARP = SOFTMAX_WARPS + 1;
  static constexpr int THREADS = (SOFTMAX_WARPS + 4) * 32;  // whole warpgroups
  // NQ = 2 (384 threads) launches at 168 registers per thread; setmaxnreg then
  // moves registers from the last warpgroup to the two softmax warpgroups.
  static constexpr bool SPLIT_REGS = NQ == 2;
  static constexpr int REG_LAUNCH = 168;   // 65536 / 384 rounded down to a multiple of 8
  static constexpr int REG_SOFTMAX = FA_REG_SOFTMAX;  // per softmax thread after setmaxnreg.inc
  static constexpr int REG_OTHER = FA_REG_OTHER;      // per thread of the last warpgroup after .dec
  static_assert(!SPLIT_REGS || SOFTMAX_WARPS * 32 * REG_SOFTMAX + 128 * REG_OTHER <= THREADS * REG_LAUNCH,
                "register split exceeds the block's launch allocation");
  // TMEM columns: S (128 fp32 per tile) then O (D per tile), allocated as a power of two.
  static constexpr uint32_t TMEM_COLS = NQ * (128 + D) <= 256 ? 256u : 512u;
  static constexpr uint32_t S_COL(int t) { return static_cast<uint32_t>(t) * 128u; }
  static constexpr uint32_t P_COL(int t) { return S_COL(t); }  // 64 columns of bf16 pairs over S
  static constexpr uint32_t O_COL(int t) { return static_cast<uint32_t>(NQ) * 128u + static_cast<uint32_t>(t * D); }
  static_assert(D == 64 || D == 128 || D == 256, "head dim");
  static_assert(QK_CHUNKS >= 1, "an e4m3 row must fill a 128-byte swizzle row");
  static_assert(NSLOT >= 2, "ring needs two slots");
  static_assert(NQ * 128 + NQ * D <= 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  // Two co-resident CTAs must not both want all 512 TMEM columns.
  static_assert(SMEM_BYTES > 114 * 1024 || TMEM_COLS <= 256, "TMEM of co-resident CTAs");
};

// Whether a forward kernel writes O through the staging buffer (FwdCfg::OST_*).
template <typename C, bool CAUSAL, bool PARTIAL, bool DEC>
__host__ __device__ constexpr bool fwd_ostage() {
  return C::OST_FITS && !CAUSAL && !PARTIAL && !DEC;
}

struct FwdParams {
  __nv_bfloat16* o;          // [BH][Nq][D]; null in partial mode
  float* lse;                // [BH][Nq], may be null
  float* o_part;             // partial mode: [n_split][BH][Nq][D] fp32, O of the split's keys; else null
  float* lse_part;           // partial mode: [n_split][BH][Nq], -inf where a row sees no key of the split
  const float* descale_qk;   // e4m3 path, one scale per tensor: {dq, dk}; else null
  // e4m3 path, one scale per 128-row block of a head (descale_qk unused):
  // dq_block[bh * nbq + query tile], dk_block[bh * nbk + key tile]; else null
  const float* dq_block;
  const float* dk_block;
  int nbq, nbk;
  // QROT: the d Hadamard signs of the rotation (null: none) and whether to
  // rotate at all; dq_out (may be null) receives each query tile's descale at
  // dq_out[bh * nbq + query tile]
  const float* qrot_signs;
  int qrot_rotate;
  float* dq_out;
  int BH;                    // batch * heads
  int Nq, Nk;                // query rows and keys per head
  int causal_off;            // Nk - Nq: key j is visible to query i iff j <= i + causal_off (causal)
  int n_qb;                  // query blocks (NQ*128 rows) per head
  int n_split;               // key splits per head (1: all keys)
  int split_tiles;           // key tiles per split
  float scale_log2;          // scale * log2(e)
  // Work items: the query blocks (query block = bh * n_qb + qb), times n_split
  // key blocks each in partial mode; n_items of them. CTA c takes items c,
  // c + gridDim.x, ... (persistent when the grid is smaller than n_items).
  int n_items;
  // snake (causal, persistent): item i is query block rank i / BH of head i % BH,
  // blocks ranked heaviest first across all heads, and CTA c takes item
  // r * gridDim.x + c in even rounds r, r * gridDim.x + gridDim.x - 1 - c in odd
  // ones, which balances work that decreases with i
  int snake;
  // Tail split (direct mode, non-causal, persistent): query blocks n_full ..
  // (units - 1), the blocks of a mostly empty last round, are computed as
  // tail_split pieces of tail_tiles key tiles each, as items n_full + k with
  // k = (block - n_full) * tail_split + piece, so that the round's CTAs share
  // them. Each warp of a piece writes its rows' O (fp32, normalised over the
  // piece's keys; [D/4][128][4] per piece and tile, so a warp's stores are
  // contiguous) and base-2 LSE to tail_o / tail_lse, then takes a ticket on its
  // group's word of tail_cnt (bits 8-63: tail_tag, a 56-bit value new for every
  // launch, so a word left by an aborted launch, or never written, counts as
  // zero; bits 0-7: pieces done). The warp whose ticket completes the group sets
  // the word back to zero, merges the pieces by their LSEs, in piece order
  // whichever piece it is, and writes O and the LSE; no warp waits for another.
  // n_full = number of query blocks (tail_split = 0) when there is no tail split.
  int n_full;
  int tail_split, tail_tiles;
  unsigned long long tail_tag;
  float* tail_o;
  float* tail_lse;
  unsigned long long* tail_cnt;
};

// Tail-split workspace of one (query tile, piece): the piece's normalised O,
// then (separately) its LSE per row.
template <int D>
__host__ __device__ constexpr size_t tail_o_floats() { return static_cast<size_t>(128) * D; }
constexpr int kTailMaxSplit = 4;

// One work item of a CTA: head, key split, first query row, first key tile and
// the key tiles its query tiles step through.
struct FwdItem {
  int bh, sp, q0, kt0, n_kv0, n_kv1, n_kv;
  int tail;  // tail-split query block index (its pieces' group), -1 if the item is whole
};

#ifndef FA_MMA_WAIT_SLEEP_NS
#define FA_MMA_WAIT_SLEEP_NS 0
#endif
// Suspend hint of the MMA issuer's wait for P (0: poll). Its wake-up latency is
// on the critical path, but a polling warp also takes issue slots from the two
// softmax warps on its sub-partition.
constexpr uint32_t kMmaWaitSleepNs = FA_MMA_WAIT_SLEEP_NS;

// Longest item (in key tiles) whose Q buffer is released right after its last
// S product rather than after its last P V product (non-causal launches).
// Measured on B200 (interleaved A/B): the early release gains 2-7% at N =
// 512-2048; on longer items it gained nothing, and on causal launches (whose
// snake order ends with short items) it cost 2-4%.
constexpr int kEarlyQMaxTiles = 24;

// Exponentials of one 32-key chunk of a row of S: p = 2^(x*s - m), packed to
// bf16 pairs into pk[0..15]; accumulates the fp32 weights, with ROUND also the
// bf16-rounded ones, into the packed-pair sums and (WITH_MAX) the raw-score max
// into mx[0..3].
template <bool WITH_MAX, bool ROUND = true>
__device__ __forceinline__ void exp_chunk32(const uint32_t* s, uint32_t* pk, uint64_t s2, uint64_t nm2,
                                            uint64_t* acc_e, uint64_t* acc_r, float* mx) {
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    float t0, t1, p0, p1;
    if (WITH_MAX) mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
    f2_unpack(f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), s2, nm2), t0, t1);
    p0 = ex2_approx(t0);
    p1 = ex2_approx(t1);
    const uint32_t q = pack_bf16x2(p0, p1);
    const int a = (c >> 1) & 1;
    acc_e[a] = f2_add(acc_e[a], f2_pack(p0, p1));
    if (ROUND) acc_r[a] = f2_add(acc_r[a], f2_pack(__uint_as_float(q << 16), __uint_as_float(q & 0xFFFF0000u)));
    pk[c >> 1] = q;
  }
}

__device__ __forceinline__ void mask_chunk32(uint32_t* s, int kbase, int kmax) {
#pragma unroll
  for (int c = 0; c < 32; ++c)
    if (kbase + c > kmax) s[c] = __float_as_uint(-INFINITY);
}

// One row of S (128 keys, from TMEM at tS) through the exponentials: the four
// 32-column loads are software-pipelined with the exps of the previous chunk
// (tcgen05.wait::ld waits for all earlier loads, so chunk c+1 is issued before
// chunk c is computed). P is packed in place: chunk c's 16 bf16 pairs go to
// s[16c .. 16c+15], scores already consumed (chunk c/2's) and never the target of
// a pending load, so only 128 registers are live. Returns the fp32 weight sum,
// and the sum that normalises O.
//
// The normalising sum is the sum of the bf16-rounded weights P holds when some
// key of the tile is masked (FULL false: the row's last tile, which holds every
// key of a row with few keys), else the fp32 sum: over a full tile of 128 keys
// the rounding errors of P average out to about 2^-9 / sqrt(128) of the sum, and
// skipping the rounded sum saves three of the eight instructions per key pair.
template <bool FULL>
__device__ __forceinline__ void softmax_row(uint32_t tS, uint32_t* s, float s_log2, float m_ref,
                                            int kbase, int kmax, bool masked, float& sum_e, float& sum_r) {
  const uint64_t s2 = f2_pack(s_log2, s_log2);
  const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
  uint64_t acc_e[2] = {0ull, 0ull}, acc_r[2] = {0ull, 0ull};
  float mx[4];  // unused: no running max
  tmem_ld32(tS + 0, &s[0]);
  tmem_wait_ld_dep32(&s[0]);
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    if (ch < 3) tmem_ld32(tS + 32 * (ch + 1), &s[32 * (ch + 1)]);
    if (masked) mask_chunk32(&s[32 * ch], kbase + 32 * ch, kmax);
    exp_chunk32<false, !FULL>(&s[32 * ch], &s[16 * ch], s2, nm2, acc_e, acc_r, mx);
    if (ch < 3) tmem_wait_ld_dep32(&s[32 * (ch + 1)]);
  }
  float e0, e1, e2, e3, r0, r1, r2, r3;
  f2_unpack(acc_e[0], e0, e1);
  f2_unpack(acc_e[1], e2, e3);
  f2_unpack(acc_r[0], r0, r1);
  f2_unpack(acc_r[1], r2, r3);
  sum_e = (e0 + e1) + (e2 + e3);
  sum_r = FULL ? sum_e : (r0 + r1) + (r2 + r3);
}

// `masked` must be warp-uniform: both paths issue tcgen05.ld.
__device__ __forceinline__ void softmax_row_dispatch(uint32_t tS, uint32_t* s, float s_log2, float m_ref, int kbase,
                                                     int kmax, bool masked, float& se, float& sr) {
  if (masked)
    softmax_row<false>(tS, s, s_log2, m_ref, kbase, kmax, true, se, sr);
  else
    softmax_row<true>(tS, s, s_log2, m_ref, kbase, kmax, false, se, sr);
}

// Raw-score max of one row of S (first tile only, before any reference exists).
__device__ __forceinline__ float row_max_tmem(uint32_t tS, uint32_t* s, int kbase, int kmax, bool masked) {
  float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
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

// Softmax warps of a DEC CTA (see attn_fwd_kernel): warp w, lane r holds query
// row r's online softmax over keys 32w .. 32w+31 of each key tile (TMEM lane
// 32w + r), then the four warps merge through shared memory.
template <int D, bool CAUSAL, bool QK_FP8, bool PARTIAL, typename C, typename P>
__device__ __forceinline__ void decode_softmax(const P& p, uint32_t tbase, uint32_t warp, uint32_t lane, int q0, int bh,
                                               int sp, int kt0, int n_kv, uint8_t* sbuf, uint64_t* bar_s,
                                               uint64_t* bar_p, uint64_t* bar_o, volatile int* abort_flag,
                                               DevStatus* st) {
  const int w = static_cast<int>(warp & 3u);  // key quarter
  const uint32_t row_addr = tbase + ((32u * w) << 16);
  const uint32_t tS = row_addr + C::S_COL(0) + 32u * w;  // this quarter's 32 columns of S
  const uint32_t tP = row_addr + C::P_COL(0);
  const uint32_t tO = row_addr + C::O_COL(0);
  const int qrow = q0 + static_cast<int>(lane);
  float s_q = p.scale_log2;
  const float* dkb = nullptr;
  if constexpr (QK_FP8) {
    if (p.dq_block != nullptr) {
      s_q *= __ldg(p.dq_block + static_cast<size_t>(bh) * p.nbq);  // Nq <= 32: query block 0
      dkb = p.dk_block + static_cast<size_t>(bh) * p.nbk + kt0;
    } else {
      s_q *= __ldg(p.descale_qk) * __ldg(p.descale_qk + 1);
    }
  }
  // last visible key, relative to this quarter's first key of the split's first tile
  const int kmax = (CAUSAL ? min(qrow + p.causal_off, p.Nk - 1) : p.Nk - 1) - kt0 * C::BN - 32 * w;
  float m_ref = -INFINITY, l_exact = 0.f, l_round = 0.f;
  bool ok = true;
  uint32_t zero[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) zero[i] = 0u;
  float dk_next = (QK_FP8 && dkb != nullptr && n_kv > 0) ? __ldg(dkb) : 1.0f;
  for (int j = 0; j < n_kv; ++j) {
    const float s_log2 = s_q * dk_next;
    if (QK_FP8 && dkb != nullptr && j + 1 < n_kv) dk_next = __ldg(dkb + j + 1);
    ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[0], j & 1, abort_flag, st, 50));
    if (!ok) break;
    tc_fence_after();
    uint32_t s[32];
    const int kbase = j * C::BN;  // this quarter's keys are kbase + 32w + c
    const bool masked = __any_sync(0xffffffffu, kbase + 31 > kmax);  // warp-uniform
    const uint64_t s2 = f2_pack(s_log2, s_log2);
    uint64_t acc_e[2] = {0ull, 0ull}, acc_r[2] = {0ull, 0ull};
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    float alpha = 1.0f;
    tmem_ld32(tS, s);
    tmem_wait_ld_dep32(s);
    if (masked) mask_chunk32(s, kbase, kmax);
    if (j == 0) {
      float a = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; c += 2) a = fmax3(a, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
      // a quarter with no visible key keeps reference 0 and zero weights (its
      // later tiles hold only later keys, so it stays empty)
      m_ref = a == -INFINITY ? 0.f : a * s_log2;
      const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
      exp_chunk32<false>(s, s, s2, nm2, acc_e, acc_r, mx);
    } else {
      uint32_t keep[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) keep[c] = s[c];
      const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
      exp_chunk32<true>(s, s, s2, nm2, acc_e, acc_r, mx);
      const float mx_s = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * s_log2;
      const bool grow = mx_s > m_ref + 8.0f;
      if (__any_sync(0xffffffffu, grow)) {
        const float m_new = grow ? mx_s : m_ref;
        alpha = ex2_approx(m_ref - m_new);
        m_ref = m_new;
        acc_e[0] = acc_e[1] = acc_r[0] = acc_r[1] = 0ull;
        const uint64_t nm2b = f2_pack(-m_ref, -m_ref);
        exp_chunk32<false>(keep, s, s2, nm2b, acc_e, acc_r, mx);
        // rescale this warp's O rows (PV of the previous tile has completed)
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
    float e0, e1, e2, e3, r0, r1, r2, r3;
    f2_unpack(acc_e[0], e0, e1);
    f2_unpack(acc_e[1], e2, e3);
    f2_unpack(acc_r[0], r0, r1);
    f2_unpack(acc_r[1], r2, r3);
    l_exact = l_exact * alpha + ((e0 + e1) + (e2 + e3));
    l_round = l_round * alpha + ((r0 + r1) + (r2 + r3));
    // P: this quarter's 16 bf16-pair columns, zeros in the other three quarters
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (q == w)  // warp-uniform
        tmem_st16(tP + 16u * q, s);
      else
        tmem_st16(tP + 16u * q, zero);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_p[0]);
  }
  if (ok && n_kv > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar_o[0], 0, abort_flag, st, 51));
  if (n_kv > 0) tc_fence_after();
  // Merge the four quarters of each row: stats through static shared memory,
  // then warps 1-3 hand their scaled O rows to warp 0 through the (now idle)
  // K/V ring. Every softmax thread passes both barriers.
  __shared__ float stat[3][4][32];
  stat[0][w][lane] = m_ref;
  stat[1][w][lane] = l_exact;
  stat[2][w][lane] = l_round;
  named_barrier_sync(1, 128);
  float M = -INFINITY;
#pragma unroll
  for (int u = 0; u < 4; ++u)
    if (stat[1][u][lane] > 0.f) M = fmaxf(M, stat[0][u][lane]);
  float le = 0.f, lr = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float a = stat[1][u][lane] > 0.f ? ex2_approx(stat[0][u][lane] - M) : 0.f;
    le += a * stat[1][u][lane];
    lr += a * stat[2][u][lane];
  }
  const float my_a = l_exact > 0.f ? ex2_approx(m_ref - M) : 0.f;
  const bool empty = le == 0.f;  // no visible key in any quarter (partial mode only)
  const float inv = empty ? 0.f : 1.0f / lr;
  const bool in_range = qrow < p.Nq;
  float* buf = reinterpret_cast<float*>(sbuf);  // [3][32][D]: quarters 1..3
  if (w > 0 && ok && n_kv > 0) {
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t ov[32];
      tmem_ld32(tO + c0, ov);
      tmem_wait_ld_dep32(ov);
      if (in_range) {
        float4* dst = reinterpret_cast<float4*>(buf + ((w - 1) * 32 + lane) * D + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(ov[4 * i]) * my_a, __uint_as_float(ov[4 * i + 1]) * my_a,
                               __uint_as_float(ov[4 * i + 2]) * my_a, __uint_as_float(ov[4 * i + 3]) * my_a);
      }
    }
  }
  named_barrier_sync(1, 128);
  if (w != 0 || !ok) return;
  const bool any = n_kv > 0;
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t ov[32];
    if (any) {
      tmem_ld32(tO + c0, ov);
      tmem_wait_ld_dep32(ov);
    }
    if (!in_range) continue;
    float o[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = any ? __uint_as_float(ov[i]) * my_a : 0.f;
    if (any) {
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const float4* src = reinterpret_cast<const float4*>(buf + (u * 32 + lane) * D + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 v = src[i];
          o[4 * i] += v.x; o[4 * i + 1] += v.y; o[4 * i + 2] += v.z; o[4 * i + 3] += v.w;
        }
      }
    }
    if constexpr (PARTIAL) {
      float4* dst = reinterpret_cast<float4*>(p.o_part + ((static_cast<size_t>(sp) * p.BH + bh) * p.Nq + qrow) * D + c0);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(bh) * p.Nq + qrow) * D + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_uint4(pack_bf16x2(o[8 * i] * inv, o[8 * i + 1] * inv), pack_bf16x2(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                            pack_bf16x2(o[8 * i + 4] * inv, o[8 * i + 5] * inv), pack_bf16x2(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
    }
  }
  if (!in_range) return;
  const float lse = empty ? -INFINITY : (M + __log2f(le)) * 0.69314718055994530942f;
  if constexpr (PARTIAL)
    p.lse_part[(static_cast<size_t>(sp) * p.BH + bh) * p.Nq + qrow] = lse;
  else if (p.lse != nullptr)
    p.lse[static_cast<size_t>(bh) * p.Nq + qrow] = lse;
}

// Epilogue of a tail-split piece for one warp's 32 query rows (see FwdParams):
// the piece's O (TMEM, weights relative to m_ref, summing to l_round) and LSE
// go to the workspace, the warp takes a ticket, and the warp whose ticket
// completes its group merges every piece by its LSE (the same combination as
// the blocks of a split: O = sum_k 2^(lse_k - L) O_k, L = log2 sum_k 2^lse_k)
// into the bf16 output and the natural-log LSE. The merge takes the pieces in
// index order, its own normalised O recomputed with the rounding it was stored
// with, so the result does not depend on which piece finished last. The CAS
// loop is not a wait: each failed attempt means another piece's ticket went in,
// so it ends within tail_split attempts; the bound only guards the status path.
template <int D, int NQ>
__device__ __forceinline__ void tail_piece_epilogue(const FwdParams& p, const FwdItem& w, int t, uint32_t warp_in_tile,
                                                 uint32_t lane, uint32_t tO, int r, int qrow, float m_ref,
                                                 float l_exact, float l_round, DevStatus* st) {
  const int ns = p.tail_split;
  const size_t grp = static_cast<size_t>(w.tail) * NQ + t;  // (tail block, query tile)
  float* const o_base = p.tail_o + grp * ns * tail_o_floats<D>();
  float* const l_base = p.tail_lse + grp * ns * 128;
  const float inv_l = 1.0f / l_round;
  const float lse2 = m_ref + __log2f(l_exact);  // base 2
  float4* const mine = reinterpret_cast<float4*>(o_base + w.sp * tail_o_floats<D>());
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t ov[32];
    tmem_ld32(tO + c0, ov);
    tmem_wait_ld_dep32(ov);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      mine[(c0 / 4 + i) * 128 + r] = make_float4(
          __fmul_rn(__uint_as_float(ov[4 * i]), inv_l), __fmul_rn(__uint_as_float(ov[4 * i + 1]), inv_l),
          __fmul_rn(__uint_as_float(ov[4 * i + 2]), inv_l), __fmul_rn(__uint_as_float(ov[4 * i + 3]), inv_l));
  }
  l_base[w.sp * 128 + r] = lse2;
  __threadfence();  // this lane's results before the ticket (release side)
  __syncwarp();
  unsigned int done = 0;
  if (lane == 0) {
    unsigned long long* cnt = p.tail_cnt + grp * 4 + warp_in_tile;
    unsigned long long cur = atomicAdd(cnt, 0ull);
    for (int a = 0; a < 64 && done == 0; ++a) {
      const unsigned long long base = (cur >> 8) == p.tail_tag ? cur : (p.tail_tag << 8);
      const unsigned long long got = atomicCAS(cnt, cur, base + 1ull);
      if (got == cur) done = static_cast<unsigned int>((base + 1ull) & 0xffull);
      cur = got;
    }
    if (done == 0 && atomicCAS(&st->code, 0u, 5u /*FA_ERR_TIMEOUT*/) == 0u) {
      st->site = 45;
      st->block = blockIdx.x;
    }
  }
  done = __shfl_sync(0xffffffffu, done, 0);
  if (done != static_cast<unsigned int>(ns)) return;  // warp-uniform
  // Every piece has its ticket: the word goes back to zero, so that the next
  // launch starts from zero even with this launch's tag (a replayed CUDA graph
  // launches with the parameters it was captured with).
  if (lane == 0) atomicExch(p.tail_cnt + grp * 4 + warp_in_tile, 0ull);
  __threadfence();  // acquire side: the other pieces' results, read through L2 below
  float lk[kTailMaxSplit], wk[kTailMaxSplit];
  float mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < kTailMaxSplit; ++k) {
    lk[k] = k < ns ? (k == w.sp ? lse2 : __ldcg(l_base + k * 128 + r)) : -INFINITY;
    mx = fmaxf(mx, lk[k]);
  }
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < kTailMaxSplit; ++k) sum += k < ns ? exp2f(lk[k] - mx) : 0.f;
  const float L = mx + log2f(sum);
#pragma unroll
  for (int k = 0; k < kTailMaxSplit; ++k) wk[k] = k < ns ? exp2f(lk[k] - L) : 0.f;
  const bool in_range = qrow < p.Nq;
  __nv_bfloat16* orow = p.o + (static_cast<size_t>(w.bh) * p.Nq + (in_range ? qrow : 0)) * D;
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t ov[32];
    tmem_ld32(tO + c0, ov);
    tmem_wait_ld_dep32(ov);
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll
    for (int k = 0; k < kTailMaxSplit; ++k) {
      if (k >= ns) continue;
      const float4* src = reinterpret_cast<const float4*>(o_base + k * tail_o_floats<D>());
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 v;
        if (k == w.sp) {
          v = make_float4(__fmul_rn(__uint_as_float(ov[4 * i]), inv_l), __fmul_rn(__uint_as_float(ov[4 * i + 1]), inv_l),
                          __fmul_rn(__uint_as_float(ov[4 * i + 2]), inv_l),
                          __fmul_rn(__uint_as_float(ov[4 * i + 3]), inv_l));
        } else {
          v = __ldcg(src + (c0 / 4 + i) * 128 + r);
        }
        acc[4 * i] = __fmaf_rn(wk[k], v.x, acc[4 * i]);
        acc[4 * i + 1] = __fmaf_rn(wk[k], v.y, acc[4 * i + 1]);
        acc[4 * i + 2] = __fmaf_rn(wk[k], v.z, acc[4 * i + 2]);
        acc[4 * i + 3] = __fmaf_rn(wk[k], v.w, acc[4 * i + 3]);
      }
    }
    if (in_range) {
      uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_uint4(pack_bf16x2(acc[8 * i], acc[8 * i + 1]), pack_bf16x2(acc[8 * i + 2], acc[8 * i + 3]),
                            pack_bf16x2(acc[8 * i + 4], acc[8 * i + 5]), pack_bf16x2(acc[8 * i + 6], acc[8 * i + 7]));
    }
  }
  if (in_range && p.lse != nullptr)
    p.lse[static_cast<size_t>(w.bh) * p.Nq + qrow] = L * 0.69314718055994530942f;
}

// Direct-mode epilogue of one warp's 32 rows of query tile t through the
// staging buffer (FwdCfg::OST_*): O / l in bf16 into 64-column boxes of 128 rows
// (128-byte swizzle), written by TMA stores that one thread of the tile issues
// (whole rows at once, rows past Nq clipped), then the LSE. The tiles take turns
// on the buffer (use u = (round * NQ + t) * OST_ROUNDS + part waits for the
// stores of use u - 1 to have read it); a tile with no rows takes its turn
// without writing, so the turns stay in step. Kept out of line: the softmax
// loop's registers and code are not shared with it. Returns ok.
template <int D, int NQ, typename C>
__device__ __noinline__ bool staged_o_epilogue(const CUtensorMap* tmO, uint8_t* sOst, uint64_t* bar_ost,
                                               uint64_t* bar_ofree, volatile int* abort_flag, DevStatus* st,
                                               float* lse, int Nq, uint32_t tO, int r, uint32_t lane, uint32_t warp,
                                               int t, int round, bool has, bool ok, float l_round, float l_exact,
                                               float m_ref, int q0, int bh, int qrow) {
  const bool issuer = (warp & 3u) == 0 && lane == 0;
  const float inv_l = has ? 1.0f / l_round : 0.f;
  if (ok && has) tc_fence_after();
#pragma unroll 1
  for (int part = 0; part < C::OST_ROUNDS && ok; ++part) {
    const int u = (round * NQ + t) * C::OST_ROUNDS + part;  // the buffer's use
    if (u > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_ofree, (u - 1) & 1, abort_flag, st, 46));
    if (!ok) break;
    if (has) {
#pragma unroll 1
      for (int cc = 0; cc < C::OST_COLS; cc += 32) {
        uint32_t ov[32];
        tmem_ld32(tO + part * C::OST_COLS + cc, ov);
        tmem_wait_ld_dep32(ov);
        uint32_t q[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          q[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
        // row r of the 64-column box holding these columns; 16-byte chunk c of
        // a row sits at c ^ (r mod 8) (the 128-byte swizzle)
        uint8_t* brow = sOst + (cc / 64) * (C::BM * 128) + r * 128;
        const int c0 = (cc % 64) / 8;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4*>(brow + (((c0 + i) ^ (r & 7)) << 4)) =
              make_uint4(q[4 * i], q[4 * i + 1], q[4 * i + 2], q[4 * i + 3]);
      }
      fence_proxy_async_shared();  // the TMA store reads the buffer through the async proxy
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_ost[t]);
    if (issuer) {
      ok = mbar_wait(&bar_ost[t], (round * C::OST_ROUNDS + part) & 1, abort_flag, st, 47 + t);
      if (ok) {
        if (has) {
#pragma unroll
          for (int b = 0; b < C::OST_BOXES; ++b)
            tma_store_3d(tmO, sOst + b * (C::BM * 128), part * C::OST_COLS + 64 * b, q0 + t * C::BM, bh);
          bulk_commit();
          bulk_wait_read_all();
        }
        mbar_arrive(bar_ofree);
      }
    }
    ok = __all_sync(0xffffffffu, ok);
  }
  if (ok && has && qrow < Nq && lse != nullptr)
    lse[static_cast<size_t>(bh) * Nq + qrow] = (m_ref + __log2f(l_exact)) * 0.69314718055994530942f;
  return ok;
}

// PARTIAL: the CTA's keys are one block of a split (p.n_split blocks) and it
// writes fp32 partial results (o_part, lse_part) instead of O and LSE.
//
// DEC (decode-shaped problems, Nq <= 32, one query tile): the Nq query rows are
// loaded four times, into TMEM lanes 0-31, 32-63, 64-95 and 96-127 of S and O
// (the Q tile map's box is 32 rows), and softmax warp w takes only keys
// 32w .. 32w+31 of every key tile for its copy of the rows: P is zero outside
// that quarter, so O lanes 32w+r accumulate query r's output over quarter w of
// the keys, each with its own online softmax. The epilogue merges the four by
// their maxima and sums (the same combination as for blocks of a split). A thread
// thus takes 32 exponentials per key tile instead of 128, which shortens the
// serial softmax -> P V -> S chain that bounds a CTA with one query tile.
template <int D, int NQ, bool CAUSAL, bool QK_FP8, bool PARTIAL, bool DEC, bool QROT = false>
__global__ void __launch_bounds__(FwdCfg<D, NQ, QK_FP8, QROT>::THREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const FwdParams p) {
  using C = FwdCfg<D, NQ, QK_FP8, QROT>;
  static_assert(!DEC || NQ == 1, "the decode layout uses one query tile");
  static_assert(!QROT || (!PARTIAL && !DEC && NQ == 2), "in-kernel Q quantisation: square launches only");
  static_assert(!DEC || C::NSLOT * C::SLOT >= 3 * 32 * D * 4, "decode merge buffer lives in the ring");
  // kernels that may take a tail split (the host sets it up only for these)
  constexpr bool TAIL = !PARTIAL && !DEC && !CAUSAL && !QROT;
  // direct-mode O through the staging buffer and TMA stores (tmO: O as
  // [BH][Nq][D] bf16, 64 x 128 boxes, 128-byte swizzle); non-causal only
  constexpr bool OSTAGE = fwd_ostage<C, CAUSAL, PARTIAL, DEC>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                // NQ tiles
  uint8_t* sRot = smem + NQ * C::Q_TILE;             // QROT: the rotation operand
  uint8_t* sRing = smem + NQ * C::Q_TILE + C::ROT_OP;  // NSLOT slots
  uint8_t* sOst = sRing + C::NSLOT * C::SLOT;          // OSTAGE: O staging

  __shared__ __align__(8) uint64_t bar_full[C::NSLOT], bar_empty[C::NSLOT];
  // bar_qfree: the S MMAs that read the current item's Q tiles are done (the
  // producer may load the next item's Q)
  __shared__ __align__(8) uint64_t bar_q, bar_qfree, bar_drain, bar_s[NQ], bar_p[NQ], bar_o[NQ];
  // QROT: bar_rot[t]: the product of query tile t and the rotation operand is
  // in its S columns (and the bf16 tile has been read); bar_qready[t]: query
  // tile t is in e4m3 (its warpgroup has converted it)
  // bar_qamax[t]: the four warps of tile t's warpgroup have posted their maxima
  __shared__ __align__(8) uint64_t bar_rot[NQ], bar_qready[NQ], bar_qamax[NQ];
  // OSTAGE: bar_ost[t]: the four warps of tile t have written their rows of the
  // staging buffer; bar_ofree: the TMA stores of the buffer's last use have read
  // it (the tiles use it in turn: use u = (round * NQ + t) * OST_ROUNDS + part)
  __shared__ __align__(8) uint64_t bar_ost[NQ], bar_ofree;
  __shared__ float qrot_red[NQ][4];  // per-warp maxima of each tile
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const uint32_t warp = warp_id(), lane = lane_id();

  // Work item `it`: head bh, key split sp, query block qb (heaviest causal blocks
  // of a head first). Key tiles of the split: kt0 .. kt0 + split_tiles - 1
  // (clipped to Nk). Query tile t steps through n_kv_of(t) of them: none if it
  // has no row (past Nq), else up to the tile holding its last visible key, so a
  // causal tile never spends a step on keys entirely in its future. The CTA
  // streams the most any tile needs.
  // The CTA's items: blockIdx.x + r * gridDim.x in round r, or the snake order.
  auto next_item = [&](int r) {
    const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    return r * g + ((p.snake && (r & 1)) ? g - 1 - c : c);
  };
  auto first_item = [&]() { return next_item(0); };
  auto item_at = [&](int it) {
    FwdItem w;
    const int n_split = PARTIAL ? p.n_split : 1;
    int unit = PARTIAL ? it / n_split : it;  // query block
    w.sp = PARTIAL ? it % n_split : 0;
    w.tail = -1;
    int span = PARTIAL ? p.split_tiles : 0;  // key tiles of a split block (0: all)
    if constexpr (TAIL) {
      if (it >= p.n_full) {
        const int k = it - p.n_full;
        w.tail = k / p.tail_split;
        w.sp = k - w.tail * p.tail_split;
        unit = p.n_full + w.tail;
        span = p.tail_tiles;
      }
    }
    w.bh = p.snake ? unit % p.BH : unit / p.n_qb;
    int qb = p.snake ? unit / p.BH : unit % p.n_qb;
    if (CAUSAL) qb = p.n_qb - 1 - qb;
    w.q0 = qb * NQ * C::BM;
    w.kt0 = w.sp * span;
    auto n_kv_of = [&](int t) {
      const int row0 = w.q0 + t * C::BM;
      if (row0 >= p.Nq) return 0;
      const int end = CAUSAL ? min(p.Nk, min(p.Nq, row0 + C::BM) + p.causal_off) : p.Nk;  // keys [0, end)
      const int tiles = (end + C::BN - 1) / C::BN;
      if (span == 0) return tiles;
      return max(0, min(tiles, w.kt0 + span) - w.kt0);
    };
    w.n_kv0 = n_kv_of(0);
    w.n_kv1 = NQ > 1 ? n_kv_of(NQ - 1) : w.n_kv0;
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
    mbar_init(&bar_ofree, 1);
    for (int t = 0; t < NQ; ++t) {
      mbar_init(&bar_ost[t], 4);
      mbar_init(&bar_s[t], 1);
      mbar_init(&bar_p[t], 4);  // one arrival per softmax warp of the tile
      mbar_init(&bar_o[t], 1);
      mbar_init(&bar_rot[t], 1);
      mbar_init(&bar_qready[t], 4);
      mbar_init(&bar_qamax[t], 4);
    }
    fence_mbar_init();
  }
  if constexpr (QROT) {
    if (p.qrot_rotate)
      build_rotation_operand<D, true>(sRot, p.qrot_signs);
    else
      build_rotation_operand<D, false>(sRot, nullptr);
    fence_proxy_async_shared();  // the tensor core reads the operand through the async proxy
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
    // Last warpgroup: MMA issuer, TMA producer, two idle warps. It gives
    // registers back so the softmax warpgroups can take them.
    if constexpr (C::SPLIT_REGS) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::REG_OTHER));
    if (warp == C::TMA_WARP && lane == 0) {
      // ---------------------------------------------------------- producer --
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int pos = 0, iter = 0;
      bool ok = true;
      for (int it = first_item(); it < p.n_items && ok; it = next_item(iter + 1), ++iter) {
      const FwdItem w = item_at(it);
      const int bh = w.bh, q0 = w.q0, kt0 = w.kt0, n_kv = w.n_kv;
      // the previous item's S MMAs read sQ until they complete
      if (iter > 0) ok = mbar_wait(&bar_qfree, (iter - 1) & 1, &abort_flag, st, 11);
      if (!ok) break;
      mbar_arrive_expect_tx(&bar_q, NQ * C::Q_TILE);
      if constexpr (DEC) {
        // rows q0 .. q0+31 into each 32-row quarter of the tile (4 KB apart per chunk)
        for (int w = 0; w < 4; ++w)
          for (int c = 0; c < C::QK_CHUNKS; ++c)
            tma_load_3d(sQ + c * (C::BM * 128) + w * 32 * 128, &tmQ, &bar_q, c * (128 / C::EQK), q0, bh);
      } else {
        for (int t = 0; t < NQ; ++t)
          for (int c = 0; c < C::Q_LOAD_CHUNKS; ++c)
            tma_load_3d(sQ + t * C::Q_TILE + c * (C::BM * 128), &tmQ, &bar_q, c * C::Q_LOAD_ELEMS, q0 + t * C::BM,
                        bh);
      }
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
              tma_load_3d(dst + c * (C::BN * 128), &tmK, &bar_full[slot], c * (128 / C::EQK), (kt0 + j) * C::BN,
                          bh);
          } else {
            mbar_arrive_expect_tx(&bar_full[slot], C::V_TILE);
            for (int c = 0; c < C::V_CHUNKS; ++c)
              tma_load_3d(dst + c * (C::BN * 128), &tmV, &bar_full[slot], c * 64, (kt0 + j) * C::BN, bh);
          }
        }
      }
      }  // items
      // Let every load this thread issued land before the CTA can exit.
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
      uint32_t pc0 = 0, pc1 = 0;  // P-barrier phases waited, per query tile
      bool ok = true;
      for (int it = first_item(); it < p.n_items && ok; it = next_item(iter + 1), ++iter) {
      const FwdItem w = item_at(it);
      const int n_kv = w.n_kv;
      auto n_kv_at = [&](int t) { return t == 0 ? w.n_kv0 : w.n_kv1; };
      ok = mbar_wait(&bar_q, iter & 1, &abort_flag, st, 20);
      if constexpr (QROT) {
        // Each query tile times the rotation operand, into the tile's S
        // columns: the previous item's last P V of the tile, which read P
        // there, was issued before (the tensor core runs them in order).
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < NQ; ++t) {
            issue_rotation<D>(tbase + C::S_COL(t), qaddr + t * C::Q_TILE, smem_u32(sRot));
            mma_commit(&bar_rot[t]);
          }
        }
      }
      // Step j of the item: P V of key tile j - 1 (j > 0), then S of key tile j
      // (j < n_kv), for each query tile. Returns false on an abort.
      auto issue_step = [&](int j) -> bool {
        bool ok = true;
        const int kpos = pos + 2 * j, vpos = pos + 2 * j - 1;
        const int kslot = kpos % C::NSLOT, vslot = (vpos + C::NSLOT) % C::NSLOT;
        if (j < n_kv) ok = mbar_wait(&bar_full[kslot], (kpos / C::NSLOT) & 1, &abort_flag, st, 21);
        if (ok && j > 0) ok = mbar_wait(&bar_full[vslot], (vpos / C::NSLOT) & 1, &abort_flag, st, 22);
        if (!ok) return false;
        tc_fence_after();
        for (int t = 0; t < NQ && ok; ++t) {
          const int n_kv_t = n_kv_at(t);
          if (j > 0 && j - 1 < n_kv_t) {
            // The single issuer polls: its wake-up is on the critical path.
            const uint32_t ph = (t == 0 ? pc0 : pc1) & 1u;
            if (t == 0) ++pc0; else ++pc1;
            // bf16 at d = 128: spin (the wake-up is on the chain; +0.2-2% on
            // B200); e4m3 and d = 64 / 256: the blocking wait (the spin
            // measured 0.5-1% slower or even there)
            ok = (QK_FP8 || D != 128) ? mbar_wait(&bar_p[t], ph, &abort_flag, st, 23, kMmaWaitSleepNs)
                                      : mbar_wait_spin(&bar_p[t], ph, &abort_flag, st, 23);
            if (!ok) break;
            tc_fence_after();
            // O_t += P_t V_{j-1}: A = P_t from TMEM (bf16 pairs), B = V tile (MN-major).
            const uint32_t vaddr = ring + vslot * C::SLOT;
#pragma unroll
            for (int kk = 0; kk < C::BN / 16; ++kk) {
              const uint64_t bdesc = sdesc_sw128(vaddr + kk * 16 * 128, C::BN * 128, 1024);
              mma_bf16_ts(tbase + C::O_COL(t), tbase + C::P_COL(t) + kk * 8, bdesc, idesc_pv,
                          (j > 1 || kk > 0) ? 1u : 0u);
            }
            if (j == n_kv_t) mma_commit(&bar_o[t]);
          }
          if (j < n_kv_t) {
            if constexpr (QROT) {
              if (j == 0) {  // this tile's Q, converted to e4m3 by its warpgroup
                ok = mbar_wait(&bar_qready[t], iter & 1, &abort_flag, st, 24 + t);
                if (!ok) break;
                tc_fence_after();
              }
            }
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
        if (!ok) return false;
        if (j > 0) mma_commit(&bar_empty[vslot]);
        if (j < n_kv) mma_commit(&bar_empty[kslot]);
        return true;
      };
      for (int j = 0; j < n_kv && ok; ++j) ok = issue_step(j);
      // bar_qfree: done when this item's S MMAs (the readers of sQ) are. For a
      // short item it is committed before the last P V products, so that the
      // next item's Q load overlaps them.
      const bool early_q = !CAUSAL && n_kv > 0 && n_kv <= kEarlyQMaxTiles;
      if (ok && early_q) mma_commit(&bar_qfree);
      if (ok) ok = issue_step(n_kv);
      if (!ok) break;
      if (!early_q) mma_commit(&bar_qfree);
      pos += 2 * n_kv;
      }  // items
      // Drain: TMEM is freed below only after every issued MMA has finished.
      mma_commit(&bar_drain);
      mbar_drain(&bar_drain, 0);
    }
  } else {
    // ----------------------------------------------------------- softmax --
    if constexpr (C::SPLIT_REGS) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(C::REG_SOFTMAX));
    if constexpr (DEC) {
      // one item per CTA (the merge buffer is the K/V ring)
      const FwdItem w = item_at(blockIdx.x);
      decode_softmax<D, CAUSAL, QK_FP8, PARTIAL, C>(p, tbase, warp, lane, w.q0, w.bh, w.sp, w.kt0, w.n_kv, sRing,
                                                    bar_s, bar_p, bar_o, &abort_flag, st);
    } else {
    const int t = static_cast<int>(warp >> 2);
    uint32_t sc = 0, oc = 0;  // phases of bar_s[t] and bar_o[t] waited
    bool ok = true;
    for (int round = 0, it = first_item(); it < p.n_items && ok; it = next_item(++round)) {
    const FwdItem w = item_at(it);
    const int bh = w.bh, q0 = w.q0, kt0 = w.kt0, sp = w.sp;
    const uint32_t lane_base = (warp & 3u) * 32u;
    const int r = static_cast<int>(lane_base + lane);  // row within the tile = TMEM lane
    const int qrow = q0 + t * C::BM + r;
    const uint32_t row_addr = tbase + (lane_base << 16);
    const uint32_t tS = row_addr + C::S_COL(t);
    const uint32_t tP = row_addr + C::P_COL(t);
    const uint32_t tO = row_addr + C::O_COL(t);
    // exp2 scale: scale * log2(e), times the descales of the query tile and (per
    // key tile, when scales are per block) of the key tile
    float s_q = p.scale_log2;
    const float* dkb = nullptr;
    if constexpr (QROT) {
      // this warpgroup's Q tile: the rotated rows from tensor memory, to e4m3
      // codes in place of the bf16 tile (which the product has finished reading)
      const bool got = __all_sync(0xffffffffu, mbar_wait(&bar_rot[t], round & 1, &abort_flag, st, 35));
      float m = 0.f;
      if (got) {
        tc_fence_after();
        m = p.qrot_rotate ? row_absmax<D, true>(tS) : row_absmax<D, false>(tS);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      // The tile's amax from the four warps' maxima. An mbarrier, not a named
      // barrier: a warp that has left after an abort leaves the others a
      // bounded wait, not a hang.
      if (lane == 0) {
        qrot_red[t][warp & 3u] = m;
        mbar_arrive(&bar_qamax[t]);  // release: the maximum is visible to the waiters
      }
      ok = got && __all_sync(0xffffffffu, mbar_wait(&bar_qamax[t], round & 1, &abort_flag, st, 36));
      if (!ok) break;
      float amax = fmaxf(fmaxf(qrot_red[t][0], qrot_red[t][1]), fmaxf(qrot_red[t][2], qrot_red[t][3]));
      if (p.qrot_rotate) amax *= HadCfg<D>::INV_SQRT_D;  // fp32 rounding is monotonic: max fl(|v| c) = fl(c max |v|)
      const float qsc = amax > 0.f ? 448.0f / amax : 1.0f;
      const float dq = amax > 0.f ? amax / 448.0f : 1.0f;
      // Rows past the end of the sequence hold zeros (TMA fill): they do not
      // change the amax, and their codes are never used.
      uint8_t* qrow_codes = sQ + t * C::Q_TILE + r * 128;
      auto put = [&](int j, const uint4& v) {  // 16 codes, at their swizzled place
        *reinterpret_cast<uint4*>(qrow_codes + ((j ^ (r & 7)) << 4)) = v;
      };
      if (p.qrot_rotate)
        row_codes<D, true>(tS, qsc, put);
      else
        row_codes<D, false>(tS, qsc, put);
      // the tensor core reads the codes through the async proxy, and the S
      // product overwrites the columns just read
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_qready[t]);
      // qrot_red[t] is written again only after the next item's bar_rot wait,
      // which follows this item's S products, which follow every warp's
      // bar_qready arrival, which follows its reads of qrot_red[t]
      if (p.dq_out != nullptr && r == 0 && q0 + t * C::BM < p.Nq)
        p.dq_out[static_cast<size_t>(bh) * p.nbq + (q0 + t * C::BM) / C::BM] = dq;
      s_q *= dq;
      dkb = p.dk_block + static_cast<size_t>(bh) * p.nbk + kt0;
    } else if constexpr (QK_FP8) {
      if (p.dq_block != nullptr) {
        if (q0 + t * C::BM < p.Nq) s_q *= __ldg(p.dq_block + static_cast<size_t>(bh) * p.nbq + (q0 + t * C::BM) / C::BM);
        dkb = p.dk_block + static_cast<size_t>(bh) * p.nbk + kt0;
      } else {
        s_q *= __ldg(p.descale_qk) * __ldg(p.descale_qk + 1);
      }
    }
    // Last visible key of this row, counted from the split's first key (so the
    // loop below works in split-relative key indices).
    const int kmax = (CAUSAL ? min(qrow + p.causal_off, p.Nk - 1) : p.Nk - 1) - kt0 * C::BN;
    float m_ref = -INFINITY;  // reference max, scaled log2 units
    float l_exact = 0.f;      // sum of the fp32 weights: gives the LSE
    float l_round = 0.f;      // sum of the bf16-rounded weights P uses: normalises O
    const int n_kv_t = t == 0 ? w.n_kv0 : w.n_kv1;
    float dk_next = (QK_FP8 && dkb != nullptr && n_kv_t > 0) ? __ldg(dkb) : 1.0f;
    for (int j = 0; j < n_kv_t; ++j) {
      const float s_log2 = s_q * dk_next;
      if (QK_FP8 && dkb != nullptr && j + 1 < n_kv_t) dk_next = __ldg(dkb + j + 1);  // in flight during this step
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[t], sc & 1u, &abort_flag, st, 30 + t));
      ++sc;
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      const int kbase = j * C::BN;  // split-relative
      // Some key of this tile is not visible to some row of this warp. Warp-uniform:
      // it selects code paths that issue tcgen05.ld, which all 32 lanes must
      // execute together (a lane-divergent .sync.aligned instruction deadlocks).
      const bool masked = __any_sync(0xffffffffu, kbase + C::BN - 1 > kmax);
      float sum_e, sum_r, alpha = 1.0f;
      if (j == 0) {
        // A row that sees no key of this split (partial mode only) has max -inf;
        // it takes reference 0, so its weights are exp2(-inf) = 0 throughout and
        // it is recognised at the end by its zero sum.
        m_ref = row_max_tmem(tS, s, kbase, kmax, masked) * s_log2;
        if (PARTIAL && m_ref == -INFINITY) m_ref = 0.f;
        softmax_row_dispatch(tS, s, s_log2, m_ref, kbase, kmax, masked, sum_e, sum_r);
      } else {
        // Exponentials against the current reference. A row whose max grew by more
        // than 8 (log2 units) has a weight above 2^8, so its tile sum exceeds 2^8:
        // only then (rare after the first tiles) is its exact max taken, and the
        // tile redone, against the new reference if the max did grow that much.
        // S is still intact: P is written only below.
        softmax_row_dispatch(tS, s, s_log2, m_ref, kbase, kmax, masked, sum_e, sum_r);
        if (__any_sync(0xffffffffu, sum_e > 256.0f)) {
          const float mx_s = row_max_tmem(tS, s, kbase, kmax, masked) * s_log2;
          const bool grow = mx_s > m_ref + 8.0f;
          const float m_new = grow ? mx_s : m_ref;
          alpha = ex2_approx(m_ref - m_new);  // 1 for rows that did not grow
          m_ref = m_new;
          softmax_row_dispatch(tS, s, s_log2, m_ref, kbase, kmax, masked, sum_e, sum_r);
          // Rescale this warp's O rows in TMEM. The PV product of tile j-1 has
          // completed (the commit that signalled S_t for tile j also covers it),
          // and PV of tile j is issued only after this warpgroup arrives below.
          if (__any_sync(0xffffffffu, grow)) {
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
      tmem_st32(tP + 0, &s[0]);
      tmem_st32(tP + 32, &s[32]);
      l_exact = l_exact * alpha + sum_e;
      l_round = l_round * alpha + sum_r;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
#ifdef FA_TEST_HOOKS
      const bool withhold = lane == 0 && warp == 0 && blockIdx.x == 0 && round == 0 && j == 1 &&
                            atomicExch(&g_fa_test_withhold_p, 0) != 0;
      if (lane == 0 && !withhold) mbar_arrive(&bar_p[t]);
#else
      if (lane == 0) mbar_arrive(&bar_p[t]);  // one arrival per warp
#endif
    }
    if (ok && n_kv_t > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar_o[t], oc & 1u, &abort_flag, st, 40 + t));
    if (n_kv_t > 0) ++oc;
    const bool in_range = qrow < p.Nq;
    if constexpr (PARTIAL) {
      if (ok) {
        // O of this split's keys in fp32 (normalised by its own weights) and its
        // LSE; a row with no key of the split gets 0 and -inf.
        const bool empty = l_exact == 0.f;
        const size_t prow = (static_cast<size_t>(sp) * p.BH + bh) * p.Nq + (in_range ? qrow : 0);
        float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D);
        if (n_kv_t > 0) tc_fence_after();
        const float inv_l = empty ? 0.f : 1.0f / l_round;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          if (n_kv_t > 0) {
            tmem_ld32(tO + c0, ov);
            tmem_wait_ld_dep32(ov);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0u;
          }
          if (in_range) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[c0 / 4 + i] = make_float4(
                  __uint_as_float(ov[4 * i]) * inv_l, __uint_as_float(ov[4 * i + 1]) * inv_l,
                  __uint_as_float(ov[4 * i + 2]) * inv_l, __uint_as_float(ov[4 * i + 3]) * inv_l);
          }
        }
        if (in_range)
          p.lse_part[prow] = empty ? -INFINITY : (m_ref + __log2f(l_exact)) * 0.69314718055994530942f;
      }
    } else if (TAIL && w.tail >= 0) {
      if (ok && n_kv_t > 0) {
        tc_fence_after();
        tail_piece_epilogue<D, NQ>(p, w, t, warp & 3u, lane, tO, r, qrow, m_ref, l_exact, l_round, st);
      }
    } else if (OSTAGE) {
      ok = staged_o_epilogue<D, NQ, C>(&tmO, sOst, bar_ost, &bar_ofree, &abort_flag, st, p.lse, p.Nq, tO, r, lane,
                                        warp, t, round, n_kv_t > 0, ok, l_round, l_exact, m_ref, q0, bh, qrow);
    } else if (ok && n_kv_t > 0) {
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
    }  // items
    // the O stores this thread issued complete before the CTA exits
    if constexpr (OSTAGE) {
      if ((warp & 3u) == 0 && lane == 0) bulk_wait_all();
    }
    }  // not DEC
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace fa

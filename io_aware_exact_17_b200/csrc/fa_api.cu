// fa_api.cu — the C ABI declared in include/fa.h: argument checks, TMA tensor
// maps, and the launches of the attention and quantisation kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <random>

#include "../../include/fa.h"
#include "attn_bwd.cuh"
#include "quant_t.cuh"
#include "attn_fwd.cuh"
#include "merge.cuh"
#include "quant.cuh"
#include "tmap.h"

namespace {

using fa::FwdCfg;
using fa::FwdParams;

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename K>
bool set_smem_once(K kernel, int bytes, unsigned long long* done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const unsigned long long bit = 1ull << (dev & 63);
  if (*done_mask & bit) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  *done_mask |= bit;
  return true;
}

// Everything one attention launch needs (argument checks are done by the caller).
struct FwdArgs {
  const void *q, *k, *v;
  void* o;              // bf16 output (direct mode)
  float* lse;           // may be null (direct mode)
  float* o_part;        // partial mode (n_split >= 1 blocks of keys, fp32); null = direct mode
  float* lse_part;
  int B, H, Nq, Nk, d;
  bool causal;
  float scale;
  fa_dtype qk_dtype;
  const float* descale_qk;
  int n_split;
  // in-kernel rotate-and-quantise of bf16 Q (fa_fwd_fp8_qrot): descale_qk then
  // holds the key-block descales only
  bool qrot = false;
  int qrot_rotate = 0;
  const float* qrot_signs = nullptr;
  float* dq_out = nullptr;
  // tail split of a direct, non-causal persistent launch (FwdParams): 0 = none
  int tail_split = 0;
  int tail_tiles = 0;
  long long n_full = 0;
  float* tail_o = nullptr;
  float* tail_lse = nullptr;
  unsigned long long* tail_cnt = nullptr;
};

constexpr int kKeyTile = 128;  // keys per K/V tile (FwdCfg::BN)

inline int key_tiles(int Nk) { return (Nk + kKeyTile - 1) / kKeyTile; }

// Query tiles per CTA: two (ping-pong) when d <= 128 and a head has more than
// one tile of queries; one for d = 256 (TMEM) and for short query blocks.
inline int nq_for(int d, int Nq) { return (d <= 128 && Nq > 128) ? 2 : 1; }

// Queries per head up to which the decode layout (four key quarters per tile) runs.
constexpr int kDecodeMaxQ = 32;

int device_sms();  // SM count of the current device (cached)

#ifndef FA_PERSISTENT
#define FA_PERSISTENT 1
#endif
constexpr bool kPersistent = FA_PERSISTENT != 0;
#ifndef FA_PERSIST_CAUSAL
#define FA_PERSIST_CAUSAL 1
#endif
constexpr bool kPersistCausal = FA_PERSIST_CAUSAL != 0;
#ifndef FA_TAIL_SPLIT
#define FA_TAIL_SPLIT 1
#endif
constexpr bool kTailSplit = FA_TAIL_SPLIT != 0;

// A new 56-bit tail-split tag for every launch that takes one: a per-process
// random start plus a launch count, never 0 (the tag of a zeroed word), so that a
// ticket word left by another launch, or never written, matches it only by a
// 2^-56 chance.
unsigned long long next_tail_tag() {
  static std::atomic<unsigned long long> count{0};
  static const unsigned long long start = [] {
    std::random_device rd;
    return (static_cast<unsigned long long>(rd()) << 32) ^ rd() ^
           static_cast<unsigned long long>(std::chrono::steady_clock::now().time_since_epoch().count());
  }();
  for (;;) {
    const unsigned long long t = (start + count.fetch_add(1ull)) & ((1ull << 56) - 1ull);
    if (t != 0ull) return t;
  }
}

template <int D, int NQ, bool CAUSAL, bool QK_FP8, bool PARTIAL, bool DEC, bool QROT = false>
fa_status launch_fwd(const FwdArgs& a, cudaStream_t stream) {
  using C = FwdCfg<D, NQ, QK_FP8, QROT>;
  const int BH = a.B * a.H;
  CUtensorMap tmQ, tmK, tmV;
  const CUtensorMapDataType qk_type = QK_FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool q_ok = QROT ? fa::make_tmap_3d(&tmQ, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.Nq, BH, 64, C::BM)
                         : fa::make_tmap_3d(&tmQ, a.q, qk_type, C::EQK, D, a.Nq, BH, 128 / C::EQK,
                                            DEC ? kDecodeMaxQ : C::BM);
  if (!q_ok || !fa::make_tmap_3d(&tmK, a.k, qk_type, C::EQK, D, a.Nk, BH, 128 / C::EQK, C::BN) ||
      !fa::make_tmap_3d(&tmV, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.Nk, BH, 64, C::BN))
    return FA_ERR_CUDA;
  // direct-mode O goes through shared memory and TMA stores where the staging
  // buffer fits (FwdCfg::OST_*); the map is unused otherwise
  constexpr bool kOStage = fa::fwd_ostage<C, CAUSAL, PARTIAL, DEC>();
  CUtensorMap tmO = tmV;
  if constexpr (kOStage) {
    if (!fa::make_tmap_3d(&tmO, a.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.Nq, BH, 64, C::BM))
      return FA_ERR_CUDA;
  }
  constexpr int kSmem = C::smem_bytes(kOStage);
  auto kernel = fa::attn_fwd_kernel<D, NQ, CAUSAL, QK_FP8, PARTIAL, DEC, QROT>;
  static unsigned long long smem_done = 0;
  if (!set_smem_once(kernel, kSmem, &smem_done)) return FA_ERR_CUDA;
  if constexpr (C::SPLIT_REGS) {
    // The kernel moves registers between warpgroups with setmaxnreg; that only
    // completes if the block was launched with the register count the split was
    // sized for. Refuse to launch otherwise (an .inc that can never be satisfied
    // would wait forever).
    static int checked = 0;  // 0 = not yet, 1 = ok, 2 = bad
    if (checked == 0) {
      cudaFuncAttributes fa_attr;
      if (cudaFuncGetAttributes(&fa_attr, kernel) != cudaSuccess) return FA_ERR_CUDA;
      checked = fa_attr.numRegs >= C::REG_LAUNCH ? 1 : 2;
    }
    if (checked != 1) return FA_ERR_UNSUPPORTED;
  }
  static_assert(C::BN == kKeyTile, "key tile");
  FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.o_part = a.o_part;
  p.lse_part = a.lse_part;
  p.descale_qk = a.descale_qk;
  p.dq_block = nullptr;
  p.dk_block = nullptr;
  p.nbq = (a.Nq + 127) / 128;
  p.nbk = (a.Nk + 127) / 128;
  p.qrot_signs = a.qrot_signs;
  p.qrot_rotate = a.qrot_rotate;
  p.dq_out = a.dq_out;
  if (QROT) {
    p.dk_block = a.descale_qk;  // key blocks only: the query blocks' are computed in the kernel
  } else if (a.qk_dtype == FA_E4M3_BLOCK) {
    // one descale per 128-row block: the query blocks of every head, then the key blocks
    p.dq_block = a.descale_qk;
    p.dk_block = a.descale_qk + static_cast<size_t>(BH) * p.nbq;
  }
  p.BH = BH;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.causal_off = a.Nk - a.Nq;
  p.n_qb = (a.Nq + NQ * C::BM - 1) / (NQ * C::BM);
  p.n_split = a.n_split;
  p.split_tiles = (key_tiles(a.Nk) + a.n_split - 1) / a.n_split;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const long long units = static_cast<long long>(p.n_qb) * BH;
  long long items = units * (PARTIAL ? a.n_split : 1);
  if (items < 1) return FA_OK;
  p.n_full = static_cast<int>(units);
  p.tail_split = 0;
  p.tail_tiles = 0;
  p.tail_tag = 0;
  p.tail_o = nullptr;
  p.tail_lse = nullptr;
  p.tail_cnt = nullptr;
  constexpr bool kTailKernel = !PARTIAL && !DEC && !CAUSAL && !QROT;
  if (kTailKernel && a.tail_split >= 2) {
    if (a.tail_split > fa::kTailMaxSplit || a.n_full < 0 || a.n_full >= units || a.tail_o == nullptr ||
        a.tail_lse == nullptr || a.tail_cnt == nullptr)
      return FA_ERR_INVALID_ARG;
    p.n_full = static_cast<int>(a.n_full);
    p.tail_split = a.tail_split;
    p.tail_tiles = a.tail_tiles;
    p.tail_tag = next_tail_tag();
    p.tail_o = a.tail_o;
    p.tail_lse = a.tail_lse;
    p.tail_cnt = a.tail_cnt;
    items = a.n_full + (units - a.n_full) * a.tail_split;
    if (items > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  }
  p.n_items = static_cast<int>(items);
  // Persistent: at most one CTA per SM, each looping over work items, so the
  // next item's Q load and first S MMA overlap the current item's last steps and
  // epilogue (non-causal: +1-6% on B200). Causal items differ in length: a plain
  // round-robin over them balanced worse than the hardware's dispatch of one CTA
  // per item (-5-11%), but ranking the query blocks heaviest first across all
  // heads and dealing them in snake order (p.snake) beats it (+11-22%). Split-key
  // causal launches and the decode layout (whose epilogue uses the K/V ring) run
  // one item per CTA.
  long long grid = items;
  const bool persist = kPersistent && !DEC && (!CAUSAL || (kPersistCausal && !PARTIAL));
  p.snake = (persist && CAUSAL) ? 1 : 0;
  if (persist) {
    const long long sms = device_sms();
    if (grid > sms) grid = sms;
  }
  kernel<<<static_cast<unsigned>(grid), C::THREADS, kSmem, stream>>>(tmQ, tmK, tmV, tmO, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, int NQ, bool QK_FP8, bool DEC>
fa_status launch_fwd_cd(const FwdArgs& a, cudaStream_t s) {
  if (a.o_part != nullptr)
    return a.causal ? launch_fwd<D, NQ, true, QK_FP8, true, DEC>(a, s)
                    : launch_fwd<D, NQ, false, QK_FP8, true, DEC>(a, s);
  return a.causal ? launch_fwd<D, NQ, true, QK_FP8, false, DEC>(a, s) : launch_fwd<D, NQ, false, QK_FP8, false, DEC>(a, s);
}

template <int D, int NQ, bool QK_FP8>
fa_status launch_fwd_c(const FwdArgs& a, cudaStream_t s) {
  if constexpr (NQ == 1) {
    if (a.Nq <= kDecodeMaxQ) return launch_fwd_cd<D, NQ, QK_FP8, true>(a, s);
  }
  return launch_fwd_cd<D, NQ, QK_FP8, false>(a, s);
}

// Kernel choice by head dimension, dtype and query length.
fa_status dispatch_fwd(const FwdArgs& a, cudaStream_t s) {
  const bool two = nq_for(a.d, a.Nq) == 2;
  if (a.qk_dtype == FA_BF16) {
    switch (a.d) {
      case 64: return two ? launch_fwd_c<64, 2, false>(a, s) : launch_fwd_c<64, 1, false>(a, s);
      case 128: return two ? launch_fwd_c<128, 2, false>(a, s) : launch_fwd_c<128, 1, false>(a, s);
      default: return launch_fwd_c<256, 1, false>(a, s);
    }
  }
  switch (a.d) {
    case 128: return two ? launch_fwd_c<128, 2, true>(a, s) : launch_fwd_c<128, 1, true>(a, s);
    default: return launch_fwd_c<256, 1, true>(a, s);
  }
}

// Checks shared by every attention entry point.
fa_status check_fwd_args(const void* q, const void* k, const void* v, int B, int H, int Nq, int Nk, int d,
                         int causal, float scale, fa_dtype qk_dtype, const float* descale_qk, int n_split) {
  if (q == nullptr || k == nullptr || v == nullptr) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || n_split < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && Nq > Nk) return FA_ERR_INVALID_ARG;  // some query would see no key
  if (!(scale > 0.0f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (qk_dtype != FA_BF16 && qk_dtype != FA_E4M3 && qk_dtype != FA_E4M3_BLOCK) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (qk_dtype != FA_BF16 && d == 64) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return FA_ERR_ALIGNMENT;
  if (qk_dtype != FA_BF16) {
    if (descale_qk == nullptr) return FA_ERR_INVALID_ARG;
    if (!aligned(descale_qk, 4)) return FA_ERR_ALIGNMENT;
  }
  const long long rows_per_cta = 128;  // the smallest query block of any kernel
  const long long n_qb = (static_cast<long long>(Nq) + rows_per_cta - 1) / rows_per_cta;
  if (n_qb * n_split * B * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * Nk > (1LL << 40)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// Bytes of the split-key workspace: the fp32 partial outputs, then (256-byte
// aligned) the partial LSEs.
size_t part_o_bytes(int B, int H, int Nq, int d, int n_split) {
  return static_cast<size_t>(n_split) * B * H * Nq * d * sizeof(float);
}
size_t part_bytes(int B, int H, int Nq, int d, int n_split) {
  const size_t o = (part_o_bytes(B, H, Nq, d, n_split) + 255) & ~static_cast<size_t>(255);
  return o + static_cast<size_t>(n_split) * B * H * Nq * sizeof(float);
}

// L2 cache bytes of the current device (looked up once per device).
double device_l2_bytes() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 126.0 * (1 << 20);
  if (cached[dev] == 0) {
    int l2 = 0;
    if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 < 1) return 126.0 * (1 << 20);
    cached[dev] = l2;
  }
  return static_cast<double>(cached[dev]);
}

int device_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) return 148;
    cached[dev] = sms;
  }
  return cached[dev];
}

// Split count for a launch of `units` CTAs per split over `tiles` key tiles,
// one CTA per SM: the count with the fewest key-tile steps on the busiest SM,
// counting four steps of fixed cost per CTA (prologue, pipeline fill, epilogue
// with the partial output) and half a step per block for the merge; ties go to
// fewer splits. (Measured on B200 for one query over 16k-128k keys: the counts
// this picks are within 2% of the best of 1, 2, 4, 8, 16.)
int pick_splits(long long units, int tiles, int sms) {
  if (units >= sms || tiles <= 2) return 1;
  double best_cost = -1.0;
  int best = 1;
  const int max_split = tiles < 128 ? tiles : 128;
  for (int ns = 1; ns <= max_split; ++ns) {
    const long long waves = (units * ns + sms - 1) / sms;
    const long long per_cta = (tiles + ns - 1) / ns + 4;
    const double cost = static_cast<double>(waves * per_cta) + (ns > 1 ? 0.5 * ns : 0.0);
    if (best_cost < 0.0 || cost < best_cost) {
      best_cost = cost;
      best = ns;
    }
  }
  return best;
}

int auto_splits(int B, int H, int Nq, int Nk, int d) {
  const int nq = nq_for(d, Nq);
  const long long units = static_cast<long long>(B) * H * ((Nq + nq * 128 - 1) / (nq * 128));
  return pick_splits(units, key_tiles(Nk), device_sms());
}

// The automatic schedule of fa_fwd_splitkv (n_split = 0): with fewer query
// blocks than SMs, every block's keys are split (auto_splits) and merged by a
// second launch; else one persistent CTA per SM over the query blocks, with a
// tail split: without causal masking, when the launch's last round is at most
// half full, the keys of that round's query blocks are split into tail_split
// pieces (as many as the round's idle CTAs allow, at most four), merged by the
// kernel itself (FwdParams). Measured on B200 at B=4, H=16, N=2048, d=128
// (68 of 512 blocks in the last round, two pieces each): +3-6%. (An earlier
// form, with one row per thread in the pieces' fp32 stores and one CTA per
// work item, was slower than no split.)
struct Plan {
  int n_split = 1;
  int nq = 1;
  long long units = 0;
  int tail_split = 0;
  int tail_tiles = 0;
  long long n_full = 0;
};

// Fewest key tiles per query block for a tail split to pay for its merge.
constexpr int kTailMinTiles = 4;

Plan plan_fwd(int B, int H, int Nq, int Nk, int d, bool causal) {
  Plan pl;
  pl.nq = nq_for(d, Nq);
  pl.units = static_cast<long long>(B) * H * ((Nq + pl.nq * 128 - 1) / (pl.nq * 128));
  const int sms = device_sms();
  if (pl.units < sms) {
    pl.n_split = pick_splits(pl.units, key_tiles(Nk), sms);
  } else if (kTailSplit && kPersistent && !causal && !(pl.nq == 1 && Nq <= kDecodeMaxQ)) {
    const long long full = pl.units / sms * sms, tail = pl.units - full;
    const int kt = key_tiles(Nk);
    if (tail > 0 && 2 * tail <= sms && kt >= kTailMinTiles) {
      long long ns = sms / tail;
      if (ns > fa::kTailMaxSplit) ns = fa::kTailMaxSplit;
      if (ns > kt) ns = kt;
      const int span = static_cast<int>((kt + ns - 1) / ns);
      ns = (kt + span - 1) / span;  // no empty piece
      if (ns >= 2) {
        pl.tail_split = static_cast<int>(ns);
        pl.tail_tiles = span;
        pl.n_full = full;
      }
    }
  }
  return pl;
}

// Tail-split workspace: the pieces' O, their LSEs, the ticket words; each part
// 256-byte aligned.
struct TailLayout {
  size_t o = 0, lse = 0, cnt = 0, bytes = 0;
};
TailLayout tail_layout(const Plan& pl, int d) {
  TailLayout t;
  if (pl.tail_split < 2) return t;
  const size_t groups = static_cast<size_t>(pl.units - pl.n_full) * pl.nq;  // (tail block, query tile)
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  t.o = 0;
  t.lse = up(groups * pl.tail_split * 128 * d * sizeof(float));
  t.cnt = t.lse + up(groups * pl.tail_split * 128 * sizeof(float));
  t.bytes = t.cnt + up(groups * 4 * sizeof(unsigned long long));
  return t;
}

size_t plan_bytes(const Plan& pl, int B, int H, int Nq, int d) {
  if (pl.tail_split >= 2) return tail_layout(pl, d).bytes;
  return pl.n_split <= 1 ? 0 : part_bytes(B, H, Nq, d, pl.n_split);
}

// Largest row count of the quantisers: TMA tile coordinates are 32-bit (such a
// tensor of bf16 rows would not fit in a GPU's memory anyway).
constexpr int64_t kQuantMaxRows = (static_cast<int64_t>(1) << 31) - 4096;

// Both quantisation passes in one cooperative launch (quant_tensor_kernel) for
// the tensors of `b`: amax_words[0 .. n-1] and counters[0 .. n-1] (the grid
// barriers' arrivals) are zeroed here. One CTA per SM (up to one per 128-row
// tile), all co-resident.
template <int D>
fa_status launch_quant_fused(const fa::QuantBatch& b, float* descale_out, int64_t rows, int rotate,
                             const float* signs, unsigned int* amax_words, unsigned int* counters,
                             cudaStream_t stream) {
  using RC = fa::RotQuantCfg<D>;
  if (counters == amax_words + b.n) {  // one contiguous scratch (the workspace entry points)
    if (cudaMemsetAsync(amax_words, 0, 2 * b.n * sizeof(unsigned int), stream) != cudaSuccess) return FA_ERR_CUDA;
  } else {
    if (cudaMemsetAsync(amax_words, 0, b.n * sizeof(unsigned int), stream) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemsetAsync(counters, 0, b.n * sizeof(unsigned int), stream) != cudaSuccess) return FA_ERR_CUDA;
  }
  if (rows == 0) {  // nothing to read: every descale is 1
    fa::fill_f32_kernel<<<1, 32, 0, stream>>>(descale_out, b.n, 1.0f);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  }
  auto kernel = rotate ? fa::quant_tensor_kernel<D, true> : fa::quant_tensor_kernel<D, false>;
  static unsigned long long smem_set[2] = {0, 0};
  if (!set_smem_once(kernel, RC::SMEM, &smem_set[rotate ? 1 : 0])) return FA_ERR_CUDA;
  const int64_t ntile = (rows + RC::BM - 1) / RC::BM;
  int64_t blocks = device_sms();  // one CTA per SM: the kernel holds all of an SM's tensor memory
  if (blocks > ntile) blocks = ntile;
  fa::QuantMaps qm;
  std::memset(&qm, 0, sizeof(qm));
  for (int t = 0; t < b.n; ++t) {
    if (!fa::make_tmap_2d(&qm.x[t], b.x[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, static_cast<uint64_t>(rows), 64,
                          RC::BM))
      return FA_ERR_CUDA;
    if (!fa::make_tmap_2d(&qm.y[t], b.out[t], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, static_cast<uint64_t>(rows),
                          RC::CROW, 32, fa::codes_swizzle<D>()))
      return FA_ERR_CUDA;
  }
  qm.n = b.n;
  int rows_i = static_cast<int>(rows);
  // The next tensor's pass 1 runs ahead of this tensor's pass 2: all of it
  // when two tensors fit in two thirds of L2 (pass 2 still finds its tensor
  // there), else the first few tiles of each CTA, to cover the grid barrier.
  const double two_tensors = 2.0 * static_cast<double>(rows) * D * 2;
  int lead = two_tensors <= device_l2_bytes() * 2.0 / 3.0 ? 0x7fffffff : 4;
  void* args[] = {&qm, &rows_i, &lead, &signs, &amax_words, &counters, &descale_out};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3(static_cast<unsigned>(blocks)),
                                  dim3(RC::THREADS + 32), args, RC::SMEM, stream) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

// One scale per 128-row block of a head (quant_block_kernel): one pass,
// persistent CTAs (one per SM) over the tiles of each head.
template <int D>
fa_status launch_quant_blocks(const void* x, void* out, float* descales, int BH, int N, int rotate,
                              const float* signs, cudaStream_t stream) {
  using RC = fa::RotQuantCfg<D>;
  auto kernel = rotate ? fa::quant_block_kernel<D, true> : fa::quant_block_kernel<D, false>;
  static unsigned long long smem_set[2] = {0, 0};
  if (!set_smem_once(kernel, RC::SMEM, &smem_set[rotate ? 1 : 0])) return FA_ERR_CUDA;
  CUtensorMap tm, tmy;
  if (!fa::make_tmap_3d(&tm, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, static_cast<uint64_t>(N),
                        static_cast<uint64_t>(BH), 64, RC::BM))
    return FA_ERR_CUDA;
  if (!fa::make_tmap_3d(&tmy, out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, static_cast<uint64_t>(N),
                        static_cast<uint64_t>(BH), RC::CROW, 32, fa::codes_swizzle<D>()))
    return FA_ERR_CUDA;
  const long long units = static_cast<long long>(BH) * ((N + RC::BM - 1) / RC::BM);
  long long grid = device_sms();
  if (grid > units) grid = units;
  kernel<<<static_cast<unsigned>(grid), RC::THREADS, RC::SMEM, stream>>>(tm, tmy, BH, N, signs, descales);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status dispatch_quant_fused(const fa::QuantBatch& b, float* descale_out, int64_t rows, int d, int rotate,
                               const float* signs, unsigned int* amax_words, unsigned int* counters,
                               cudaStream_t s) {
  switch (d) {
    case 64: return launch_quant_fused<64>(b, descale_out, rows, rotate, signs, amax_words, counters, s);
    case 128: return launch_quant_fused<128>(b, descale_out, rows, rotate, signs, amax_words, counters, s);
    default: return launch_quant_fused<256>(b, descale_out, rows, rotate, signs, amax_words, counters, s);
  }
}

template <int D>
fa_status launch_merge(const float* o_part, const float* lse_part, int n_part, int64_t rows, void* o, float* lse,
                       cudaStream_t stream) {
  const int64_t warps_per_block = fa::kMergeThreads / 32;
  int64_t blocks = (rows + warps_per_block - 1) / warps_per_block;
  const int64_t cap = static_cast<int64_t>(device_sms()) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  fa::lse_merge_kernel<D><<<static_cast<unsigned>(blocks), fa::kMergeThreads, 0, stream>>>(
      o_part, lse_part, n_part, rows, static_cast<__nv_bfloat16*>(o), lse);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status dispatch_merge(const float* o_part, const float* lse_part, int n_part, int64_t rows, int d, void* o,
                         float* lse, cudaStream_t s) {
  switch (d) {
    case 64: return launch_merge<64>(o_part, lse_part, n_part, rows, o, lse, s);
    case 128: return launch_merge<128>(o_part, lse_part, n_part, rows, o, lse, s);
    default: return launch_merge<256>(o_part, lse_part, n_part, rows, o, lse, s);
  }
}


}  // namespace

// ------------------------------------------------------------- backward --
inline size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline int bwd_npad(int N) { return (N + 127) / 128 * 128; }

size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  const size_t BH = static_cast<size_t>(B) * H;
  return round256(BH * N * d * sizeof(float)) + 2 * round256(BH * bwd_npad(N) * sizeof(float));
}

template <int D, bool CAUSAL>
fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                     void* dq, void* dk, void* dv, int B, int H, int N, float scale, void* workspace,
                     cudaStream_t stream) {
  using C = fa::BwdCfg<D>;
  const int BH = B * H;
  const int Npad = bwd_npad(N);
  float* dq_acc = static_cast<float*>(workspace);
  float* nlse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                         round256(static_cast<size_t>(BH) * N * D * sizeof(float)));
  float* dvec = nlse2 + round256(static_cast<size_t>(BH) * Npad * sizeof(float)) / sizeof(float);
  CUtensorMap tmQ, tmK, tmV, tmdO, tmdQ;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!fa::make_tmap_3d(&tmQ, q, bf, 2, D, N, BH, 64, 128) || !fa::make_tmap_3d(&tmK, k, bf, 2, D, N, BH, 64, 128) ||
      !fa::make_tmap_3d(&tmV, v, bf, 2, D, N, BH, 64, 128) || !fa::make_tmap_3d(&tmdO, dout, bf, 2, D, N, BH, 64, 128))
    return FA_ERR_CUDA;
  // the fp32 dQ accumulator, reduced into in tiles of 32 rows x 32 columns
  if (!fa::make_tmap_3d(&tmdQ, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, N, BH, 32, 32)) return FA_ERR_CUDA;
  // dK and dV, stored in 64-column boxes of 128 key rows (d = 128 kernel)
  CUtensorMap tmdK, tmdV;
  if (!fa::make_tmap_3d(&tmdK, dk, bf, 2, D, N, BH, 64, 128) || !fa::make_tmap_3d(&tmdV, dv, bf, 2, D, N, BH, 64, 128))
    return FA_ERR_CUDA;
  const long long rows = static_cast<long long>(BH) * Npad;
  {
    const long long per_block = 8LL * (32 / (D / 8));  // rows one pass of a block covers
    long long blocks = (rows + per_block - 1) / per_block;
    const long long cap = static_cast<long long>(device_sms()) * 16;
    if (blocks > cap) blocks = cap;
    fa::attn_bwd_prep_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, nlse2, dvec, dq_acc, BH,
        N, Npad);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  // The main kernel and the dQ conversion are launched with programmatic
  // stream serialisation: each may start (set up, load K and V) while the
  // kernel before it finishes, and waits for it (griddepcontrol.wait) before
  // reading what it wrote.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  // d = 128: the two softmax warpgroups ping-pong over half steps of 64 queries
  auto kernel = D == 128 ? fa::attn_bwd_pp_kernel<CAUSAL> : fa::attn_bwd_kernel<D, CAUSAL>;
  const int smem_bytes = D == 128 ? fa::BwdPpCfg::SMEM_BYTES : C::SMEM_BYTES;
  static unsigned long long smem_done = 0;
  if (!set_smem_once(kernel, smem_bytes, &smem_done)) return FA_ERR_CUDA;
  fa::BwdParams p;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.nlse2 = nlse2;
  p.dvec = dvec;
  p.BH = BH;
  p.N = N;
  p.Npad = Npad;
  p.n_t = Npad / 128;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(static_cast<long long>(BH) * p.n_t));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, tmQ, tmK, tmV, tmdO, tmdQ, tmdK, tmdV, p) != cudaSuccess) return FA_ERR_CUDA;
  }
  const long long n4 = static_cast<long long>(BH) * N * D / 4;
  const long long cap = static_cast<long long>(device_sms()) * 8;
  const long long blocks = (n4 + 255) / 256 < cap ? (n4 + 255) / 256 : cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa::attn_bwd_dq_kernel, reinterpret_cast<const float4*>(dq_acc), static_cast<uint2*>(dq),
                         n4, scale) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 int causal, float scale, fa_dtype qk_dtype, const float* descale_qk, void* stream) {
  const fa_status chk = check_fwd_args(q, k, v, B, H, N, N, d, causal, scale, qk_dtype, descale_qk, 1);
  if (chk != FA_OK) return chk;
  if (o == nullptr) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16)) return FA_ERR_ALIGNMENT;
  if (lse != nullptr && !aligned(lse, 4)) return FA_ERR_ALIGNMENT;
  FwdArgs a{q, k, v, o, lse, nullptr, nullptr, B, H, N, N, d, causal != 0, scale, qk_dtype, descale_qk, 1};
  return dispatch_fwd(a, static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_fp8_qrot(const void* q, const void* k8, const void* v, void* o, float* lse, int B, int H, int N,
                          int d, int causal, float scale, const float* dk_blocks, int rotate, const float* signs,
                          float* dq_blocks_out, void* stream) {
  const fa_status chk = check_fwd_args(q, k8, v, B, H, N, N, d, causal, scale, FA_E4M3_BLOCK, dk_blocks, 1);
  if (chk != FA_OK) return chk;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (o == nullptr || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16)) return FA_ERR_ALIGNMENT;
  if (lse != nullptr && !aligned(lse, 4)) return FA_ERR_ALIGNMENT;
  if (signs != nullptr && !aligned(signs, 16)) return FA_ERR_ALIGNMENT;
  if (dq_blocks_out != nullptr && !aligned(dq_blocks_out, 4)) return FA_ERR_ALIGNMENT;
  FwdArgs a{q, k8, v, o, lse, nullptr, nullptr, B, H, N, N, d, causal != 0, scale, FA_E4M3_BLOCK, dk_blocks, 1};
  a.qrot = true;
  a.qrot_rotate = rotate;
  a.qrot_signs = rotate ? signs : nullptr;
  a.dq_out = dq_blocks_out;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return causal ? launch_fwd<128, 2, true, true, false, false, true>(a, s)
                : launch_fwd<128, 2, false, true, false, false, true>(a, s);
}

int fa_fwd_splitkv_splits(int B, int H, int Nq, int Nk, int d) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return 1;
  return auto_splits(B, H, Nq, Nk, d);
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int n_split) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || n_split < 0) return 0;
  if (d != 64 && d != 128 && d != 256) return 0;
  if (n_split == 0) {
    // enough for the automatic schedule with either mask
    const size_t a = plan_bytes(plan_fwd(B, H, Nq, Nk, d, false), B, H, Nq, d);
    const size_t c = plan_bytes(plan_fwd(B, H, Nq, Nk, d, true), B, H, Nq, d);
    return a > c ? a : c;
  }
  return n_split <= 1 ? 0 : part_bytes(B, H, Nq, d, n_split);
}

fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                         int Nk, int d, int causal, float scale, fa_dtype qk_dtype, const float* descale_qk,
                         int n_split, void* workspace, size_t workspace_bytes, void* stream) {
  if (n_split < 0 || B < 1 || H < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  Plan pl;
  if (n_split == 0 && d >= 64 && d <= 256) {
    pl = plan_fwd(B, H, Nq, Nk, d, causal != 0);
    n_split = pl.n_split;
  }
  if (n_split == 0) n_split = 1;
  const fa_status chk = check_fwd_args(q, k, v, B, H, Nq, Nk, d, causal, scale, qk_dtype, descale_qk, n_split);
  if (chk != FA_OK) return chk;
  if (o == nullptr) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16)) return FA_ERR_ALIGNMENT;
  if (lse != nullptr && !aligned(lse, 4)) return FA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_split == 1) {
    FwdArgs a{q, k, v, o, lse, nullptr, nullptr, B, H, Nq, Nk, d, causal != 0, scale, qk_dtype, descale_qk, 1};
    if (pl.tail_split >= 2) {
      const TailLayout tl = tail_layout(pl, d);
      if (workspace == nullptr || workspace_bytes < tl.bytes) return FA_ERR_INVALID_ARG;
      if (!aligned(workspace, 256)) return FA_ERR_ALIGNMENT;
      char* ws = static_cast<char*>(workspace);
      a.tail_split = pl.tail_split;
      a.tail_tiles = pl.tail_tiles;
      a.n_full = pl.n_full;
      a.tail_o = reinterpret_cast<float*>(ws + tl.o);
      a.tail_lse = reinterpret_cast<float*>(ws + tl.lse);
      a.tail_cnt = reinterpret_cast<unsigned long long*>(ws + tl.cnt);
    }
    return dispatch_fwd(a, s);
  }
  if (workspace == nullptr || workspace_bytes < part_bytes(B, H, Nq, d, n_split)) return FA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return FA_ERR_ALIGNMENT;
  float* o_part = static_cast<float*>(workspace);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             ((part_o_bytes(B, H, Nq, d, n_split) + 255) & ~static_cast<size_t>(255)));
  FwdArgs a{q, k, v, nullptr, nullptr, o_part, lse_part, B, H, Nq, Nk, d, causal != 0, scale, qk_dtype, descale_qk,
            n_split};
  const fa_status r = dispatch_fwd(a, s);
  if (r != FA_OK) return r;
  return dispatch_merge(o_part, lse_part, n_split, static_cast<int64_t>(B) * H * Nq, d, o, lse, s);
}

fa_status fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int H,
                         int Nq, int Nk, int d, int causal, float scale, fa_dtype qk_dtype, const float* descale_qk,
                         int n_split, void* stream) {
  const fa_status chk = check_fwd_args(q, k, v, B, H, Nq, Nk, d, causal, scale, qk_dtype, descale_qk, n_split);
  if (chk != FA_OK) return chk;
  if (o_part == nullptr || lse_part == nullptr) return FA_ERR_INVALID_ARG;
  if (!aligned(o_part, 16) || !aligned(lse_part, 4)) return FA_ERR_ALIGNMENT;
  FwdArgs a{q, k, v, nullptr, nullptr, o_part, lse_part, B, H, Nq, Nk, d, causal != 0, scale, qk_dtype, descale_qk,
            n_split};
  return dispatch_fwd(a, static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  return bwd_workspace_bytes(B, H, N, d);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || dout == nullptr || lse == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr || workspace == nullptr)
    return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;  // d = 256: dK and dV alone fill TMEM
  if (static_cast<long long>(B) * H * (bwd_npad(N) / 128) > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * N > (1LL << 40)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 256))
    return FA_ERR_ALIGNMENT;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return causal ? launch_bwd<64, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, workspace, s)
                  : launch_bwd<64, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, workspace, s);
  return causal ? launch_bwd<128, true>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, workspace, s)
                : launch_bwd<128, false>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, workspace, s);
}

fa_status fa_lse_merge(const float* o_part, const float* lse_part, int n_part, int64_t rows, int d, void* o,
                       float* lse, void* stream) {
  if (o_part == nullptr || lse_part == nullptr || o == nullptr) return FA_ERR_INVALID_ARG;
  if (n_part < 1 || rows < 1 || rows > (static_cast<int64_t>(1) << 40)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned(o_part, 16) || !aligned(lse_part, 4) || !aligned(o, 16)) return FA_ERR_ALIGNMENT;
  if (lse != nullptr && !aligned(lse, 4)) return FA_ERR_ALIGNMENT;
  return dispatch_merge(o_part, lse_part, n_part, rows, d, o, lse, static_cast<cudaStream_t>(stream));
}

fa_status fa_hadamard_quant(const void* x, void* out, float* descale_out, int64_t rows, int d, int rotate,
                            const float* signs, void* workspace, size_t workspace_bytes, void* stream) {
  if (descale_out == nullptr || workspace == nullptr) return FA_ERR_INVALID_ARG;
  if (rows < 0 || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || out == nullptr)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < FA_QUANT_WORKSPACE_BYTES) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (rows > kQuantMaxRows) return FA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(descale_out, 4))
    return FA_ERR_ALIGNMENT;
  if (signs != nullptr && !aligned(signs, 16)) return FA_ERR_ALIGNMENT;
  const float* sg = rotate ? signs : nullptr;
  fa::QuantBatch b = {};
  b.x[0] = static_cast<const __nv_bfloat16*>(x);
  b.out[0] = static_cast<uint8_t*>(out);
  b.n = 1;
  unsigned int* ws = static_cast<unsigned int*>(workspace);  // word 0: amax, word 1: barrier counter (n = 1)
  return dispatch_quant_fused(b, descale_out, rows, d, rotate, sg, ws, ws + 1, static_cast<cudaStream_t>(stream));
}

fa_status fa_quant_v_transposed(const void* v, void* out_t, float* descale_out, int BH, int N, int d,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (v == nullptr || out_t == nullptr || descale_out == nullptr || workspace == nullptr) return FA_ERR_INVALID_ARG;
  if (BH < 1 || N < 1 || BH > 65535) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < FA_QUANT_WORKSPACE_BYTES) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(BH) * N > kQuantMaxRows) return FA_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(out_t, 16) || !aligned(workspace, 16) || !aligned(descale_out, 4))
    return FA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int* amax_word = static_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(amax_word, 0, sizeof(unsigned int), s) != cudaSuccess) return FA_ERR_CUDA;
  const int64_t n16 = static_cast<int64_t>(BH) * N * d / 8;
  long long blocks = (n16 + 4095) / 4096;  // 4 chunks of 16 bytes per thread and step
  const long long cap = static_cast<long long>(device_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  fa::quant_t_amax_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<const uint4*>(v), n16, amax_word);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>((N + fa::kQuantTPos - 1) / fa::kQuantTPos), static_cast<unsigned>(BH));
  const auto* x = static_cast<const __nv_bfloat16*>(v);
  auto* o = static_cast<uint8_t*>(out_t);
  switch (d) {
    case 64: fa::quant_t_kernel<64><<<grid, 256, 0, s>>>(x, o, N, amax_word, descale_out); break;
    case 128: fa::quant_t_kernel<128><<<grid, 256, 0, s>>>(x, o, N, amax_word, descale_out); break;
    default: fa::quant_t_kernel<256><<<grid, 256, 0, s>>>(x, o, N, amax_word, descale_out); break;
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_hadamard_quant_multi(const void* const* xs, void* const* outs, float* descales, int ntensors,
                                  int64_t rows, int d, int rotate, const float* signs, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (xs == nullptr || outs == nullptr || descales == nullptr || workspace == nullptr) return FA_ERR_INVALID_ARG;
  if (ntensors < 1 || ntensors > fa::kQuantBatch) return FA_ERR_INVALID_ARG;
  if (rows < 0 || rows > kQuantMaxRows || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < FA_QUANT_WORKSPACE_BYTES) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned(descales, 4) || !aligned(workspace, 16)) return FA_ERR_ALIGNMENT;
  if (signs != nullptr && !aligned(signs, 16)) return FA_ERR_ALIGNMENT;
  fa::QuantBatch b = {};
  for (int i = 0; i < ntensors; ++i) {
    if (rows > 0 && (xs[i] == nullptr || outs[i] == nullptr)) return FA_ERR_INVALID_ARG;
    if (!aligned(xs[i], 16) || !aligned(outs[i], 16)) return FA_ERR_ALIGNMENT;
    b.x[i] = static_cast<const __nv_bfloat16*>(xs[i]);
    b.out[i] = static_cast<uint8_t*>(outs[i]);
  }
  b.n = ntensors;
  unsigned int* ws = static_cast<unsigned int*>(workspace);  // words 0 .. n-1: amax, n .. 2n-1: barrier counters
  return dispatch_quant_fused(b, descales, rows, d, rotate, rotate ? signs : nullptr, ws, ws + ntensors,
                              static_cast<cudaStream_t>(stream));
}

fa_status fa_hadamard_quant_blocks(const void* x, void* out, float* descales, int BH, int N, int d, int rotate,
                                   const float* signs, void* stream) {
  if (x == nullptr || out == nullptr || descales == nullptr) return FA_ERR_INVALID_ARG;
  if (BH < 1 || N < 1 || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const long long nb = (static_cast<long long>(N) + 127) / 128;  // 128-row scale blocks per head
  if (nb * BH > 0x7fffffffLL || static_cast<long long>(BH) * N > (1LL << 40)) return FA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(descales, 4)) return FA_ERR_ALIGNMENT;
  if (signs != nullptr && !aligned(signs, 16)) return FA_ERR_ALIGNMENT;
  const float* sg = rotate ? signs : nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_quant_blocks<64>(x, out, descales, BH, N, rotate, sg, s);
    case 128: return launch_quant_blocks<128>(x, out, descales, BH, N, rotate, sg, s);
    default: return launch_quant_blocks<256>(x, out, descales, BH, N, rotate, sg, s);
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free quantisation (fa_hadamard_quant_noalloc).
//
// The scratch of the quantiser (one amax word per tensor, then one grid
// barrier counter per tensor of a launch) lives in this file-scope device array
// instead of a caller workspace. Every device that
// loads the library holds it until the process exits. In host code the name
// g_noalloc_scratch is only a host-side stand-in, never a device address: the
// kernels get the address cudaGetSymbolAddress returns, looked up once per
// device with that device current.
namespace {

constexpr int kNoallocMaxTensors = 64;
static __device__ __align__(256) unsigned int g_noalloc_scratch[kNoallocMaxTensors + fa::kQuantBatch];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
unsigned int* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use).
fa_status noalloc_scratch(unsigned int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<unsigned int*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status fa_hadamard_quant_noalloc(const void* const* xs, void* const* outs, float* descales, int ntensors,
                                    int64_t rows, int d, int rotate, const float* signs, void* stream) {
  if (xs == nullptr || outs == nullptr || descales == nullptr) return FA_ERR_INVALID_ARG;
  if (ntensors < 1 || ntensors > kNoallocMaxTensors) return FA_ERR_INVALID_ARG;  // scratch holds 64 amax words
  if (rows < 0 || rows > kQuantMaxRows || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned(descales, 4)) return FA_ERR_ALIGNMENT;
  if (signs != nullptr && !aligned(signs, 16)) return FA_ERR_ALIGNMENT;
  for (int i = 0; i < ntensors; ++i) {
    if (rows > 0 && (xs[i] == nullptr || outs[i] == nullptr)) return FA_ERR_INVALID_ARG;
    if (!aligned(xs[i], 16) || !aligned(outs[i], 16)) return FA_ERR_ALIGNMENT;
  }
  unsigned int* scratch = nullptr;
  const fa_status sst = noalloc_scratch(&scratch);
  if (sst != FA_OK) return sst;
  const float* sg = rotate ? signs : nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Up to kQuantBatch tensors per launch; word i of the array is tensor i's
  // amax and the last kQuantBatch words the launch's barrier counters, all
  // zeroed by the launch on this stream, so what an earlier call left there
  // does not matter.
  for (int i0 = 0; i0 < ntensors; i0 += fa::kQuantBatch) {
    fa::QuantBatch b = {};
    b.n = ntensors - i0 < fa::kQuantBatch ? ntensors - i0 : fa::kQuantBatch;
    for (int i = 0; i < b.n; ++i) {
      b.x[i] = static_cast<const __nv_bfloat16*>(xs[i0 + i]);
      b.out[i] = static_cast<uint8_t*>(outs[i0 + i]);
    }
    const fa_status r = dispatch_quant_fused(b, descales + i0, rows, d, rotate, sg, scratch + i0,
                                             scratch + kNoallocMaxTensors, s);
    if (r != FA_OK) return r;
  }
  return FA_OK;
}

const char* fa_status_string(fa_status st) {
  switch (st) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported head dimension or dtype";
    case FA_ERR_ALIGNMENT: return "misaligned pointer";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
  }
  return "unknown status";
}

fa_status fa_device_status(int* code, unsigned int* site, unsigned int* block) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  fa::DevStatus h;
  if (cudaMemcpyFromSymbol(&h, fa::g_fa_status, sizeof(h)) != cudaSuccess) return FA_ERR_CUDA;
  const fa::DevStatus zero = {0, 0, 0, 0};
  if (cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (code) *code = static_cast<int>(h.code);
  if (site) *site = h.site;
  if (block) *block = h.block;
  return FA_OK;
}

int fa_abi_version(void) { return 6; }

#ifdef FA_TEST_HOOKS
// Test build only (not declared in include/, not in the product library): arm
// the withheld P arrival of the next forward launch on the current device.
int fa_test_withhold_p_arrive(int on) {
  const int v = on ? 1 : 0;
  return cudaMemcpyToSymbol(fa::g_fa_test_withhold_p, &v, sizeof(v)) == cudaSuccess ? 0 : 1;
}
#endif

}  // extern "C"

// fa_api.cu — the C ABI declared in include/fa.h: argument checks, TMA tensor
// maps, and the launches of the attention and quantisation kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "attn_fwd.cuh"
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

template <int D, int NQ, bool CAUSAL, bool QK_FP8>
fa_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                     float scale, const float* descale_qk, cudaStream_t stream) {
  using C = FwdCfg<D, NQ, QK_FP8>;
  const int BH = B * H;
  CUtensorMap tmQ, tmK, tmV;
  const CUtensorMapDataType qk_type = QK_FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!fa::make_tmap_3d(&tmQ, q, qk_type, C::EQK, D, N, BH, 128 / C::EQK, C::BM) ||
      !fa::make_tmap_3d(&tmK, k, qk_type, C::EQK, D, N, BH, 128 / C::EQK, C::BN) ||
      !fa::make_tmap_3d(&tmV, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, N, BH, 64, C::BN))
    return FA_ERR_CUDA;
  auto kernel = fa::attn_fwd_kernel<D, NQ, CAUSAL, QK_FP8>;
  static unsigned long long smem_done = 0;
  if (!set_smem_once(kernel, C::SMEM_BYTES, &smem_done)) return FA_ERR_CUDA;
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
  FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.descale_qk = descale_qk;
  p.N = N;
  p.n_qb = (N + NQ * C::BM - 1) / (NQ * C::BM);
  p.scale_log2 = scale * 1.4426950408889634f;
  const long long grid = static_cast<long long>(p.n_qb) * BH;
  kernel<<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D>
fa_status launch_quant(const void* x, void* out, float* descale_out, int64_t rows, int rotate, const float* signs,
                       unsigned int* amax, cudaStream_t stream) {
  using QC = fa::QuantCfg<D>;
  if (cudaMemsetAsync(amax, 0, sizeof(unsigned int), stream) != cudaSuccess) return FA_ERR_CUDA;
  const int64_t steps = (rows + QC::ROWS_PER_STEP - 1) / QC::ROWS_PER_STEP;  // warp-steps of work
  const int64_t warps_per_block = fa::kQuantThreads / 32;
  int64_t blocks = (steps + warps_per_block - 1) / warps_per_block;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 resident blocks of 256 threads per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  uint8_t* ob = static_cast<uint8_t*>(out);
  if (rotate) {
    fa::quant_amax_kernel<D, true><<<static_cast<unsigned>(blocks), fa::kQuantThreads, 0, stream>>>(xb, rows, signs, amax);
    fa::quant_apply_kernel<D, true>
        <<<static_cast<unsigned>(blocks), fa::kQuantThreads, 0, stream>>>(xb, ob, rows, signs, amax, descale_out);
  } else {
    fa::quant_amax_kernel<D, false><<<static_cast<unsigned>(blocks), fa::kQuantThreads, 0, stream>>>(xb, rows, nullptr, amax);
    fa::quant_apply_kernel<D, false>
        <<<static_cast<unsigned>(blocks), fa::kQuantThreads, 0, stream>>>(xb, ob, rows, nullptr, amax, descale_out);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Both quantisation passes in one cooperative launch (quant_fused_kernel): the
// workspace holds the amax word and the grid barrier's counter, zeroed here.
template <int D>
fa_status launch_quant_fused(const void* x, void* out, float* descale_out, int64_t rows, int rotate,
                             const float* signs, unsigned int* ws, cudaStream_t stream) {
  using FC = fa::FusedCfg<D>;
  if (cudaMemsetAsync(ws, 0, 2 * sizeof(unsigned int), stream) != cudaSuccess) return FA_ERR_CUDA;
  auto kernel = rotate ? fa::quant_fused_kernel<D, true> : fa::quant_fused_kernel<D, false>;
  // Co-resident blocks per SM and SM count, looked up once per device (this is
  // host time in front of a ~10 us kernel).
  static int cached_per_sm[2][64] = {};
  static int cached_sms[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FA_ERR_UNSUPPORTED;
  int& per_sm = cached_per_sm[rotate ? 1 : 0][dev];
  int& sms = cached_sms[dev];
  if (sms == 0 && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FA_ERR_CUDA;
  if (per_sm == 0 &&
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, fa::kFusedThreads, 0) != cudaSuccess)
    return FA_ERR_CUDA;
  if (per_sm < 1 || sms < 1) return FA_ERR_CUDA;
  const int64_t steps = (rows + FC::RPW - 1) / FC::RPW;  // warp-steps of work
  int64_t blocks = (steps + fa::kFusedThreads / 32 - 1) / (fa::kFusedThreads / 32);
  const int64_t cap = static_cast<int64_t>(per_sm) * sms;  // all blocks co-resident
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  uint8_t* ob = static_cast<uint8_t*>(out);
  void* args[] = {&xb, &ob, &rows, &signs, &ws, &descale_out};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3(static_cast<unsigned>(blocks)),
                                  dim3(fa::kFusedThreads), args, 0, stream) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 int causal, float scale, fa_dtype qk_dtype, const float* descale_qk, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (qk_dtype != FA_BF16 && qk_dtype != FA_E4M3) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (qk_dtype == FA_E4M3 && d == 64) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return FA_ERR_ALIGNMENT;
  if (lse != nullptr && !aligned(lse, 4)) return FA_ERR_ALIGNMENT;
  if (qk_dtype == FA_E4M3) {
    if (descale_qk == nullptr) return FA_ERR_INVALID_ARG;
    if (!aligned(descale_qk, 4)) return FA_ERR_ALIGNMENT;
  }
  const int rows_per_cta = 128;  // the smallest query block of any kernel
  const long long n_qb = (static_cast<long long>(N) + rows_per_cta - 1) / rows_per_cta;
  if (n_qb * B * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool c = causal != 0;
  if (qk_dtype == FA_BF16) {
    switch (d) {
      case 64: return c ? launch_fwd<64, 2, true, false>(q, k, v, o, lse, B, H, N, scale, nullptr, s)
                        : launch_fwd<64, 2, false, false>(q, k, v, o, lse, B, H, N, scale, nullptr, s);
      case 128: return c ? launch_fwd<128, 2, true, false>(q, k, v, o, lse, B, H, N, scale, nullptr, s)
                         : launch_fwd<128, 2, false, false>(q, k, v, o, lse, B, H, N, scale, nullptr, s);
      default: return c ? launch_fwd<256, 1, true, false>(q, k, v, o, lse, B, H, N, scale, nullptr, s)
                        : launch_fwd<256, 1, false, false>(q, k, v, o, lse, B, H, N, scale, nullptr, s);
    }
  }
  switch (d) {
    case 128: return c ? launch_fwd<128, 2, true, true>(q, k, v, o, lse, B, H, N, scale, descale_qk, s)
                       : launch_fwd<128, 2, false, true>(q, k, v, o, lse, B, H, N, scale, descale_qk, s);
    default: return c ? launch_fwd<256, 1, true, true>(q, k, v, o, lse, B, H, N, scale, descale_qk, s)
                      : launch_fwd<256, 1, false, true>(q, k, v, o, lse, B, H, N, scale, descale_qk, s);
  }
}

fa_status fa_hadamard_quant(const void* x, void* out, float* descale_out, int64_t rows, int d, int rotate,
                            const float* signs, void* workspace, size_t workspace_bytes, void* stream) {
  if (descale_out == nullptr || workspace == nullptr) return FA_ERR_INVALID_ARG;
  if (rows < 0 || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || out == nullptr)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < FA_QUANT_WORKSPACE_BYTES) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (rows > (static_cast<int64_t>(1) << 40)) return FA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(descale_out, 4))
    return FA_ERR_ALIGNMENT;
  if (signs != nullptr && !aligned(signs, 16)) return FA_ERR_ALIGNMENT;
  const float* sg = rotate ? signs : nullptr;
  unsigned int* amax = static_cast<unsigned int*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_quant_fused<64>(x, out, descale_out, rows, rotate, sg, amax, s);
    case 128: return launch_quant_fused<128>(x, out, descale_out, rows, rotate, sg, amax, s);
    default: return launch_quant_fused<256>(x, out, descale_out, rows, rotate, sg, amax, s);
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free quantisation (fa_hadamard_quant_noalloc).
//
// The scratch of the quantiser (one amax word per tensor) lives in this
// file-scope device array instead of a caller workspace. Every device that
// loads the library holds it until the process exits. In host code the name
// g_noalloc_scratch is only a host-side stand-in, never a device address: the
// kernels get the address cudaGetSymbolAddress returns, looked up once per
// device with that device current.
namespace {

constexpr int kNoallocScratchBytes = 256;
constexpr int kNoallocMaxTensors = kNoallocScratchBytes / static_cast<int>(sizeof(unsigned int));  // 64
static __device__ __align__(256) unsigned int g_noalloc_scratch[kNoallocMaxTensors];

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
  if (ntensors < 1 || ntensors > kNoallocMaxTensors) return FA_ERR_INVALID_ARG;  // scratch holds 64 words
  if (rows < 0 || rows > (static_cast<int64_t>(1) << 40) || (rotate != 0 && rotate != 1)) return FA_ERR_INVALID_ARG;
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
  for (int i = 0; i < ntensors; ++i) {
    // Word i of the array is tensor i's amax; launch_quant zeroes it first on
    // this stream, so what an earlier call left there does not matter.
    fa_status r;
    switch (d) {
      case 64: r = launch_quant<64>(xs[i], outs[i], descales + i, rows, rotate, sg, scratch + i, s); break;
      case 128: r = launch_quant<128>(xs[i], outs[i], descales + i, rows, rotate, sg, scratch + i, s); break;
      default: r = launch_quant<256>(xs[i], outs[i], descales + i, rows, rotate, sg, scratch + i, s); break;
    }
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

int fa_abi_version(void) { return 1; }

}  // extern "C"

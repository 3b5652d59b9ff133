// tmap.h — host-side construction of TMA tensor maps without linking libcuda:
// cuTensorMapEncodeTiled is fetched through the runtime's driver entry point.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cstdint>

namespace fa {

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// A 3-D row-major tensor [dim2][dim1][dim0] (dim0 contiguous) of elements of
// `esize` bytes, tiled in boxes of box0 x box1 x 1 with the given swizzle
// (128-byte by default). Out-of-range elements of a box read as zero and are
// not written by stores. Returns false on failure.
inline bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int esize,
                         uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0, uint32_t box1,
                         CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = get_encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0 * static_cast<uint64_t>(esize), dim0 * dim1 * static_cast<uint64_t>(esize)};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A 2-D row-major tensor [dim1][dim0] (dim0 contiguous), tiled in boxes of
// box0 x box1 with the given swizzle (128-byte by default; box0 * esize must
// not exceed the swizzle span). Out-of-range elements of a box read as zero
// and are not written by stores. Returns false on failure.
inline bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int esize, uint64_t dim0,
                         uint64_t dim1, uint32_t box0, uint32_t box1,
                         CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = get_encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {dim0, dim1};
  cuuint64_t strides[1] = {dim0 * static_cast<uint64_t>(esize)};
  cuuint32_t box[2] = {box0, box1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fa

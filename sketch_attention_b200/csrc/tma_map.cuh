// Tensor maps (TMA descriptors) of the tensor-core kernels, and their shared-memory limit: row-major
// matrices [outer, inner] of 2-byte elements (bf16 or fp16) copied in boxes of box_inner x box_outer
// elements.
// cuTensorMapEncodeTiled is taken from the driver once per process.  The
// encoder checks the base (16-byte aligned), the row pitch (a multiple of 16
// bytes) and the box; a kernel's box x coordinate must itself be a multiple of
// 8 elements (16 bytes), which every caller's coordinates are (0, 64, 16 j).
#pragma once
#include <cuda.h>

#include <mutex>
#include <string>

#include "common.cuh"

namespace sa {

using TmaEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline TmaEncodeFn tma_encode_fn() {
  static TmaEncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      fn = (TmaEncodeFn)q;
  });
  return fn;
}

// pitch: elements between consecutive rows (default: inner); elements past `inner`
// or `outer` read as zero
inline sa_status tma_map_2byte(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                               uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz,
                               uint64_t pitch = 0) {
  TmaEncodeFn enc = tma_encode_fn();
  if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {(pitch ? pitch : inner) * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return SA_OK;
}
inline sa_status tma_map_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz,
                              uint64_t pitch = 0) {
  return tma_map_2byte(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, outer, box_inner, box_outer, swz, pitch);
}

// A kernel's dynamic shared-memory limit is an attribute of the device's context: set it once
// per device (bit `device` of *done), under `mu`.
inline void set_smem_limit_once(const void* kernel, int bytes, unsigned long long* done, std::mutex& mu) {
  const int dev = device_info().device & 63;
  std::lock_guard<std::mutex> lock(mu);
  if (*done & (1ull << dev)) return;
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  *done |= 1ull << dev;
}

}  // namespace sa

// Host helpers for the tcgen05 GEMM: 2-D bf16 tensor maps with 128-byte swizzle
// (cuTensorMapEncodeTiled fetched through the runtime's driver entry point, so the
// library does not link libcuda) and the launch of a GEMM configuration.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "tc_gemm.cuh"

namespace dspark {
namespace tc {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A bf16 matrix of `rows` x `cols` (cols contiguous, row stride `ld` elements) seen by
// TMA in boxes of box_cols x box_rows (box_cols * 2 = 128 bytes).  Reads outside the
// matrix return zeros.
inline bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                     uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An FP32 output seen by tensor stores of 32 x 32 blocks (128-byte swizzle): a matrix
// of `rows` x `cols` (row stride `ld` elements), or `planes` such matrices `plane`
// elements apart (3-D).  Blocks reaching past the matrix are clipped.
inline bool make_out_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                         uint64_t planes = 0, uint64_t plane = 0) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {cols, rows, planes};
  const cuuint64_t strides[2] = {ld * 4, plane * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, planes ? 3 : 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

// D[M, N] = A . B^T over K (A is M x K, B is N x K in the math), operands as described
// by their tensor maps; work split into `ksplit` slices of K.  With `m_bound`, rows m
// with m_base + m >= *m_bound (a count the device holds) are skipped.  Returns the
// launch error.
template <int BN, bool A_MN, bool B_MN, int STAGES, class Epi>
cudaError_t gemm(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K, int ksplit, const Epi& epi,
                 uint32_t* status, cudaStream_t s, const int32_t* m_bound = nullptr, int m_base = 0,
                 const CUtensorMap* out = nullptr) {
  if (Epi::kTma && out == nullptr) return cudaErrorInvalidValue;
  WorkMap wm;
  wm.m_bound = m_bound;
  wm.m_base = m_base;
  wm.m_tiles = (M + BM - 1) / BM;
  wm.n_tiles = (N + BN - 1) / BN;
  wm.kchunks = (K + BK - 1) / BK;
  wm.ksplit = std::max(1, std::min(ksplit, wm.kchunks));
  const int W = wm.m_tiles * wm.n_tiles * wm.ksplit;
  auto kern = gemm_kernel<BN, A_MN, B_MN, STAGES, Epi>;
  constexpr size_t smem = gemm_smem_bytes<BN, STAGES>();
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] { attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)); });
  if (attr_err != cudaSuccess) return attr_err;
  const int grid = std::min(W, sm_count());
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kThreads, smem, s>>>(a, b, out ? *out : a, wm, epi, status);
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace dspark

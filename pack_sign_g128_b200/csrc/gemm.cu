// w1_gemm: prefill-regime 1-bit group-128 product on tcgen05 tensor cores.
//
//   y[m,n] = sum_g s[n,g] * sum_{k in g} (1 - 2 bit[n,k]) x[m,k]
//
// Two kernels on the caller's stream (the sign GEMM of sign_gemm.cu):
//  1. sg_prep_kernel: xs[m] = fp16(x[m] * 2^c_m), an exact power-of-two per
//     token putting max |x[m]| in [2^14, 2^15) (fp16 holds every bf16
//     significand; the scale keeps the row inside fp16's range).
//  2. sg_gemm_kernel with the group scales: the weight operand is +-s[n,g] in
//     fp16 -- the scale with the sign bit of the weight -- so the blockwise
//     scale is applied inside the tensor core and all of K accumulates in one
//     fp32 TMEM tile per 128 x 128 output tile; the epilogue multiplies by
//     2^-c_m.  Every product is exact; the only rounding is fp32 accumulation.
// xs and the token scales live in the caller's workspace.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <mutex>

#include "w1_common.cuh"

namespace w1 {

template <bool HALF_OUT>
cudaError_t launch_sg_gemm(const SgParams& p, const void* bmat, int64_t bcols, cudaStream_t stream, int num_sms);
cudaError_t launch_sg_prep(const uint16_t* x, const uint16_t* bdiag, const uint16_t* mid, int64_t n, int64_t r,
                          int64_t B, __half* xs, float* cscale, float* dscale, float* dinv, cudaStream_t stream);

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix, box {64 cols, box_rows},
// 128-byte swizzle, zero fill out of bounds.
bool make_tmap_bf16_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D uint32 tensor map over row-major sign words [rows][words], box
// {box_words, 16 rows}, swizzle equal to the box row bytes (16 B: none, 32, 64
// or 128 B), zero fill out of bounds.
bool make_tmap_u32_rows(CUtensorMap* map, const void* base, int64_t rows, int64_t words, int box_words) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(words), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(words) * 4};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_words), 16};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (box_words * 4 == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  if (box_words * 4 == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  if (box_words * 4 == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D uint32 tensor map over row-major sign words [rows][words]: box {32 words
// (8 groups of 128 weights), box_rows}, 128-byte swizzle, zero fill out of
// bounds (rows past N, words past K / 32).
bool make_tmap_u32_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t words, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || box_rows < 1 || box_rows > 256) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(words), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(words) * 4};
  cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t gemm_workspace_bytes(int64_t M, int64_t K) {
  const size_t xs_bytes = (static_cast<size_t>(M) * K * 2 + 1023) / 1024 * 1024;
  return xs_bytes + (static_cast<size_t>(M) * 4 + 255) / 256 * 256;
}

cudaError_t launch_gemm(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                        const uint16_t* x, int64_t M, float* y, void* workspace, cudaStream_t stream,
                        int num_sms) {
  const size_t xs_bytes = (static_cast<size_t>(M) * K * 2 + 1023) / 1024 * 1024;
  __half* xs = static_cast<__half*>(workspace);
  float* cscale = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + xs_bytes);
  cudaError_t err = launch_sg_prep(x, nullptr, nullptr, K, 0, M, xs, cscale, nullptr, nullptr, stream);
  if (err != cudaSuccess) return err;
  SgParams p = {};
  p.signs = signs;
  p.gscales = scales;
  p.s1 = cscale;
  p.out_f = y;
  p.M = static_cast<int>(M);
  p.rows = static_cast<int>(N);
  p.K = static_cast<int>(K);
  return launch_sg_gemm<false>(p, xs, K, stream, num_sms);
}

}  // namespace w1

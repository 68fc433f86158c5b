// w1_gemm: prefill-regime 1-bit group-128 product on tcgen05 tensor cores.
//
//   y[m,n] = sum_g s[n,g] * sum_{k in g} (1 - 2 bit[n,k]) x[m,k]
//
// Swap-AB formulation, one CTA per SM, persistent over 128 x 128 output tiles
// (128 weight rows n  x  128 tokens m):
//   D^T[n, m] (TMEM, fp32)  =  A[n, k] (TMEM, +-1 bf16)  x  X[m, k]^T (smem, bf16)
//  * warp 0      TMA producer: X tiles (128 tokens x 128 k) with 128B swizzle.
//  * warp 1      MMA issuer: per 128-wide K chunk (one scale group), 8 MMAs
//                (K = 16 each) into a fresh TMEM chunk buffer.
//  * warps 2-5   expanders: thread = weight row = TMEM lane.  Each 128-bit
//                sign chunk becomes 64 columns of +-1 bf16 pairs written with
//                tcgen05.st -- the expanded weights never touch shared memory.
//  * warps 6-9   promoters: thread = weight row.  Read the finished chunk
//                from TMEM, acc[m] += s[n,g] * chunk[m] in registers (the
//                blockwise-scale fold), and store y at the end of the tile.
// Every chunk product is exact in the tensor core (+-1 times bf16) with fp32
// accumulation, so the only rounding is fp32 accumulation.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <mutex>

#include "w1_common.cuh"

namespace w1 {

namespace gemm {
constexpr int BN = 128;           // weight rows per tile (MMA M, TMEM lanes)
constexpr int BM = 128;           // tokens per tile (MMA N)
constexpr int BK = 128;           // K per chunk (one scale group)
constexpr int NSX = 4;            // X smem stages
constexpr int NSA = 4;            // A (expanded weights) TMEM stages
constexpr int kThreads = 320;     // 10 warps
constexpr int kXStageBytes = BM * BK * 2;  // 32 KB
constexpr uint32_t kIdesc = idesc_f16(BN, BM, 1, 1);
// TMEM columns: [0, 256) two chunk buffers of BM fp32 columns; [256, 512) A stages.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol0 = 256;

struct Smem {
  alignas(1024) unsigned char x[NSX][kXStageBytes];
  uint64_t full_x[NSX], empty_x[NSX];
  uint64_t full_a[NSA], empty_a[NSA];
  uint64_t full_c[2], empty_c[2];
  uint32_t tmem_base;
};
}  // namespace gemm

struct GemmParams {
  const uint32_t* signs;
  const uint16_t* scales;
  float* y;
  int M, N, K;
  int MT, NT, NK;  // m tiles, n tiles, k chunks
};

__global__ void __launch_bounds__(gemm::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmParams p) {
  using namespace gemm;
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSX; ++i) {
      mbar_init(&sm.full_x[i], 1);
      mbar_init(&sm.empty_x[i], 1);
    }
    for (int i = 0; i < NSA; ++i) {
      mbar_init(&sm.full_a[i], 128);
      mbar_init(&sm.empty_a[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.full_c[i], 1);
      mbar_init(&sm.empty_c[i], 128);
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_x) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();

  const int ntiles = p.MT * p.NT;
  const int NK = p.NK;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (X)
    if (lane == 0) {
      uint32_t c = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int mt = tile % p.MT;
        for (int kc = 0; kc < NK; ++kc, ++c) {
          const int s = c % NSX;
          if (!mbar_wait(&sm.empty_x[s], ((c / NSX) & 1) ^ 1)) goto done_prod;
          mbar_arrive_expect_tx(&sm.full_x[s], kXStageBytes);
          tma_load_2d(sm.x[s], &tmap_x, kc * BK, mt * BM, &sm.full_x[s]);
          tma_load_2d(sm.x[s] + kXStageBytes / 2, &tmap_x, kc * BK + 64, mt * BM, &sm.full_x[s]);
        }
      }
    done_prod:;
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t c = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        for (int kc = 0; kc < NK; ++kc, ++c) {
          const int sx = c % NSX, sa = c % NSA, cb = c & 1;
          if (!mbar_wait(&sm.full_x[sx], (c / NSX) & 1)) goto done_mma;
          if (!mbar_wait(&sm.full_a[sa], (c / NSA) & 1)) goto done_mma;
          if (!mbar_wait(&sm.empty_c[cb], ((c >> 1) & 1) ^ 1)) goto done_mma;
          tc_fence_after();
          const uint32_t xbase = smem_u32(sm.x[sx]);
          const uint32_t d = tmem + cb * BM;
          const uint32_t a = tmem + kAcol0 + sa * 64;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t baddr = xbase + (kk >> 2) * (kXStageBytes / 2) + (kk & 3) * 32;
            tc_mma_ts(d, a + kk * 8, smem_desc_sw128(baddr), kIdesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(&sm.empty_x[sx]);
          tc_commit(&sm.empty_a[sa]);
          tc_commit(&sm.full_c[cb]);
        }
      }
    done_mma:;
    }
  } else if (warp < 6) {
    // ------------------------------------------------ expanders
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;  // row within tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t wrow = p.K >> 5;
    uint32_t c = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      const int nt = tile / p.MT;
      const int n = nt * BN + rl;
      const bool valid = n < p.N;
      const uint4* wp = reinterpret_cast<const uint4*>(p.signs + static_cast<int64_t>(valid ? n : 0) * wrow);
      uint4 nxt = valid ? __ldg(wp) : make_uint4(0, 0, 0, 0);
      for (int kc = 0; kc < NK; ++kc, ++c) {
        const uint4 cur = nxt;
        if (kc + 1 < NK && valid) nxt = __ldg(wp + kc + 1);
        const int sa = c % NSA;
        if (!mbar_wait_warp(&sm.empty_a[sa], ((c / NSA) & 1) ^ 1)) goto done_exp;
        tc_fence_after();
        const uint32_t words[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[32];
#pragma unroll
          for (int wi = 0; wi < 2; ++wi) {
            const uint32_t w = words[half * 2 + wi];
#pragma unroll
            for (int pp = 0; pp < 16; ++pp) {
              // pair (k, k+1) = bits (2pp, 2pp+1): signs to bit 15 and bit 31
              const uint32_t src = (pp < 8) ? w : (w >> 16);
              const int b = 2 * (pp & 7);
              const uint32_t m = src & (3u << b);
              const uint32_t t = m * (0x40008000u >> b);
              r[wi * 16 + pp] = (t & 0x80008000u) | 0x3F803F80u;
            }
          }
          tmem_st32(tmem + lane_addr + kAcol0 + sa * 64 + half * 32, r);
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.full_a[sa]);
      }
    }
  done_exp:;
  } else {
    // ------------------------------------------------ promoters + epilogue
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int NG = p.K >> 7;
    uint32_t c = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      const int mt = tile % p.MT, nt = tile / p.MT;
      const int n = nt * BN + rl;
      const bool valid = n < p.N;
      const uint16_t* sp = p.scales + static_cast<int64_t>(valid ? n : 0) * NG;
      float acc[BM];
#pragma unroll
      for (int j = 0; j < BM; ++j) acc[j] = 0.f;
      uint16_t s_next = valid ? __ldg(sp) : 0;
      for (int kc = 0; kc < NK; ++kc, ++c) {
        const float s = __half2float(__ushort_as_half(s_next));
        if (kc + 1 < NK && valid) s_next = __ldg(sp + kc + 1);
        const int cb = c & 1;
        if (!mbar_wait_warp(&sm.full_c[cb], (c >> 1) & 1)) goto done_prom;
        tc_fence_after();
#pragma unroll
        for (int q4 = 0; q4 < BM / 32; ++q4) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + cb * BM + q4 * 32, r);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[q4 * 32 + j] = fmaf(s, __uint_as_float(r[j]), acc[q4 * 32 + j]);
        }
        tc_fence_before();
        mbar_arrive(&sm.empty_c[cb]);
      }
      if (valid) {
        float* yp = p.y + static_cast<int64_t>(mt) * BM * p.N + n;
        const int mrem = min(BM, p.M - mt * BM);
#pragma unroll
        for (int j = 0; j < BM; ++j)
          if (j < mrem) __stcs(yp + static_cast<int64_t>(j) * p.N, acc[j]);
      }
    }
  done_prom:;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  pdl_launch_dependents();
}

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

cudaError_t launch_gemm(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                        const uint16_t* x, int64_t M, float* y, cudaStream_t stream, int num_sms) {
  using namespace gemm;
  CUtensorMap tmap;
  if (!make_tmap_bf16_sw128(&tmap, x, M, K, BM)) return cudaErrorInvalidValue;
  GemmParams p = {};
  p.signs = signs;
  p.scales = scales;
  p.y = y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.MT = static_cast<int>((M + BM - 1) / BM);
  p.NT = static_cast<int>((N + BN - 1) / BN);
  p.NK = static_cast<int>(K / BK);
  const int ntiles = p.MT * p.NT;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t err = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ntiles < num_sms ? ntiles : num_sms));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_kernel, tmap, p);
}

}  // namespace w1

// DBF chain for many batch rows (B > 8) on tcgen05 tensor cores.
//
//   y = a (.) ( U . ( mid (.) ( V . ( b (.) x ) ) ) )      ("LLM binarization
//   episode 01: DBF", section 4 -- the chain, evaluated in order)
//
// Both binary products are plain +-1 contractions (no group scales), so each
// 128 x 128 output tile accumulates all of K in one TMEM accumulator:
//  1. dbf_prep_kernel: x_s[t] = fp16( b (.) x[t] * 2^c_t ) with a per-row
//     power of two putting max |b x| in [2^14, 2^15) (exact scaling; fp16
//     keeps 11 significant bits of b x, which bf16 would not), and the row's
//     L1 norm, from which a second power of two d_t bounds |mid (.) h| * 2^d_t
//     below 2^15 so the fp16 intermediate cannot overflow.
//  2. dbf_gemm<phase 1>: D = V . x_s^T (A = +-1 fp16 rows of V expanded into
//     TMEM, B = x_s by TMA); epilogue h_s[t][j] = fp16(mid_j D 2^(d_t - c_t)).
//  3. dbf_gemm<phase 2>: D = U . h_s^T; epilogue y[t][i] = a_i D 2^-d_t.
// Products of +-1 and fp16 are exact; accumulation is fp32.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "w1_common.cuh"

namespace w1 {

bool make_tmap_bf16_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows);

namespace dbftc {
constexpr int BN = 128, BM = 128, BK = 128;
constexpr int NSX = 4, NSA = 4;
constexpr int kThreads = 320;
constexpr int kXStage = BM * BK * 2;
constexpr uint32_t kIdesc = idesc_f16(BN, BM, 0, 0);  // fp16 x fp16 -> fp32
constexpr uint32_t kAcol0 = 256;

struct Smem {
  alignas(1024) unsigned char x[NSX][kXStage];
  uint64_t full_x[NSX], empty_x[NSX];
  uint64_t full_a[NSA], empty_a[NSA];
  uint64_t full_c[2], empty_c[2];
  uint32_t tmem_base;
};

// Workspace of the tensor path (after the 256-byte barrier header):
// per-row scales (float [B] 2^-c_t, float [B] 2^d_t), x_s fp16 [B][n],
// h_s fp16 [B][r].
struct Ws {
  size_t cscale, dscale, dinv, xs, hs, total;
};
__host__ __device__ inline Ws ws_layout(int64_t B, int64_t r, int64_t n) {
  Ws w;
  size_t off = 256;
  w.cscale = off;
  off += (4 * B + 255) / 256 * 256;
  w.dscale = off;
  off += (4 * B + 255) / 256 * 256;
  w.dinv = off;
  off += (4 * B + 255) / 256 * 256;
  w.xs = off;
  off += (2 * B * n + 1023) / 1024 * 1024;
  w.hs = off;
  off += (2 * B * r + 1023) / 1024 * 1024;
  w.total = off;
  return w;
}
}  // namespace dbftc

// One CTA per batch row.
__global__ void __launch_bounds__(256) dbf_prep_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ bdiag,
                                                       const uint16_t* __restrict__ mid, int n, int r,
                                                       __half* __restrict__ xs, float* __restrict__ cscale,
                                                       float* __restrict__ dscale, float* __restrict__ dinv) {
  pdl_wait();
  __shared__ float red[2][8];
  const int t = blockIdx.x;
  const uint16_t* xr = x + static_cast<int64_t>(t) * n;
  float mx = 0.f, l1 = 0.f;
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const float v = __uint_as_float(static_cast<uint32_t>(xr[k]) << 16) * __half2float(__ushort_as_half(bdiag[k]));
    mx = fmaxf(mx, fabsf(v));
    l1 += fabsf(v);
  }
  float mm = 0.f;
  for (int j = threadIdx.x; j < r; j += blockDim.x) mm = fmaxf(mm, fabsf(__half2float(__ushort_as_half(mid[j]))));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, o);
    mm = fmaxf(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, o));
  }
  __shared__ float red_mm[8];
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = mx;
    red[1][threadIdx.x >> 5] = l1;
    red_mm[threadIdx.x >> 5] = mm;
  }
  __syncthreads();
  mx = 0.f;
  l1 = 0.f;
  mm = 0.f;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) {
    mx = fmaxf(mx, red[0][i]);
    l1 += red[1][i];
    mm = fmaxf(mm, red_mm[i]);
  }
  // c: max |b x| 2^c in [2^14, 2^15);  d: mm * l1 * 2^d <= 2^15 (l1 rounded up)
  int c = 0, d = 0;
  if (mx > 0.f) {
    int E;
    frexpf(mx, &E);  // mx < 2^E
    c = 15 - E;
  }
  if (mm > 0.f && l1 > 0.f) {
    int E;
    frexpf(mm * l1 * 1.0001f, &E);  // < 2^E
    d = 15 - E;
  }
  const float cs = ldexpf(1.f, c);
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const float v = __uint_as_float(static_cast<uint32_t>(xr[k]) << 16) * __half2float(__ushort_as_half(bdiag[k]));
    xs[static_cast<int64_t>(t) * n + k] = __float2half_rn(v * cs);
  }
  if (threadIdx.x == 0) {
    cscale[t] = ldexpf(1.f, -c);
    dscale[t] = ldexpf(1.f, d);
    dinv[t] = ldexpf(1.f, -d);
  }
  pdl_launch_dependents();
}

struct DbfGemmParams {
  const uint32_t* signs;   // [rows][K/32]
  const uint16_t* rdiag;   // [rows] fp16: mid (phase 1) or a (phase 2)
  const float* s1;         // per token: 2^-c (phase 1) or 2^-d (phase 2)
  const float* s2;         // per token: 2^d (phase 1) or unused
  __half* out_h;           // phase 1 output [M][rows]
  float* out_f;            // phase 2 output [M][rows]
  int M, rows, K, MT, NT, NK;
};

template <bool PHASE1>
__global__ void __launch_bounds__(dbftc::kThreads, 1)
    dbf_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const DbfGemmParams p) {
  using namespace dbftc;
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_b) : "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();
  const int ntiles = p.MT * p.NT;
  const int NK = p.NK;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t c = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int mt = tile % p.MT;
        for (int kc = 0; kc < NK; ++kc, ++c) {
          const int s = c % NSX;
          if (!mbar_wait(&sm.empty_x[s], ((c / NSX) & 1) ^ 1)) goto done_prod;
          mbar_arrive_expect_tx(&sm.full_x[s], kXStage);
          tma_load_2d(sm.x[s], &tmap_b, kc * BK, mt * BM, &sm.full_x[s]);
          tma_load_2d(sm.x[s] + kXStage / 2, &tmap_b, kc * BK + 64, mt * BM, &sm.full_x[s]);
        }
      }
    done_prod:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t c = 0, tl = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
        const int cb = tl & 1;
        if (!mbar_wait(&sm.empty_c[cb], ((tl >> 1) & 1) ^ 1)) goto done_mma;
        tc_fence_after();
        const uint32_t d = tmem + cb * BM;
        for (int kc = 0; kc < NK; ++kc, ++c) {
          const int sx = c % NSX, sa = c % NSA;
          if (!mbar_wait(&sm.full_x[sx], (c / NSX) & 1)) goto done_mma;
          if (!mbar_wait(&sm.full_a[sa], (c / NSA) & 1)) goto done_mma;
          tc_fence_after();
          const uint32_t xbase = smem_u32(sm.x[sx]);
          const uint32_t a = tmem + kAcol0 + sa * 64;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t baddr = xbase + (kk >> 2) * (kXStage / 2) + (kk & 3) * 32;
            tc_mma_ts(d, a + kk * 8, smem_desc_sw128(baddr), kIdesc, (kc > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&sm.empty_x[sx]);
          tc_commit(&sm.empty_a[sa]);
        }
        tc_commit(&sm.full_c[cb]);
      }
    done_mma:;
    }
  } else if (warp < 6) {
    // expanders: +-1 fp16 pairs (0x3C00 = 1.0) into TMEM, thread = row
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t wrow = p.K >> 5;
    uint32_t c = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      const int nt = tile / p.MT;
      const int n = nt * BN + rl;
      const bool valid = n < p.rows;
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
          uint32_t rr[32];
#pragma unroll
          for (int wi = 0; wi < 2; ++wi) {
            const uint32_t w = words[half * 2 + wi];
#pragma unroll
            for (int pp = 0; pp < 16; ++pp) {
              const uint32_t src = (pp < 8) ? w : (w >> 16);
              const int b = 2 * (pp & 7);
              const uint32_t m = src & (3u << b);
              const uint32_t tt = m * (0x40008000u >> b);
              rr[wi * 16 + pp] = (tt & 0x80008000u) | 0x3C003C00u;
            }
          }
          tmem_st32(tmem + lane_addr + kAcol0 + sa * 64 + half * 32, rr);
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.full_a[sa]);
      }
    }
  done_exp:;
  } else {
    // epilogue: one accumulator per tile, scaled by the row diagonal and the token scales
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t tl = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
      const int mt = tile % p.MT, nt = tile / p.MT;
      const int n = nt * BN + rl;
      const bool valid = n < p.rows;
      const float rd = valid ? __half2float(__ushort_as_half(p.rdiag[n])) : 0.f;
      const int cb = tl & 1;
      if (!mbar_wait_warp(&sm.full_c[cb], (tl >> 1) & 1)) goto done_epi;
      tc_fence_after();
      const int mrem = min(BM, p.M - mt * BM);
#pragma unroll
      for (int q4 = 0; q4 < BM / 32; ++q4) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_addr + cb * BM + q4 * 32, rr);
        tc_wait_ld();
        if (valid) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = q4 * 32 + j;
            if (m < mrem) {
              const int64_t tok = static_cast<int64_t>(mt) * BM + m;
              if (PHASE1) {
                const float v = rd * __uint_as_float(rr[j]) * (__ldg(p.s1 + tok) * __ldg(p.s2 + tok));
                p.out_h[tok * p.rows + n] = __float2half_rn(v);
              } else {
                p.out_f[tok * p.rows + n] = rd * __uint_as_float(rr[j]) * __ldg(p.s1 + tok);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.empty_c[cb]);
    }
  done_epi:;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ host side

size_t dbf_tc_workspace_bytes(int64_t r, int64_t n, int64_t B) { return dbftc::ws_layout(B, r, n).total; }

template <bool PHASE1>
static cudaError_t launch_dbf_gemm(const DbfGemmParams& p, const void* bmat, int64_t bcols, cudaStream_t stream,
                                   int num_sms) {
  using namespace dbftc;
  CUtensorMap tm;
  // fp16 and bf16 share the 2-byte element layout the tensor map describes
  if (!make_tmap_bf16_sw128(&tm, bmat, p.M, bcols, BM)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t err =
      cudaFuncSetAttribute(dbf_gemm_kernel<PHASE1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int ntiles = p.MT * p.NT;
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
  return cudaLaunchKernelEx(&cfg, dbf_gemm_kernel<PHASE1>, tm, p);
}

cudaError_t launch_dbf_tc(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                          const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B, float* y,
                          void* workspace, cudaStream_t stream, int num_sms) {
  using namespace dbftc;
  const Ws L = ws_layout(B, r, n);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  float* cs = reinterpret_cast<float*>(ws + L.cscale);
  float* ds = reinterpret_cast<float*>(ws + L.dscale);
  float* di = reinterpret_cast<float*>(ws + L.dinv);
  __half* xs = reinterpret_cast<__half*>(ws + L.xs);
  __half* hs = reinterpret_cast<__half*>(ws + L.hs);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(B));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, dbf_prep_kernel, x, b, mid, static_cast<int>(n), static_cast<int>(r), xs,
                                       cs, ds, di);
  if (err != cudaSuccess) return err;
  DbfGemmParams p1 = {};
  p1.signs = B2;
  p1.rdiag = mid;
  p1.s1 = cs;
  p1.s2 = ds;
  p1.out_h = hs;
  p1.M = static_cast<int>(B);
  p1.rows = static_cast<int>(r);
  p1.K = static_cast<int>(n);
  p1.MT = static_cast<int>((B + BM - 1) / BM);
  p1.NT = static_cast<int>((r + BN - 1) / BN);
  p1.NK = static_cast<int>(n / BK);
  err = launch_dbf_gemm<true>(p1, xs, n, stream, num_sms);
  if (err != cudaSuccess) return err;
  // phase 2 undoes the intermediate's scale: s1 = 2^-d
  DbfGemmParams p2 = {};
  p2.signs = B1;
  p2.rdiag = a;
  p2.s1 = di;
  p2.out_f = y;
  p2.M = static_cast<int>(B);
  p2.rows = static_cast<int>(m);
  p2.K = static_cast<int>(r);
  p2.MT = p1.MT;
  p2.NT = static_cast<int>((m + BN - 1) / BN);
  p2.NK = static_cast<int>(r / BK);
  return launch_dbf_gemm<false>(p2, hs, r, stream, num_sms);
}

}  // namespace w1

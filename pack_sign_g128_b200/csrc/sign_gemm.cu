// Tensor-core product of 1-bit weight rows with many token rows (tcgen05),
// shared by w1_gemm (group-128 scales) and the DBF chain (+-1 factors with
// diagonals):
//
//   D[n][m] = sum_k (1 - 2 bit[n][k]) * s[n][k/128] * xs[m][k]
//
// ("1-bit group-128 sign packing": y = sum_g s_g sum_{k in g} sign * x; the
// group scale is folded into the weight operand, which is exact because s is
// an fp16 value and a sign flip only sets its top bit.)
//  * sg_prep_kernel: xs = fp16(x * 2^c_t) per token row (exact scaling).
//  * sg_gemm_kernel: one CTA per SM, persistent over output tiles of 128
//    weight rows x BM tokens (BM = 256, or 128 when 256-token tiles would not
//    fill the GPU), swap-AB: D^T (TMEM, fp32, two accumulators of BM columns)
//    = A (+-s fp16) x xs^T (shared memory, fp16, by TMA), 128 x BM x 16 MMAs.
//    A sits in shared memory (BM = 256) or in TMEM (BM = 128: row = lane, k
//    pairs along the columns, beside the accumulators), which takes its
//    writes and the MMA's reads of it off shared memory.  Pipeline stages are
//    128 wide in K (one scale group, two 64-wide 128-byte swizzle atoms of
//    xs), 2 deep at BM = 256 (192 KB), 4 deep with A in TMEM (128 KB):
//    warp 0 TMA producer (xs: two BM x 64 boxes per stage, whose transaction
//    bytes complete on the stage's full barrier); warp 1 MMA issuer (one wait
//    per stage, then 8 MMAs, all of K into one accumulator per tile); 4 or 8
//    expander warps (thread = weight row, all of a stage or one 64-wide half:
//    sign words + the group scale -> fp16 pairs +-s, written as 16-byte
//    chunks in the 128B-swizzled K-major layout the MMA reads, or as TMEM
//    columns; words prefetched 4 stages ahead in registers); 4 epilogue warps
//    (thread = TMEM lane: row diagonal and token scale, store), draining one
//    accumulator while the MMA fills the other.
// Products of +-s and fp16 are exact in the tensor core; accumulation is fp32.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "w1_common.cuh"

namespace w1 {

bool make_tmap_bf16_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows);

namespace sg {
// Expander warps per CTA for 256- and 128-token tiles, and where 128-token
// tiles keep the weight operand.  Measured (one B200, the 4096^3 DBF chain at
// 512 rows / the 2048 x 14336 x 4096 GEMM forced to 128-token tiles):
// shared memory, 4 expanders 0.089 ms / 0.300 ms; TMEM, 4: 0.083 / 0.300;
// TMEM, 8: 0.077 / 0.284.  256-token tiles: 8 expanders no faster (0.208 vs
// 0.203 ms), and TMEM has no room for their weight stages beside two
// 256-column accumulators.
constexpr int kExp256 = 4;
constexpr int kExp128 = 8;
constexpr bool kTmemA128 = true;
constexpr int BN = 128;   // weight rows per tile (MMA M, TMEM lanes)
constexpr int BK = 128;   // K per scale group
// K per pipeline stage: one scale group in two 64-wide (128-byte) swizzle
// atoms, so the MMA issuer's one barrier wait per stage covers 8 MMAs
constexpr int BKS = 128;
// Warps: 0 TMA producer, 1 MMA issuer, 2 .. 2+EXP-1 expanders, then 4 epilogue
// warps.  EXP = 4 (thread = weight row, whole stage) or 8 (thread = weight
// row, one 64-wide atom of the stage).
template <int EXP>
constexpr int threads_for() { return (2 + EXP + 4) * 32; }
constexpr int kAAtom = BN * 128;        // bytes of one 64-wide atom of the weight stage (16 KB)
constexpr int kAStage = 2 * kAAtom;     // 32 KB

// BMT tokens per tile (MMA N): 256 when there are enough tiles to fill the
// GPU, 128 for few token rows (more tiles, each MMA half as long).  TA: the
// weight operand lives in TMEM (128-token tiles only), so shared memory holds
// only the token stages, 4 deep.
template <int BMT, bool TA>
struct Smem {
  static_assert(!TA || BMT == 128, "TMEM weight operand: 128-token tiles");
  static constexpr int NS = TA ? 4 : BMT == 256 ? 2 : 3;  // stages (128 / 192 KB)
  static constexpr int kXAtom = BMT * 128;                // bytes of one 64-wide atom of the token stage
  static constexpr int kXStage = 2 * kXAtom;
  alignas(1024) unsigned char x[NS][kXStage];
  alignas(1024) unsigned char a[TA ? 1 : NS][TA ? 16 : kAStage];
  uint64_t full[NS], empty[NS];
  uint64_t full_c[2], empty_c[2];
  uint32_t tmem_base;
};
}  // namespace sg

// Activation prep, one CTA per token row t:
//   xs[t] = fp16( b (.) x[t] * 2^c_t ), 2^c_t putting max |b x| in [2^14, 2^15)
// (exact power-of-two scaling; fp16 keeps all 8 significant bits of a bf16
// product with a unit diagonal, and 11 of b x), cscale[t] = 2^-c_t.  With a
// middle diagonal `mid`, also d_t with max|mid| * ||b x||_1 * 2^d_t <= 2^15
// (dscale = 2^d, dinv = 2^-d) so that an fp16 intermediate cannot overflow.
// bdiag == nullptr means b = 1; mid == nullptr skips d.
__global__ void __launch_bounds__(256) sg_prep_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ bdiag,
                                                      const uint16_t* __restrict__ mid, int n, int r,
                                                      __half* __restrict__ xs, float* __restrict__ cscale,
                                                      float* __restrict__ dscale, float* __restrict__ dinv) {
  // 16-byte vectors (8 values); the row stays in registers between the
  // reductions and the conversion when n <= 8 * 256 * kMaxV, else it is re-read.
  constexpr int kMaxV = 4;
  pdl_wait();
  __shared__ float red[3][8];
  const int t = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * n);
  const uint4* br = reinterpret_cast<const uint4*>(bdiag);
  const int nv = n >> 3;
  auto values = [&](int i, const uint4& u, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[2 * q] = __uint_as_float(w[q] << 16);
      v[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
    if (bdiag) {
      const uint4 bb = __ldg(br + i);
      const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&bw[q]));
        v[2 * q] *= f.x;
        v[2 * q + 1] *= f.y;
      }
    }
  };
  uint4 keep[kMaxV];
  float mx = 0.f, l1 = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxV; ++j) {
    const int i = threadIdx.x + 256 * j;
    keep[j] = i < nv ? __ldg(xr + i) : make_uint4(0, 0, 0, 0);
    if (i < nv) {
      float v[8];
      values(i, keep[j], v);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        mx = fmaxf(mx, fabsf(v[q]));
        l1 += fabsf(v[q]);
      }
    }
  }
  for (int i = threadIdx.x + 256 * kMaxV; i < nv; i += 256) {
    float v[8];
    values(i, __ldg(xr + i), v);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      mx = fmaxf(mx, fabsf(v[q]));
      l1 += fabsf(v[q]);
    }
  }
  // max |mid| (the same for every row): 16-byte loads, independent partial
  // maxima, so the loads are in flight together (r % 8 == 0, 16-byte aligned)
  float mm = 0.f;
  if (mid) {
    const uint4* mv = reinterpret_cast<const uint4*>(mid);
    float m4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int j = threadIdx.x; j < (r >> 3); j += blockDim.x) {
      const uint4 u = __ldg(mv + j);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[q]));
        m4[q] = fmaxf(m4[q], fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    mm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, o);
    mm = fmaxf(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, o));
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = mx;
    red[1][threadIdx.x >> 5] = l1;
    red[2][threadIdx.x >> 5] = mm;
  }
  __syncthreads();
  mx = 0.f;
  l1 = 0.f;
  mm = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mx = fmaxf(mx, red[0][i]);
    l1 += red[1][i];
    mm = fmaxf(mm, red[2][i]);
  }
  // c: max |b x| 2^c in [2^14, 2^15);  d: mm * l1 * 2^d <= 2^15 (l1 rounded up)
  // (both at most 126: 2^c, 2^d and their inverses stay normal floats)
  int c = 0, d = 0;
  if (mx > 0.f) {
    int E;
    frexpf(mx, &E);  // mx < 2^E
    c = min(15 - E, 126);
  }
  if (mm > 0.f && l1 > 0.f) {
    int E;
    frexpf(mm * l1 * 1.0001f, &E);  // < 2^E
    d = min(15 - E, 126);
  }
  const float cs = ldexpf(1.f, c);
  uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<int64_t>(t) * n);
  auto convert = [&](int i, const uint4& u) {
    float v[8];
    values(i, u, v);
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __half2 h2 = __floats2half2_rn(v[2 * q] * cs, v[2 * q + 1] * cs);
      o[q] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  };
#pragma unroll
  for (int j = 0; j < kMaxV; ++j) {
    const int i = threadIdx.x + 256 * j;
    if (i < nv) convert(i, keep[j]);
  }
  for (int i = threadIdx.x + 256 * kMaxV; i < nv; i += 256) convert(i, __ldg(xr + i));
  if (threadIdx.x == 0) {
    cscale[t] = ldexpf(1.f, -c);
    if (dscale) dscale[t] = ldexpf(1.f, d);
    if (dinv) dinv[t] = ldexpf(1.f, -d);
  }
  pdl_launch_dependents();
}

// D[n][m] = sum_k A[n][k] xs[m][k],  A[n][k] = (1 - 2 bit[n][k]) * s[n][k/128]
// (s = 1 without group scales): an exact fp16 value, so every product is exact
// and all of K accumulates in one fp32 TMEM tile.
struct SgParams {
  const uint32_t* signs;   // [rows][K/32]
  const uint16_t* gscales; // [rows][K/128] fp16 group scales, or nullptr (+-1)
  const uint16_t* rdiag;   // [rows] fp16 row diagonal (mid, a), or nullptr (1)
  const float* s1;         // per token: 2^-c (phase 1) or 2^-d (phase 2)
  const float* s2;         // per token: 2^d (phase 1) or unused
  __half* out_h;           // phase 1 output [M][rows]
  float* out_f;            // phase 2 output [M][rows]
  int M, rows, K, MT, NT, NK;
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <bool PHASE1, int BM, int EXP, bool TA>
__global__ void __launch_bounds__(sg::threads_for<EXP>(), 1)
    sg_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const SgParams p) {
  using namespace sg;
  using S = Smem<BM, TA>;
  static_assert(EXP == 4 || EXP == 8, "expander warps");
  constexpr int kWpr = 16 / EXP;  // sign words per expander thread and stage
  constexpr int kXStage = S::kXStage, kXAtom = S::kXAtom, NS = S::NS;
  constexpr uint32_t kIdesc = idesc_f16(BN, BM, 0, 0);  // fp16 x fp16 -> fp32
  // TMEM: two accumulators of BM columns; with TA also NS weight stages of
  // BKS / 2 columns (row = lane, k pairs along the columns) from column 2 BM
  constexpr uint32_t kACol = 2 * BM;
  constexpr uint32_t kTmemCols = TA ? 512 : 2 * BM;
  static_assert(!TA || kACol + NS * (BKS / 2) <= kTmemCols, "TMEM columns");
  extern __shared__ unsigned char smem_raw[];
  S& sm = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      // one barrier per stage: the expanders' 32 EXP arrivals plus the producer's
      // arrival with the activation tile's transaction bytes (one wait for the MMA issuer)
      mbar_init(&sm.full[i], 32 * EXP + 1);
      mbar_init(&sm.empty[i], 1);
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
  if (warp == 0 && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_b) : "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();
  const int ntiles = p.MT * p.NT;
  const int NKS = p.NK * (BK / BKS);  // stages per tile (one per scale group)
  const int my_tiles = (ntiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                       static_cast<int>(gridDim.x);

  if (warp == 0) {
    if (lane == 0) {
      uint32_t c = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int mt = tile % p.MT;
        for (int ks = 0; ks < NKS; ++ks, ++c) {
          const int s = c % NS;
          if (!mbar_wait(&sm.empty[s], ((c / NS) & 1) ^ 1)) goto done_prod;
          mbar_arrive_expect_tx(&sm.full[s], kXStage);
          tma_load_2d(sm.x[s], &tmap_b, ks * BKS, mt * BM, &sm.full[s]);
          tma_load_2d(sm.x[s] + kXAtom, &tmap_b, ks * BKS + 64, mt * BM, &sm.full[s]);
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
        for (int ks = 0; ks < NKS; ++ks, ++c) {
          const int s = c % NS;
          if (!mbar_wait(&sm.full[s], (c / NS) & 1)) goto done_mma;
          tc_fence_after();
          const uint32_t xbase = smem_u32(sm.x[s]);
#pragma unroll
          for (int kk = 0; kk < BKS / 16; ++kk) {
            const uint32_t xo = (kk >> 2) * kXAtom + (kk & 3) * 32;
            if constexpr (TA) {
              tc_mma_ts(d, tmem + kACol + s * (BKS / 2) + kk * 8, smem_desc_sw128(xbase + xo), kIdesc,
                        (ks > 0 || kk > 0) ? 1u : 0u);
            } else {
              const uint32_t ao = (kk >> 2) * kAAtom + (kk & 3) * 32;
              tc_mma_ss(d, smem_desc_sw128(smem_u32(sm.a[s]) + ao), smem_desc_sw128(xbase + xo), kIdesc,
                        (ks > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(&sm.empty[s]);
        }
        tc_commit(&sm.full_c[cb]);
      }
    done_mma:;
    }
  } else if (warp < 2 + EXP) {
    // expanders: thread = weight row = TMEM lane (and, with 8 expander warps,
    // one of the stage's two 64-wide halves).  Per stage: 4 sign words (one
    // scale group, 128 k) + the group scale -> 64 fp16 pairs +-s (s = the
    // group scale, or 0x3C00 = 1.0; the sign bit comes straight from the
    // word), stored as 16-byte chunks of the row in the two 128B-swizzled
    // K-major atoms, or (TA) as 16 TMEM columns per word in the row's lane.
    // Words and scales stream through a kPf-deep register ring over this
    // CTA's (tile, stage) sequence so L2 latency hides behind kPf stages.  8
    // deep measured slower on the 4096^3 DBF chain at 512 rows: 0.114 vs
    // 0.075 ms with 4 expander warps; with 8, 0.095 ms where 4 expander
    // warps at depth 4 took 0.083 on the same GPU.
    constexpr int kPf = 4;
    const int rl = (warp & 3) * 32 + lane;  // a warp reaches TMEM lanes 32 (warp % 4) ..
    const int half = EXP == 8 ? (warp - 2) >> 2 : 0;  // the atom this thread writes (8 expander warps)
    const int64_t wrow = p.K >> 5;
    int ld_tile = blockIdx.x, ld_ks = 0;
    auto fetch = [&](uint4& w, uint32_t& sc) {
      w = make_uint4(0, 0, 0, 0);
      sc = 0x3C00u;
      if (ld_tile < ntiles) {
        const int n = (ld_tile / p.MT) * BN + rl;
        if (n < p.rows) {  // a row's words are 16-byte aligned (K % 128 == 0)
          if (EXP == 4) {
            w = __ldg(reinterpret_cast<const uint4*>(p.signs + static_cast<int64_t>(n) * wrow) + ld_ks);
          } else {
            const uint2 h2 =
                __ldg(reinterpret_cast<const uint2*>(p.signs + static_cast<int64_t>(n) * wrow) + 2 * ld_ks + half);
            w.x = h2.x;
            w.y = h2.y;
          }
          if (p.gscales) sc = __ldg(p.gscales + static_cast<int64_t>(n) * p.NK + ld_ks);
        }
        if (++ld_ks == NKS) {
          ld_ks = 0;
          ld_tile += gridDim.x;
        }
      }
    };
    uint4 wr[kPf];
    uint32_t sr[kPf];
#pragma unroll
    for (int j = 0; j < kPf; ++j) fetch(wr[j], sr[j]);
    const int my_stages = my_tiles * NKS;
    const uint32_t row_off = static_cast<uint32_t>(rl) * 128u;
    const uint32_t sw = static_cast<uint32_t>(rl & 7);
    uint32_t c = 0;
    for (int c0 = 0; c0 < my_stages; c0 += kPf) {
#pragma unroll
      for (int j = 0; j < kPf; ++j) {
        if (c0 + j >= my_stages) break;
        const uint4 cur = wr[j];
        const uint32_t ss = sr[j] * 0x00010001u;  // the scale in both fp16 halves
        fetch(wr[j], sr[j]);
        const int s = c % NS;
        if (!mbar_wait_warp(&sm.empty[s], ((c / NS) & 1) ^ 1)) goto done_exp;
        if constexpr (TA) tc_fence_after();  // the stage's MMAs (commit) before its TMEM is rewritten
        const uint32_t abase = TA ? tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kACol + s * (BKS / 2) +
                                        static_cast<uint32_t>(half * (BKS / 4))
                                  : smem_u32(sm.a[s]) + row_off + static_cast<uint32_t>(half * kAAtom);
        const uint32_t words[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
        for (int wi = 0; wi < kWpr; ++wi) {
          const uint32_t w = words[wi];
          uint32_t rr[16];
#pragma unroll
          for (int pp = 0; pp < 16; ++pp) {
            const uint32_t src = (pp < 8) ? w : (w >> 16);
            const int b = 2 * (pp & 7);
            const uint32_t m = src & (3u << b);
            const uint32_t tt = m * (0x40008000u >> b);
            rr[pp] = (tt & 0x80008000u) | ss;
          }
          if constexpr (TA) {
            tmem_st16(abase + wi * 16, rr);  // columns: k pairs 16 wi .. 16 wi + 15 of this part
          } else {
            const uint32_t ab = abase + static_cast<uint32_t>((wi >> 1) * kAAtom);  // atom wi / 2
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t chunk = static_cast<uint32_t>((wi & 1) * 4 + q);
              st_shared_v4(ab + ((chunk ^ sw) << 4), rr[4 * q], rr[4 * q + 1], rr[4 * q + 2], rr[4 * q + 3]);
            }
          }
        }
        if constexpr (TA) {
          tc_wait_st();
          tc_fence_before();
        } else {
          fence_async_shared();
        }
        mbar_arrive(&sm.full[s]);
        ++c;
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
      const float rd = valid ? (p.rdiag ? __half2float(__ushort_as_half(p.rdiag[n])) : 1.0f) : 0.f;
      const int cb = tl & 1;
      if (!mbar_wait_warp(&sm.full_c[cb], (tl >> 1) & 1)) goto done_epi;
      tc_fence_after();
      const int mrem = min(BM, p.M - mt * BM);
#pragma unroll 1
      for (int q4 = 0; q4 < BM / 32; ++q4) {
        if (q4 * 32 >= mrem) break;
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
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ host side

template <bool PHASE1, int BM, int EXP, bool TA>
static cudaError_t launch_sg_gemm_bm(SgParams p, const void* bmat, int64_t bcols, cudaStream_t stream, int num_sms) {
  using namespace sg;
  p.MT = (p.M + BM - 1) / BM;
  p.NT = (p.rows + BN - 1) / BN;
  p.NK = p.K / BK;
  CUtensorMap tm;
  // fp16 and bf16 share the 2-byte element layout the tensor map describes; box {64, BM}
  if (!make_tmap_bf16_sw128(&tm, bmat, p.M, bcols, BM)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem<BM, TA>) + 1024;
  auto kern = sg_gemm_kernel<PHASE1, BM, EXP, TA>;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int ntiles = p.MT * p.NT;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ntiles < num_sms ? ntiles : num_sms));
  cfg.blockDim = dim3(threads_for<EXP>());
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tm, p);
}

// p: signs, gscales, rdiag, s1, s2, outputs, M, rows, K (tiles are derived here).
// Token tile: 256 when that gives at least one tile per SM, else 128.
// Expander warps: kExp256 / kExp128 by token tile (the expansion of a stage
// costs the same whatever the tile; a 128-token tile's MMAs take half as
// long).  Weight operand of 128-token tiles: kTmemA128 (TMEM or shared memory).
template <bool PHASE1>
cudaError_t launch_sg_gemm(const SgParams& p, const void* bmat, int64_t bcols, cudaStream_t stream, int num_sms) {
  const int nt = (p.rows + sg::BN - 1) / sg::BN;
  const int tiles256 = ((p.M + 255) / 256) * nt;
  const int force = knob(kKnobSgBm);  // tuning knobs: token tile, expander warps, weight operand
  const int fexp = knob(kKnobSgExp);
  const int fa = knob(kKnobSgA);
  if (force == 256 || (force != 128 && tiles256 >= num_sms)) {
    if (fexp == 8 || (fexp != 4 && sg::kExp256 == 8))
      return launch_sg_gemm_bm<PHASE1, 256, 8, false>(p, bmat, bcols, stream, num_sms);
    return launch_sg_gemm_bm<PHASE1, 256, 4, false>(p, bmat, bcols, stream, num_sms);
  }
  const bool ta = fa == 2 || (fa != 1 && sg::kTmemA128);
  const bool e8 = fexp == 8 || (fexp != 4 && sg::kExp128 == 8);
  if (ta) {
    return e8 ? launch_sg_gemm_bm<PHASE1, 128, 8, true>(p, bmat, bcols, stream, num_sms)
              : launch_sg_gemm_bm<PHASE1, 128, 4, true>(p, bmat, bcols, stream, num_sms);
  }
  return e8 ? launch_sg_gemm_bm<PHASE1, 128, 8, false>(p, bmat, bcols, stream, num_sms)
            : launch_sg_gemm_bm<PHASE1, 128, 4, false>(p, bmat, bcols, stream, num_sms);
}

cudaError_t launch_sg_prep(const uint16_t* x, const uint16_t* bdiag, const uint16_t* mid, int64_t n, int64_t r,
                          int64_t B, __half* xs, float* cscale, float* dscale, float* dinv, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(B));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sg_prep_kernel, x, bdiag, mid, static_cast<int>(n), static_cast<int>(r), xs, cscale,
                            dscale, dinv);
}

}  // namespace w1

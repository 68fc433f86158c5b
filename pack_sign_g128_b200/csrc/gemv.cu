// w1_gemv: decode-regime 1-bit group-128 product, 1 <= B <= 8 vectors.
//
//   y[b,n] = sum_g s[n,g] * sum_{k in g} (1 - 2 bit[n,k]) x[b,k]
//
// Design (sm_100a):
//  * Sign expansion.  One PRMT per 4 weights turns sign bits into int8 bytes
//    {0, -1} (= -bit), using the selector bits of the packed word directly:
//    a table whose 8 entries are 0x00/0xFF keyed on bit 0, 1 or 2 of each
//    nibble extracts that bit of four nibbles at once (bit 3 uses w >> 3).
//    Then sum (1-2b) x = X + 2 * sum(-b) x with X = sum x.
//  * Activations as exact fixed point.  Per (batch row, 128-group) x is scaled
//    by 2^(22-E) (E from the group max), rounded to a 23-bit integer and split
//    into three signed int8 digits (planes).  Products run on mma.sync
//    m16n8k32 s8 tensor cores with exact s32 accumulation per group; the three
//    digit sums are recombined in int32, converted once, and scaled by
//    s[n,g] * 2^(E-22).  Error <= 2^(E-23) per element, far inside 1e-3 of
//    sum |s x|.
//  * K order inside one MMA is free: x digits are staged in shared memory in
//    exactly the order the bit extraction produces, so the canonical weight
//    layout is read unchanged (the DBF post, section 5 items 7-8: repack the
//    activation locally, keep the weight file canonical).
//  * Memory: a cluster of S CTAs splits K; each CTA streams its rows' K-slice
//    of sign words with 1-D bulk copies (all stages issued up front when they
//    fit), and the S partial results are reduced through distributed shared
//    memory in a fixed order (deterministic, no atomics, no workspace).
//  * Programmatic dependent launch: before waiting on the previous kernel the
//    CTA only prefetches its weight bytes into L2.
#include <cstdint>
#include <cuda_fp16.h>
#include <mutex>

#include "w1_common.cuh"

namespace w1 {

struct GemvParams {
  const uint32_t* signs;
  const uint16_t* scales;
  const uint16_t* x;
  float* y;
  int64_t N;        // total rows of the matrix (row stride of y)
  int64_t K;
  int64_t row_base; // first row handled by this launch
  int rows;         // rows handled by this launch
  int NG;           // K / 128
  int S;            // cluster size (K split)
  int ns;           // pipeline stages
  int max_tiles;    // max 16-row tiles per cluster
  int max_ng;       // max groups per CTA
};

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;

template <int NB>
struct GemvLayout {
  static constexpr int NT = (NB <= 4) ? 2 : 3;
};

__host__ __device__ inline int gemv_rowstride(int ng) {
  // bytes per row slice in a stage; an odd multiple of 16 keeps the 8 rows of
  // a warp's LDS.32 on distinct banks
  int rs = ng * 16;
  if ((ng & 1) == 0) rs += 16;
  return rs;
}

__host__ __device__ inline int round_up(int v, int a) { return (v + a - 1) / a * a; }

struct GemvSmem {
  int stages, xq, xsum, xf, sc, part, bars, total;
};

template <int NB>
__host__ __device__ inline GemvSmem gemv_smem_layout(int ns, int max_tiles, int max_ng) {
  constexpr int NT = GemvLayout<NB>::NT;
  GemvSmem L;
  int off = 0;
  L.stages = off;
  off += ns * 16 * gemv_rowstride(max_ng);
  off = round_up(off, 128);
  L.xq = off;
  off += max_ng * 4 * NT * 256;
  L.xsum = off;
  off += max_ng * NB * 4;
  L.xf = off;
  off += max_ng * NB * 4;
  off = round_up(off, 16);
  L.sc = off;
  off += max_tiles * 16 * max_ng * 2;
  off = round_up(off, 16);
  L.part = off;
  off += NB * max_tiles * 16 * 4;
  off = round_up(off, 8);
  L.bars = off;
  off += 2 * ns * 8;
  L.total = round_up(off, 128);
  return L;
}

// -(bit q + 4i of w) for i = 0..3, as int8 bytes; the shifted copies of w are
// precomputed (w3 = w >> 3, w16 = w >> 16, w19 = w >> 19).
__device__ __forceinline__ uint32_t extract_q(int q, uint32_t w, uint32_t w3, uint32_t w16,
                                              uint32_t w19) {
  switch (q) {
    case 0: return prmt(0xFF00FF00u, 0xFF00FF00u, w);
    case 1: return prmt(0xFFFF0000u, 0xFFFF0000u, w);
    case 2: return prmt(0x00000000u, 0xFFFFFFFFu, w);
    case 3: return prmt(0xFF00FF00u, 0xFF00FF00u, w3);
    case 4: return prmt(0xFF00FF00u, 0xFF00FF00u, w16);
    case 5: return prmt(0xFFFF0000u, 0xFFFF0000u, w16);
    case 6: return prmt(0x00000000u, 0xFFFFFFFFu, w16);
    default: return prmt(0xFF00FF00u, 0xFF00FF00u, w19);
  }
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

template <int NB>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
  constexpr int NT = GemvLayout<NB>::NT;
  extern __shared__ __align__(128) unsigned char smem[];
  const GemvSmem L = gemv_smem_layout<NB>(p.ns, p.max_tiles, p.max_ng);
  unsigned char* stages = smem + L.stages;
  unsigned char* xq = smem + L.xq;
  int* xsum = reinterpret_cast<int*>(smem + L.xsum);
  float* xf = reinterpret_cast<float*>(smem + L.xf);
  uint16_t* sc = reinterpret_cast<uint16_t*>(smem + L.sc);
  float* part = reinterpret_cast<float*>(smem + L.part);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + p.ns;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = p.S;
  const int crank = static_cast<int>(cluster_ctarank());
  const int q = static_cast<int>(cluster_id_x());
  const int Q = static_cast<int>(nclusters_x());

  // ---- work split: cluster -> 16-row tiles, CTA -> K groups
  const int T16 = (p.rows + 15) >> 4;
  const int tq0 = static_cast<int>((static_cast<int64_t>(q) * T16) / Q);
  const int tq1 = static_cast<int>((static_cast<int64_t>(q + 1) * T16) / Q);
  const int ntiles = tq1 - tq0;
  const int g0 = (crank * p.NG) / S;
  const int g1 = ((crank + 1) * p.NG) / S;
  const int ng = g1 - g0;
  const int rowstride = gemv_rowstride(ng);
  const int stage_bytes = 16 * rowstride;
  const int64_t wrow = p.K >> 5;            // words per weight row
  const int64_t r_first = p.row_base + static_cast<int64_t>(tq0) * 16;
  const int rows_c = min(ntiles * 16, static_cast<int>(p.row_base + p.rows - r_first));

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbarrier_init();
  }
  // L2 prefetch of this CTA's weight bytes (safe before the dependency wait:
  // a prefetch returns no data to the kernel)
  if (warp == kConsumerWarps) {
    for (int r = lane; r < rows_c; r += 32) {
      const int64_t row = r_first + r;
      bulk_prefetch_l2(p.signs + row * wrow + 4 * g0, static_cast<uint32_t>(ng * 16));
      prefetch_l2(p.scales + row * p.NG + g0);
    }
  }
  __syncthreads();
  pdl_wait();

  // ---- producer: issue the first stages immediately
  auto issue_tile = [&](int it) {
    const int s = it % p.ns;
    const int64_t row0 = r_first + static_cast<int64_t>(it) * 16;
    const int64_t nr64 = p.row_base + p.rows - row0;
    const int nr = nr64 < 16 ? static_cast<int>(nr64) : 16;
    if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nr * ng * 16));
    __syncwarp();
    if (lane < nr) {
      bulk_g2s(stages + s * stage_bytes + lane * rowstride, p.signs + (row0 + lane) * wrow + 4 * g0,
               static_cast<uint32_t>(ng * 16), &full[s]);
    }
  };
  const int first = min(ntiles, p.ns);
  if (warp == kConsumerWarps) {
    for (int it = 0; it < first; ++it) issue_tile(it);
  }

  // ---- x preparation (all warps): zero the digit planes, then quantise
  {
    uint4* z = reinterpret_cast<uint4*>(xq);
    const int n16 = ng * 4 * NT * 256 / 16;
    for (int i = threadIdx.x; i < n16; i += kGemvThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  {
    const int sub = lane & 7;       // 8 lanes per (b, group) item
    const int t = sub >> 1;         // word within group
    const int hh = sub & 1;         // half word (bits 16*hh .. 16*hh+15)
    const int items = NB * ng;
    for (int base = warp * 4; base < items; base += (kConsumerWarps + 1) * 4) {
      const int item = base + (lane >> 3);
      const bool valid = item < items;
      const int b = valid ? item / ng : 0;
      const int gl = valid ? item - b * ng : 0;
      float v[16];
      if (valid) {
        const uint16_t* xp = p.x + static_cast<int64_t>(b) * p.K + 128 * (g0 + gl) + 32 * t + 16 * hh;
        const uint4 u0 = *reinterpret_cast<const uint4*>(xp);
        const uint4 u1 = *reinterpret_cast<const uint4*>(xp + 8);
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
          v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(v[i]));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
      int E = 0;
      if (mx > 0.f) frexpf(mx, &E);  // mx = f * 2^E, f in [0.5, 1)
      const int sf = 22 - E;
      const int sf1 = sf / 2, sf2 = sf - sf1;
      const float m1 = __uint_as_float(static_cast<uint32_t>(sf1 + 127) << 23);
      const float m2 = __uint_as_float(static_cast<uint32_t>(sf2 + 127) << 23);
      uint32_t e[16];
      uint32_t bsum = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // x * 2^sf rounded to an integer via the 1.5*2^23 magic constant:
        // bits = 0x4B400000 + round(x * 2^sf) exactly for |x 2^sf| < 2^22
        const uint32_t bits = __float_as_uint(fmaf(v[i] * m1, m2, 12582912.0f));
        bsum += bits;
        e[i] = (bits - 0x4ABF7F80u) ^ 0x00808080u;  // three signed digit bytes
      }
      int xs = static_cast<int>(bsum - 16u * 0x4B400000u);
      xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 1);
      xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 2);
      xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 4);
      if (valid) {
        if (sub == 0) {
          xsum[gl * NB + b] = xs;
          xf[gl * NB + b] = ldexpf(1.0f, E - 22);
        }
        // columns of the three planes of batch row b
        const int jt_hi = (b < 4) ? 0 : 2;
        const int c_hi = 2 * (b & 3);
        const int c_lo = (b < 4) ? 2 * b : 2 * (b - 4) + 1;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          // elements r, r+4, r+8, r+12 of this lane share q = r + 4*hh
          const uint32_t e0 = e[r], e1 = e[r + 4], e2 = e[r + 8], e3 = e[r + 12];
          const uint32_t p01 = prmt(e0, e1, 0x5140u), p23 = prmt(e2, e3, 0x5140u);
          const uint32_t d0 = prmt(p01, p23, 0x5410u);
          const uint32_t d1 = prmt(p01, p23, 0x7632u);
          const uint32_t d2 = prmt(prmt(e0, e1, 0x0062u), prmt(e2, e3, 0x0062u), 0x5410u);
          const int qq = r + 4 * hh;
          const int m = qq >> 1, h = qq & 1;
          unsigned char* slot = xq + ((gl * 4 + m) * NT) * 256 + t * 8 + h * 4;
          *reinterpret_cast<uint32_t*>(slot + jt_hi * 256 + c_hi * 32) = d2;
          *reinterpret_cast<uint32_t*>(slot + jt_hi * 256 + (c_hi + 1) * 32) = d1;
          *reinterpret_cast<uint32_t*>(slot + 1 * 256 + c_lo * 32) = d0;
        }
      }
    }
  }
  // ---- scales of this CTA's rows and groups -> shared memory
  for (int i = threadIdx.x; i < rows_c * ng; i += kGemvThreads) {
    const int r = i / ng, gl = i - r * ng;
    sc[r * ng + gl] = p.scales[(r_first + r) * p.NG + g0 + gl];
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---- producer: remaining tiles as stages free up
    for (int it = first; it < ntiles; ++it) {
      const int s = it % p.ns;
      if (!mbar_wait_warp(&empty[s], ((it / p.ns) - 1) & 1)) break;
      issue_tile(it);
    }
  } else {
    // ---- consumers
    const int g = lane >> 2, t = lane & 3;
    for (int it = warp; it < ntiles; it += kConsumerWarps) {
      const int s = it % p.ns;
      if (!mbar_wait_warp(&full[s], (it / p.ns) & 1)) break;
      const unsigned char* st = stages + s * stage_bytes;
      const int rl0 = it * 16;  // local row of the tile within this cluster
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      for (int gl = 0; gl < ng; ++gl) {
        const uint32_t wA = *reinterpret_cast<const uint32_t*>(st + g * rowstride + (4 * gl + t) * 4);
        const uint32_t wB =
            *reinterpret_cast<const uint32_t*>(st + (g + 8) * rowstride + (4 * gl + t) * 4);
        const uint32_t wA3 = wA >> 3, wA16 = wA >> 16, wA19 = wA >> 19;
        const uint32_t wB3 = wB >> 3, wB16 = wB >> 16, wB19 = wB >> 19;
        int C[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) C[j][0] = C[j][1] = C[j][2] = C[j][3] = 0;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          uint32_t a[4];
          a[0] = extract_q(2 * m, wA, wA3, wA16, wA19);
          a[1] = extract_q(2 * m, wB, wB3, wB16, wB19);
          a[2] = extract_q(2 * m + 1, wA, wA3, wA16, wA19);
          a[3] = extract_q(2 * m + 1, wB, wB3, wB16, wB19);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const uint2 bb = *reinterpret_cast<const uint2*>(xq + ((gl * 4 + m) * NT + j) * 256 +
                                                            g * 32 + t * 8);
            mma_s8_16832(C[j], a, bb.x, bb.y, C[j]);
          }
        }
        const int rA = rl0 + g, rB = rl0 + g + 8;
        const float sA = (rA < rows_c) ? __half2float(__ushort_as_half(sc[rA * ng + gl])) : 0.f;
        const float sB = (rB < rows_c) ? __half2float(__ushort_as_half(sc[rB * ng + gl])) : 0.f;
#pragma unroll
        for (int be = 0; be < 2; ++be) {
          const int b = t + 4 * be;
          if (b < NB) {
            const int jh = be ? 2 : 0;
            const int X = xsum[gl * NB + b];
            const float f = xf[gl * NB + b];
            const int VA = X + 131072 * C[jh][0] + 512 * C[jh][1] + 2 * C[1][be ? 1 : 0];
            const int VB = X + 131072 * C[jh][2] + 512 * C[jh][3] + 2 * C[1][be ? 3 : 2];
            acc[0][be] = fmaf(sA * f, static_cast<float>(VA), acc[0][be]);
            acc[1][be] = fmaf(sB * f, static_cast<float>(VB), acc[1][be]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      const int rA = rl0 + g, rB = rl0 + g + 8;
#pragma unroll
      for (int be = 0; be < 2; ++be) {
        const int b = t + 4 * be;
        if (b < NB) {
          if (rA < rows_c) part[b * (p.max_tiles * 16) + rA] = acc[0][be];
          if (rB < rows_c) part[b * (p.max_tiles * 16) + rB] = acc[1][be];
        }
      }
    }
  }
  pdl_launch_dependents();
  // ---- cluster reduction of the S partial sums, fixed order
  cluster_sync();
  {
    const int r_lo = (crank * rows_c) / S;
    const int r_hi = ((crank + 1) * rows_c) / S;
    const int span = r_hi - r_lo;
    const uint32_t part_base = smem_u32(part);
    for (int i = threadIdx.x; i < span * NB; i += kGemvThreads) {
      const int b = i / span, r = r_lo + (i - b * span);
      const uint32_t off = static_cast<uint32_t>((b * (p.max_tiles * 16) + r) * 4);
      float sum = 0.f;
      for (int c = 0; c < S; ++c) sum += ld_dsmem_f32(map_shared_rank(part_base + off, c));
      p.y[static_cast<int64_t>(b) * p.N + r_first + r] = sum;
    }
  }
  cluster_sync();
}

// ------------------------------------------------------------------ host side

template <int NB>
static cudaError_t launch_gemv_nb(const GemvParams& base, int Q, int S, cudaStream_t stream,
                                  int smem_cap) {
  GemvParams p = base;
  p.S = S;
  const int T16 = (p.rows + 15) / 16;
  p.max_tiles = (T16 + Q - 1) / Q;
  p.max_ng = (p.NG + S - 1) / S;
  const int stage_bytes = 16 * gemv_rowstride(p.max_ng);
  // stage count: every tile if it fits, else what the budget allows
  const GemvSmem L0 = gemv_smem_layout<NB>(0, p.max_tiles, p.max_ng);
  int ns = p.max_tiles;
  const int budget = smem_cap - L0.total - 256;
  if (ns * (stage_bytes + 16) > budget) ns = budget / (stage_bytes + 16);
  if (ns < 1) return cudaErrorInvalidConfiguration;
  p.ns = ns;
  const GemvSmem L = gemv_smem_layout<NB>(ns, p.max_tiles, p.max_ng);
  cudaError_t err = cudaFuncSetAttribute(gemv_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L.total);
  if (err != cudaSuccess) return err;
  if (S > 8) {
    err = cudaFuncSetAttribute(gemv_kernel<NB>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(Q * S));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(L.total);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NB>, p);
}

// Largest number of co-resident clusters of size S for this kernel/smem.
template <int NB>
static int gemv_max_clusters(int S, int smem_bytes) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(S * 64));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(gemv_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, gemv_kernel<NB>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Choose the K split S (cluster size) and the number of clusters Q so that
// every cluster is co-resident (one wave) and the per-CTA work is smallest.
template <int NB>
static void gemv_plan(int64_t rows, int NG, int num_sms, int smem_cap, int* Q_out, int* S_out) {
  const int T16 = static_cast<int>((rows + 15) / 16);
  double best = 1e300;
  int bq = 1, bs = 1;
  for (int S = 1; S <= 8; S *= 2) {
    if (S > NG) break;
    int Q = num_sms / S;
    const int occ = gemv_max_clusters<NB>(S, smem_cap);
    if (occ > 0 && occ < Q) Q = occ;
    if (Q > T16) Q = T16;
    if (Q < 1) Q = 1;
    const double tiles = static_cast<double>((T16 + Q - 1) / Q);
    const double groups = static_cast<double>((NG + S - 1) / S);
    // weights: ~0.6 issue slots per weight; x prep: ~9 per element per cluster
    const double cost = tiles * groups * 2048.0 * (0.55 + 0.05 * NB) + NB * groups * 128.0 * 9.0 +
                        (S > 1 ? 1500.0 : 0.0);
    if (cost < best * 0.98) {
      best = cost;
      bq = Q;
      bs = S;
    }
  }
  *Q_out = bq;
  *S_out = bs;
}

struct GemvPlanEntry {
  int64_t rows;
  int NG, NB, sms, cap, dev, Q, S;
};
static GemvPlanEntry g_plan_cache[64];
static int g_plan_count = 0;
static std::mutex g_plan_mu;

static bool gemv_plan_cached(int64_t rows, int NG, int NB, int sms, int cap, int* Q, int* S) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_plan_mu);
  for (int i = 0; i < g_plan_count; ++i) {
    const GemvPlanEntry& e = g_plan_cache[i];
    if (e.rows == rows && e.NG == NG && e.NB == NB && e.sms == sms && e.cap == cap && e.dev == dev) {
      *Q = e.Q;
      *S = e.S;
      return true;
    }
  }
  return false;
}
static void gemv_plan_store(int64_t rows, int NG, int NB, int sms, int cap, int Q, int S) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_plan_mu);
  const int i = g_plan_count < 64 ? g_plan_count++ : static_cast<int>((rows + NG) & 63);
  g_plan_cache[i] = GemvPlanEntry{rows, NG, NB, sms, cap, dev, Q, S};
}

cudaError_t launch_gemv(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                        const uint16_t* x, int B, float* y, cudaStream_t stream, int num_sms,
                        int smem_cap) {
  const int NG = static_cast<int>(K / 128);
  // rows per launch bounded so that per-CTA scale / partial buffers fit
  const int64_t max_rows = 32768;
  for (int64_t r0 = 0; r0 < N; r0 += max_rows) {
    const int rows = static_cast<int>((N - r0) < max_rows ? (N - r0) : max_rows);
    int Q = 1, S = 1;
    if (!gemv_plan_cached(rows, NG, B, num_sms, smem_cap, &Q, &S)) {
    switch (B) {
      case 1: gemv_plan<1>(rows, NG, num_sms, smem_cap, &Q, &S); break;
      case 2: gemv_plan<2>(rows, NG, num_sms, smem_cap, &Q, &S); break;
      case 3: gemv_plan<3>(rows, NG, num_sms, smem_cap, &Q, &S); break;
      case 4: gemv_plan<4>(rows, NG, num_sms, smem_cap, &Q, &S); break;
      case 5: gemv_plan<5>(rows, NG, num_sms, smem_cap, &Q, &S); break;
      case 6: gemv_plan<6>(rows, NG, num_sms, smem_cap, &Q, &S); break;
      case 7: gemv_plan<7>(rows, NG, num_sms, smem_cap, &Q, &S); break;
      default: gemv_plan<8>(rows, NG, num_sms, smem_cap, &Q, &S); break;
    }
    gemv_plan_store(rows, NG, B, num_sms, smem_cap, Q, S);
    }
    GemvParams p = {};
    p.signs = signs;
    p.scales = scales;
    p.x = x;
    p.y = y;
    p.N = N;
    p.K = K;
    p.row_base = r0;
    p.rows = rows;
    p.NG = NG;
    cudaError_t err;
    switch (B) {
      case 1: err = launch_gemv_nb<1>(p, Q, S, stream, smem_cap); break;
      case 2: err = launch_gemv_nb<2>(p, Q, S, stream, smem_cap); break;
      case 3: err = launch_gemv_nb<3>(p, Q, S, stream, smem_cap); break;
      case 4: err = launch_gemv_nb<4>(p, Q, S, stream, smem_cap); break;
      case 5: err = launch_gemv_nb<5>(p, Q, S, stream, smem_cap); break;
      case 6: err = launch_gemv_nb<6>(p, Q, S, stream, smem_cap); break;
      case 7: err = launch_gemv_nb<7>(p, Q, S, stream, smem_cap); break;
      default: err = launch_gemv_nb<8>(p, Q, S, stream, smem_cap); break;
    }
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace w1

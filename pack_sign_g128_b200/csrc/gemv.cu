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
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "gemv_core.cuh"

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

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// 16 consecutive bf16 activations as fp32.
__device__ __forceinline__ void load16_bf16(const uint16_t* p, float (&v)[16]) {
  const uint4 u0 = *reinterpret_cast<const uint4*>(p);
  const uint4 u1 = *reinterpret_cast<const uint4*>(p + 8);
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
    v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
  }
}

template <int NB>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GemvSmem L = gemv_smem_layout<NB>(p.ns, p.max_tiles, p.max_ng);
  GemvSmemView v;
  v.stages = smem + L.stages;
  v.ns = p.ns;
  v.full = reinterpret_cast<uint64_t*>(smem + L.bars);
  v.empty = v.full + p.ns;
  GemvXView xv;
  xv.xq = smem + L.xq;
  xv.xsum = reinterpret_cast<int*>(smem + L.xsum);
  xv.xf = reinterpret_cast<float*>(smem + L.xf);
  xv.sc = reinterpret_cast<uint16_t*>(smem + L.sc);
  xv.part = reinterpret_cast<float*>(smem + L.part);
  xv.part_stride = p.max_tiles * 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int crank = static_cast<int>(cluster_ctarank());
  const Split sp = make_split(p.rows, p.row_base, p.NG, p.S, crank, static_cast<int>(cluster_id_x()),
                              static_cast<int>(nclusters_x()));
  const int64_t wrow = p.K >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ns; ++s) {
      mbar_init(&v.full[s], 1);
      mbar_init(&v.empty[s], 1);
    }
    fence_mbarrier_init();
  }
  if (warp == kProducerWarp) prefetch_weights(sp, p.signs, wrow, p.scales, p.NG, lane);
  __syncthreads();
  pdl_wait();
  // the next kernel in the stream may start now: its CTAs only prefetch their
  // own weights into L2 until this grid has completed
  pdl_launch_dependents();

  int first = 0;
  if (warp == kProducerWarp) first = issue_first_tiles(v, sp, p.signs, wrow, lane);

  // activations -> digit planes; scales of this CTA's rows and groups -> smem
  const uint16_t* xb = p.x;
  const int64_t K = p.K;
  quantise_input<NB>(xv, sp,
                     [&](int b, int k, float (&vv)[16]) { load16_bf16(xb + static_cast<int64_t>(b) * K + k, vv); },
                     kGemvThreads);
  stage_scales(xv, sp, p.scales, p.NG, kGemvThreads);
  __syncthreads();

  if (warp == kProducerWarp)
    produce_rest(v, sp, p.signs, wrow, first, lane);
  else
    consume_tiles<NB, true>(v, xv, sp, warp, lane);
  cluster_sync();
  float* y = p.y;
  const int64_t N = p.N;
  cluster_reduce<NB>(xv, sp, p.S, crank, [&](int b, int64_t row, float val) { y[b * N + row] = val; },
                     kGemvThreads);
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
    if (const char* f = getenv("W1_GEMV_SPLIT")) {  // tuning knob: force the K split
      const int fs = atoi(f);
      if (fs == 1 || fs == 2 || fs == 4 || fs == 8) {
        if (fs != S) Q = (num_sms / fs < (rows + 15) / 16) ? num_sms / fs : static_cast<int>((rows + 15) / 16);
        S = fs;
      }
    }
    if (getenv("W1_VERBOSE")) fprintf(stderr, "w1_gemv plan: rows=%d K=%lld B=%d -> clusters=%d split=%d\n", rows,
                                      static_cast<long long>(K), B, Q, S);
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

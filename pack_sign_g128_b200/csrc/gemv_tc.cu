// w1_gemv on tcgen05 tensor cores (kind::i8).
//
//   y[b,n] = sum_g s[n,g] * sum_{k in g} (1 - 2 bit[n,k]) x[b,k]
//
// One thread owns one weight row (one TMEM lane) and, per round, one 128-wide
// K group of it:
//  * Signs -> int8.  One PRMT per 4 weights turns the bits of a sign word into
//    bytes {0, -1} (a byte table of 0x00/0xFF keyed on bit 0, 1 or 2 of each
//    selector nibble; bit 3 via w >> 3, the upper half via w >> 16).  The 32
//    words of bytes of a group are written straight into TMEM (tcgen05.st):
//    the expanded weights never touch shared memory.
//  * Activations -> exact fixed point.  Per (batch row, group) x is scaled by
//    2^(22-E) (E from the group max), rounded to a 23-bit integer and split
//    into three signed int8 digits; the digits sit in shared memory as the MMA
//    B operand (3 columns per batch row, 128B swizzle).  Error <= 2^(E-23)
//    per element, ~32x inside the 1e-3 bound.
//  * One control thread issues 4 MMAs (K = 32) per group into that group's own
//    s32 accumulator slot; the owning thread reads the slot back and forms
//    sum (1-2b) x = X + 2 (65536 D_hi + 256 D_mid + D_lo), then s * 2^(E-22).
//  * A and accumulator slots are double-buffered so the expansion of round
//    r + 1 overlaps the MMAs of round r.  K is split over the four warps that
//    share a TMEM lane quarter and, for large B x K, over a cluster of CTAs;
//    partial sums are reduced in a fixed order through (distributed) shared
//    memory: deterministic, no atomics, no workspace.
//  * Sign words and scales are loaded with plain 16-byte loads issued right
//    after the dependency wait, all of them at once.
// The K order inside each MMA is free; the x digits are placed in exactly the
// order the bit extraction produces, so the canonical weight bytes are read
// unchanged.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cuda_fp16.h>
#include <mutex>

#include "w1_common.cuh"

namespace w1 {

namespace gtc {
constexpr int kWorkerWarps = 16;
constexpr int kThreads = (kWorkerWarps + 1) * 32;
constexpr int kCtl = kWorkerWarps;   // control warp
constexpr int kMaxGroups = 32;       // K groups per CTA (per thread: 8)
constexpr int kMaxRounds = kMaxGroups / 4;

template <int NB>
struct Cfg {
  static constexpr int N = (3 * NB <= 8) ? 8 : (3 * NB <= 16) ? 16 : 32;  // MMA N (digit columns)
  static constexpr int TILE = N * 128;                                   // B tile bytes per group
  static constexpr uint32_t IDESC = idesc_i8(128, N);
  // TMEM: A slots [buf][slot] 32 columns each at 0..255, D slots N columns from 256
  static constexpr uint32_t DCOL0 = 256;
  static constexpr uint32_t COLS = (256 + 2 * 4 * N) <= 256 ? 256 : 512;
};
}  // namespace gtc

struct GemvTcParams {
  const uint32_t* signs;
  const uint16_t* scales;
  const uint16_t* x;
  float* y;
  int N, K, NG;
  int S;       // cluster size (K split)
  int max_ng;  // max groups per CTA
  int early;   // read weights before the grid dependency wait
};

template <int NB>
struct GemvTcSmem {
  int xb, xsum, xf, part, inbox, bars, total;
};

template <int NB>
__host__ __device__ inline GemvTcSmem<NB> gemv_tc_layout(int max_ng) {
  using C = gtc::Cfg<NB>;
  GemvTcSmem<NB> L;
  int off = 0;
  L.xb = off;
  off += max_ng * C::TILE;
  L.xsum = off;
  off += max_ng * NB * 4;
  L.xf = off;
  off += max_ng * NB * 4;
  off = (off + 15) / 16 * 16;
  L.part = off;
  off += 4 * NB * 128 * 4;
  L.inbox = off;  // cluster reduction: [S][NB][ceil(rows / S)] floats, S x ceil(128 / S) <= 136
  off += NB * 136 * 4;
  off = (off + 7) / 8 * 8;
  L.bars = off;
  off += 4 * 8 + 16;
  L.total = (off + 127) / 128 * 128 + 1024;  // + slack for the 1024-aligned base
  // The kernel takes all 512 TMEM columns: ask for enough shared memory that
  // no second CTA of it can be resident on the same SM.
  if (L.total < 120 * 1024) L.total = 120 * 1024;
  return L;
}

// -(bit q + 4i of w), i = 0..3, as int8 bytes.
__device__ __forceinline__ uint32_t tc_extract(int q, uint32_t w) {
  switch (q) {
    case 0: return prmt(0xFF00FF00u, 0xFF00FF00u, w);
    case 1: return prmt(0xFFFF0000u, 0xFFFF0000u, w);
    case 2: return prmt(0x00000000u, 0xFFFFFFFFu, w);
    case 3: return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 3);
    case 4: return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 16);
    case 5: return prmt(0xFFFF0000u, 0xFFFF0000u, w >> 16);
    case 6: return prmt(0x00000000u, 0xFFFFFFFFu, w >> 16);
    default: return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 19);
  }
}

template <int NB>
__global__ void __launch_bounds__(gtc::kThreads, 1) gemv_tc_kernel(const GemvTcParams p) {
  using C = gtc::Cfg<NB>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemvTcSmem<NB> L = gemv_tc_layout<NB>(p.max_ng);
  unsigned char* xb = smem + L.xb;
  int* xsum = reinterpret_cast<int*>(smem + L.xsum);
  float* xf = reinterpret_cast<float*>(smem + L.xf);
  float* part = reinterpret_cast<float*>(smem + L.part);
  uint64_t* a_ready = reinterpret_cast<uint64_t*>(smem + L.bars);  // [2]
  uint64_t* d_ready = a_ready + 2;                                  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(a_ready + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p.S > 1) cluster_arrive_relaxed();  // matched by the wait before the first remote store
  const int crank = static_cast<int>(cluster_ctarank());
  const int q = static_cast<int>(cluster_id_x()), Q = static_cast<int>(nclusters_x());
  // rows of this cluster, groups of this CTA
  const int r0 = static_cast<int>((static_cast<int64_t>(q) * p.N) / Q);
  const int r1 = static_cast<int>((static_cast<int64_t>(q + 1) * p.N) / Q);
  const int R = r1 - r0;  // <= 128
  const int g0 = (crank * p.NG) / p.S;
  const int ng = ((crank + 1) * p.NG) / p.S - g0;
  const int NR = (ng + 3) >> 2;  // rounds of 4 groups

  if (threadIdx.x == 0) {
    mbar_init(&a_ready[0], gtc::kWorkerWarps);
    mbar_init(&a_ready[1], gtc::kWorkerWarps);
    mbar_init(&d_ready[0], 1);
    mbar_init(&d_ready[1], 1);
    fence_mbarrier_init();
  }
  if (warp == gtc::kCtl) {
    tmem_alloc(tmem_slot, C::COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (!p.early) {
    pdl_wait();
    pdl_launch_dependents();
  }

  // ---- worker identity: TMEM lane quarter lq, K part kp; row rr = 32 lq + lane
  const int lq = warp & 3, kp = warp >> 2;
  const int rr = 32 * lq + lane;
  const bool row_ok = (warp < gtc::kWorkerWarps) && (rr < R);
  const int64_t row = r0 + (row_ok ? rr : 0);
  // ---- this thread's sign words and scales: a 4-round-deep prefetch window
  constexpr int kWin = 4;
  uint4 wv[kWin];
  uint16_t sv[kWin];
  const uint4* wp = reinterpret_cast<const uint4*>(p.signs + row * (p.K >> 5)) + g0 + kp;
  const uint16_t* spp = p.scales + row * p.NG + g0 + kp;
  auto load_words = [&](int r, uint4& w) {
    w = (row_ok && (4 * r + kp) < ng) ? __ldcs(wp + 4 * r) : make_uint4(0, 0, 0, 0);
  };
  auto load_scale = [&](int r, uint16_t& sc) {
    sc = (row_ok && (4 * r + kp) < ng) ? __ldg(spp + 4 * r) : static_cast<uint16_t>(0);
  };
#pragma unroll
  for (int r = 0; r < kWin; ++r) {
    load_words(r, wv[r]);
    load_scale(r, sv[r]);
  }
  if (p.early) {  // weights were written before the previous kernel began (W1_GEMV_STATIC_WEIGHTS)
    pdl_wait();
    pdl_launch_dependents();
  }

  // ---- activations -> int8 digit tiles (B operand) in shared memory
  {
    // zero the digit rows no batch row uses
    if (3 * NB < C::N) {
      const int per = (C::N - 3 * NB) * 128 / 16;  // 16-byte chunks per group
      for (int i = threadIdx.x; i < ng * per; i += gtc::kThreads) {
        const int gl = i / per, c = i - gl * per;
        *reinterpret_cast<uint4*>(xb + gl * C::TILE + 3 * NB * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    const int sub = lane & 7, t = sub >> 1, hh = sub & 1;
    const int items = NB * ng;
    // item = (batch row b, group gl): 8 lanes x 16 elements.  Two items per
    // lane in flight: the next item's loads are issued before this one's math.
    auto load_item = [&](int item, uint4 (&u)[2]) {
      u[0] = make_uint4(0, 0, 0, 0);
      u[1] = make_uint4(0, 0, 0, 0);
      if (item < items) {
        const int b = item / ng, gl = item - b * ng;
        const uint16_t* xp = p.x + static_cast<int64_t>(b) * p.K + 128 * (g0 + gl) + 32 * t + 16 * hh;
        u[0] = *reinterpret_cast<const uint4*>(xp);
        u[1] = *reinterpret_cast<const uint4*>(xp + 8);
      }
    };
    auto process = [&](const uint4 (&u)[2], int item) {
      const bool valid = item < items;
      const int b = valid ? item / ng : 0;
      const int gl = valid ? item - b * ng : 0;
      float v[16];
      const uint32_t w[8] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(v[i]));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
      int E = 0;
      if (mx > 0.f) frexpf(mx, &E);  // mx = f 2^E, f in [0.5, 1)
      const int sf = 22 - E, sf1 = sf / 2, sf2 = sf - sf1;
      const float m1 = __uint_as_float(static_cast<uint32_t>(sf1 + 127) << 23);
      const float m2 = __uint_as_float(static_cast<uint32_t>(sf2 + 127) << 23);
      uint32_t e[16];
      uint32_t bsum = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // 0x4B400000 + round(x 2^sf), exact for |x 2^sf| < 2^22 (1.5 * 2^23 trick)
        const uint32_t bits = __float_as_uint(fmaf(v[i] * m1, m2, 12582912.0f));
        bsum += bits;
        e[i] = (bits - 0x4ABF7F80u) ^ 0x00808080u;  // bytes: signed digits lo, mid, hi
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
        unsigned char* tile = xb + gl * C::TILE;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          // elements r, r+4, r+8, r+12 of this lane are bits q&3 + 4i of word t, q = r + 4 hh:
          // k-slots 32 t + 4 q + i of the MMA
          const uint32_t e0 = e[r], e1 = e[r + 4], e2 = e[r + 8], e3 = e[r + 12];
          const uint32_t p01 = prmt(e0, e1, 0x5140u), p23 = prmt(e2, e3, 0x5140u);
          const uint32_t dlo = prmt(p01, p23, 0x5410u);
          const uint32_t dmid = prmt(p01, p23, 0x7632u);
          const uint32_t dhi = prmt(prmt(e0, e1, 0x0062u), prmt(e2, e3, 0x0062u), 0x5410u);
          const int qq = r + 4 * hh;
          const int chunk = 2 * t + (qq >> 2);
          const int within = 4 * (qq & 3);
          const uint32_t dd[3] = {dhi, dmid, dlo};
#pragma unroll
          for (int pl = 0; pl < 3; ++pl) {
            const int n = 3 * b + pl;  // digit column
            *reinterpret_cast<uint32_t*>(tile + n * 128 + ((chunk ^ (n & 7)) << 4) + within) = dd[pl];
          }
        }
      }
    };
    constexpr int kStep = (gtc::kThreads / 32) * 4;  // items per pass of the CTA
    const int i0 = warp * 4 + (lane >> 3);
    uint4 xa[2], xb[2];
    load_item(i0, xa);
    for (int j = 0; warp * 4 + j * kStep < items; j += 2) {  // trip count uniform per warp
      load_item(i0 + (j + 1) * kStep, xb);
      process(xa, i0 + j * kStep);
      if (warp * 4 + (j + 1) * kStep >= items) break;
      load_item(i0 + (j + 2) * kStep, xa);
      process(xb, i0 + (j + 1) * kStep);
    }
  }
  fence_async_shared();
  __syncthreads();

  float acc[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = 0.f;

  if (warp == gtc::kCtl) {
    // ---------------------------------------------- MMA issue (one thread)
    if (lane == 0) {
      const uint32_t xbase = smem_u32(xb);
      for (int r = 0; r < NR; ++r) {
        const int buf = r & 1;
        if (!mbar_wait(&a_ready[buf], (r >> 1) & 1)) break;
        tc_fence_after();
        for (int slot = 0; slot < 4; ++slot) {
          const int gl = 4 * r + slot;
          if (gl >= ng) break;
          const uint32_t d = tmem + C::DCOL0 + (buf * 4 + slot) * C::N;
          const uint32_t a = tmem + (buf * 4 + slot) * 32;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_i8_ts(d, a + kk * 8, smem_desc_sw128(xbase + gl * C::TILE + kk * 32), C::IDESC, kk > 0 ? 1u : 0u);
        }
        tc_commit(&d_ready[buf]);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------- workers
    const uint32_t lane_addr = static_cast<uint32_t>(32 * lq) << 16;
    bool live = true;
#pragma unroll
    for (int r = 0; r <= gtc::kMaxRounds; ++r) {
      if (r > NR || !live) break;
      if (r < NR) {
        // expand this round's group into A slot (r & 1, kp)
        const uint4 w4 = wv[r % kWin];
        if (r + kWin < gtc::kMaxRounds) load_words(r + kWin, wv[r % kWin]);
        const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
        uint32_t a[32];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int qq = 0; qq < 8; ++qq) a[8 * t + qq] = tc_extract(qq, words[t]);
        tmem_st32(tmem + lane_addr + ((r & 1) * 4 + kp) * 32, a);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_ready[r & 1]);
      }
      if (r >= 1) {
        // fold the previous round's group
        const int pr = r - 1, buf = pr & 1;
        if (!mbar_wait_warp(&d_ready[buf], (pr >> 1) & 1)) {
          live = false;
          break;
        }
        tc_fence_after();
        const int gl = 4 * pr + kp;
        uint32_t dv[C::N];
        const uint32_t dadr = tmem + lane_addr + C::DCOL0 + (buf * 4 + kp) * C::N;
        if constexpr (C::N == 8) tmem_ld8(dadr, *reinterpret_cast<uint32_t(*)[8]>(dv));
        else if constexpr (C::N == 16) tmem_ld16(dadr, *reinterpret_cast<uint32_t(*)[16]>(dv));
        else tmem_ld32(dadr, *reinterpret_cast<uint32_t(*)[32]>(dv));
        tc_wait_ld();
        tc_fence_before();
        if (gl < ng) {
          const float s = __half2float(__ushort_as_half(sv[pr % kWin]));
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const int X = xsum[gl * NB + b];
            const float f = xf[gl * NB + b];
            const int V = X + 131072 * static_cast<int>(dv[3 * b]) + 512 * static_cast<int>(dv[3 * b + 1]) +
                          2 * static_cast<int>(dv[3 * b + 2]);
            acc[b] = fmaf(s * f, static_cast<float>(V), acc[b]);
          }
        }
        if (pr + kWin < gtc::kMaxRounds) load_scale(pr + kWin, sv[pr % kWin]);
      }
    }
    // K-part partials of this row
#pragma unroll
    for (int b = 0; b < NB; ++b) part[(kp * NB + b) * 128 + rr] = acc[b];
  }
  tc_fence_before();
  __syncthreads();  // every partial written; every MMA complete (the workers waited for them)
  tc_fence_after();
  if (warp == gtc::kCtl) tmem_dealloc(tmem, C::COLS);
  // ---- reduce: the 4 K parts here (fixed order), then the S CTAs of the
  // cluster: each CTA stores its per-row sums straight into the owning CTA's
  // inbox (DSMEM) and one cluster barrier later the owner adds them in order.
  if (p.S == 1) {
    for (int i = threadIdx.x; i < R * NB; i += gtc::kThreads) {
      const int b = i / R, r = i - b * R;
      float sum = 0.f;
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) sum += part[(k4 * NB + b) * 128 + r];
      p.y[static_cast<int64_t>(b) * p.N + r0 + r] = sum;
    }
  } else {
    float* inbox = reinterpret_cast<float*>(smem + L.inbox);
    const int chunk = (R + p.S - 1) / p.S;
    cluster_wait();  // every CTA of the cluster has started (arrived at kernel entry)
    for (int i = threadIdx.x; i < R * NB; i += gtc::kThreads) {
      const int b = i / R, r = i - b * R;
      float sum = 0.f;
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) sum += part[(k4 * NB + b) * 128 + r];
      const int owner = r / chunk, ro = r - owner * chunk;
      const uint32_t local = smem_u32(inbox + (crank * NB + b) * chunk + ro);
      st_dsmem_f32(map_shared_rank(local, static_cast<uint32_t>(owner)), sum);
    }
    cluster_sync();
    const int lo = crank * chunk, hi = min(R, lo + chunk), span = hi - lo;
    for (int i = threadIdx.x; i < span * NB; i += gtc::kThreads) {
      const int b = i / span, ro = i - b * span;
      float sum = 0.f;
      for (int c = 0; c < p.S; ++c) sum += inbox[(c * NB + b) * chunk + ro];
      p.y[static_cast<int64_t>(b) * p.N + r0 + lo + ro] = sum;
    }
  }
}

// ------------------------------------------------------------------ host side

template <int NB>
static int gemv_tc_max_clusters(int S, int smem_bytes) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(S * 64));
  cfg.blockDim = dim3(gtc::kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (ensure_dyn_smem(reinterpret_cast<const void*>(gemv_tc_kernel<NB>), smem_bytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, gemv_tc_kernel<NB>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

struct GemvTcPlan {
  int Q, S, max_ng, smem;
};

// Rows per CTA <= 128 (one TMEM lane each), groups per CTA <= 32; among the
// K splits that allow it, prefer ~100-128 rows per CTA and few rounds.
template <int NB>
static bool gemv_tc_plan(int N, int NG, int num_sms, int force_s, GemvTcPlan* out) {
  double best = 1e300;
  bool found = false;
  for (int S = 1; S <= 8; S *= 2) {
    if (force_s && S != force_s) continue;
    if (S > NG) break;
    const int max_ng = (NG + S - 1) / S;
    if (max_ng > gtc::kMaxGroups) continue;
    const int smem = gemv_tc_layout<NB>(max_ng).total;
    if (smem > 200 * 1024) continue;
    int Q = num_sms / S;
    const int occ = gemv_tc_max_clusters<NB>(S, smem);
    if (occ > 0 && occ < Q) Q = occ;
    if (Q < 1) continue;
    if ((N + Q - 1) / Q > 128) continue;
    if (Q > N) Q = N;
    const int rows = (N + Q - 1) / Q;
    const int rounds = (max_ng + 3) / 4;
    // work per CTA ~ rows * groups spread over 4 K parts; latency ~ rounds
    const double cost = rounds * 0.35 + static_cast<double>(rows) * max_ng / (128.0 * 4.0) * 0.05 +
                        (S > 1 ? 0.3 : 0.0) + 0.02 * NB * max_ng;
    if (cost < best) {
      best = cost;
      *out = GemvTcPlan{Q, S, max_ng, smem};
      found = true;
    }
  }
  return found;
}

struct GemvTcPlanEntry {
  int N, NG, NB, sms, dev, force;
  bool ok;
  GemvTcPlan plan;
};
static GemvTcPlanEntry g_tc_plan_cache[64];
static int g_tc_plan_count = 0;
static std::mutex g_tc_plan_mu;

// Cached plan lookup; false when the shape is outside this kernel's limits.
template <int NB>
static bool gemv_tc_cached_plan(int N, int NG, int num_sms, int force_s, GemvTcPlan* out) {
  int force = force_s;
  if (!force)
    force = knob(kKnobGemvSplit);  // tuning knob: force the K split
  if (force != 1 && force != 2 && force != 4 && force != 8) force = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(g_tc_plan_mu);
    for (int i = 0; i < g_tc_plan_count; ++i) {
      const GemvTcPlanEntry& e = g_tc_plan_cache[i];
      if (e.N == N && e.NG == NG && e.NB == NB && e.sms == num_sms && e.dev == dev && e.force == force) {
        *out = e.plan;
        return e.ok;
      }
    }
  }
  GemvTcPlan plan = {};
  const bool ok = gemv_tc_plan<NB>(N, NG, num_sms, force, &plan);
  std::lock_guard<std::mutex> lock(g_tc_plan_mu);
  const int i = g_tc_plan_count < 64 ? g_tc_plan_count++ : (N + NG + NB) & 63;
  g_tc_plan_cache[i] = GemvTcPlanEntry{N, NG, NB, num_sms, dev, force, ok, plan};
  *out = plan;
  return ok;
}

template <int NB>
static cudaError_t launch_gemv_tc_nb(const GemvTcParams& base, cudaStream_t stream, int num_sms, int force_s) {
  GemvTcPlan plan;
  if (!gemv_tc_cached_plan<NB>(base.N, base.NG, num_sms, force_s, &plan)) return cudaErrorNotSupported;
  if (knob(kKnobVerbose))
    fprintf(stderr, "w1_gemv(tc) plan: N=%d NG=%d B=%d -> clusters=%d split=%d groups=%d smem=%d\n", base.N,
            base.NG, NB, plan.Q, plan.S, plan.max_ng, plan.smem);
  GemvTcParams p = base;
  p.S = plan.S;
  p.max_ng = plan.max_ng;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(gemv_tc_kernel<NB>), plan.smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.Q * plan.S));
  cfg.blockDim = dim3(gtc::kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(plan.S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemv_tc_kernel<NB>, p);
}

// Returns cudaErrorNotSupported when the shape is outside this kernel's plan
// (the caller then uses the mma.sync kernel).
cudaError_t launch_gemv_tc(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K, const uint16_t* x,
                           int B, float* y, bool static_weights, cudaStream_t stream, int num_sms, int force_s) {
  if (N > (int64_t)1 << 30) return cudaErrorNotSupported;
  GemvTcParams p = {};
  p.signs = signs;
  p.scales = scales;
  p.x = x;
  p.y = y;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.NG = static_cast<int>(K / 128);
  p.early = static_weights ? 1 : 0;
  switch (B) {
    case 1: return launch_gemv_tc_nb<1>(p, stream, num_sms, force_s);
    case 2: return launch_gemv_tc_nb<2>(p, stream, num_sms, force_s);
    case 3: return launch_gemv_tc_nb<3>(p, stream, num_sms, force_s);
    case 4: return launch_gemv_tc_nb<4>(p, stream, num_sms, force_s);
    case 5: return launch_gemv_tc_nb<5>(p, stream, num_sms, force_s);
    case 6: return launch_gemv_tc_nb<6>(p, stream, num_sms, force_s);
    case 7: return launch_gemv_tc_nb<7>(p, stream, num_sms, force_s);
    default: return launch_gemv_tc_nb<8>(p, stream, num_sms, force_s);
  }
}

}  // namespace w1

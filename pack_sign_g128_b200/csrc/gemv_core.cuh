// Building blocks of the int8-MMA GEMV shared by w1_gemv and the small-batch
// DBF chain.  See gemv.cu for the design.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "w1_common.cuh"

namespace w1 {

constexpr int kConsumerWarps = 16;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;
constexpr int kProducerWarp = kConsumerWarps;

template <int NB>
struct GemvLayout {
  // n-tiles of the MMA.  B <= 2: one tile, columns (hi, mid) of rows 0, 1 at
  // 0-3 and lo digits at 4, 5.  B > 2: tile 0 = (hi, mid) digits of batch
  // rows 0-3, tile 1 = lo digits of rows t and t+4, tile 2 = (hi, mid) digits
  // of rows 4-7.
  static constexpr int NT = (NB <= 2) ? 1 : (NB <= 4) ? 2 : 3;
  static constexpr int N0 = NB < 4 ? NB : 4;
  static constexpr int N1 = NB > 4 ? NB - 4 : 0;
  static constexpr int COLS = 3 * NB;            // used digit columns
  static constexpr int BLOCK = COLS * 32;         // bytes per (group, k-step) block
};

// Compact index of MMA column c of n-tile j among the used columns, or -1.
template <int NB>
__host__ __device__ inline int digit_col(int j, int c) {
  using L = GemvLayout<NB>;
  if (L::NT == 1) {
    if (j != 0) return -1;
    if (c < 2 * NB) return c;
    return (c >= 4 && c - 4 < NB) ? 2 * NB + (c - 4) : -1;
  }
  if (j == 0) return c < 2 * L::N0 ? c : -1;
  if (j == 1) {
    const int t = c >> 1;
    if ((c & 1) == 0) return t < L::N0 ? 2 * L::N0 + t : -1;
    return t < L::N1 ? 3 * L::N0 + t : -1;
  }
  return c < 2 * L::N1 ? 3 * L::N0 + L::N1 + c : -1;
}

__host__ __device__ inline int round_up(int v, int a) { return (v + a - 1) / a * a; }

// Consumer warps sharing one 16-row tile (each takes a K sub-range).
__host__ __device__ inline int gemv_wpt(int max_tiles) {
  const int w = max_tiles > 0 ? kConsumerWarps / max_tiles : kConsumerWarps;
  return w < 1 ? 1 : w;
}

// Work of one CTA in one product: its cluster's 16-row tiles and its K groups.
struct Split {
  int ntiles;       // 16-row tiles of this cluster
  int g0, ng;       // K groups [g0, g0 + ng) of this CTA
  int nbox;         // TMA boxes per tile (each bw groups wide)
  int wpt;          // consumer warps per tile (K sub-ranges of a tile)
  int rows_c;       // valid rows of this cluster
  int64_t r_first;  // first row of this cluster
};

__device__ inline Split make_split(int rows, int64_t row_base, int NG, int S, int crank, int q, int Q, int bw,
                                   int gq, int max_tiles) {
  Split s;
  const int T16 = (rows + 15) >> 4;
  const int tq0 = static_cast<int>((static_cast<int64_t>(q) * T16) / Q);
  const int tq1 = static_cast<int>((static_cast<int64_t>(q + 1) * T16) / Q);
  s.ntiles = tq1 - tq0;
  // K split in units of gq groups (a multiple of the box width)
  const int units = (NG + gq - 1) / gq;
  const int u0 = (crank * units) / S, u1 = ((crank + 1) * units) / S;
  s.g0 = u0 * gq;
  s.ng = min(NG, u1 * gq) - s.g0;
  if (s.ng < 0) s.ng = 0;
  s.nbox = (s.ng + bw - 1) / bw;
  // the same in every CTA (peers read each other's partial buffers)
  s.wpt = gemv_wpt(max_tiles);
  s.r_first = row_base + static_cast<int64_t>(tq0) * 16;
  const int64_t left = row_base + rows - s.r_first;
  s.rows_c = static_cast<int>(left < s.ntiles * 16 ? left : s.ntiles * 16);
  return s;
}

// Shared-memory views of one product.
struct GemvSmemView {
  unsigned char* stages;  // ns stages of (nbox_max x 16 rows x 16 bw bytes), 1024-aligned
  int ns;
  int stage_bytes;
  uint64_t* full;
  uint64_t* empty;
};
struct GemvXView {
  unsigned char* xq;  // digit planes: [group][k-step][COLS][4 lanes][8 bytes]
  int* xsum;          // [group][NB] sum of fixed-point x
  float* xf;          // [group][NB] 2^(E - 22)
  uint16_t* sc;       // [row][group] fp16 scales (if any)
  float* part;        // [wpt][NB][part_stride] partial sums of this CTA
  int part_stride;
};

// Producer: the boxes of tile `it` (16 rows x bw groups each) into its stage.
__device__ inline void issue_tile(const GemvSmemView& v, const Split& sp, const CUtensorMap* tmap, int bw, int it) {
  const int s = it % v.ns;
  const int row0 = static_cast<int>(sp.r_first) + it * 16;
  const int box_bytes = 16 * 16 * bw;
  mbar_arrive_expect_tx(&v.full[s], static_cast<uint32_t>(sp.nbox * box_bytes));
  for (int j = 0; j < sp.nbox; ++j)
    tma_load_2d(v.stages + s * v.stage_bytes + j * box_bytes, tmap, (sp.g0 + j * bw) * 4, row0, &v.full[s]);
}

__device__ inline int issue_first_tiles(const GemvSmemView& v, const Split& sp, const CUtensorMap* tmap, int bw) {
  const int first = min(sp.ntiles, v.ns);
  for (int it = 0; it < first; ++it) issue_tile(v, sp, tmap, bw, it);
  return first;
}

// Remaining tiles as stages free up (single thread).
__device__ inline void produce_rest(const GemvSmemView& v, const Split& sp, const CUtensorMap* tmap, int bw,
                                    int first) {
  for (int it = first; it < sp.ntiles; ++it) {
    const int s = it % v.ns;
    if (!mbar_wait(&v.empty[s], ((it / v.ns) - 1) & 1)) break;
    issue_tile(v, sp, tmap, bw, it);
  }
}

// Quantise this CTA's K-slice of the NB input rows into int8 digit planes.
// load(b, k, v) fills v[0..15] with input elements k .. k+15 of row b (fp32).
// Each (row, group) uses the exponent E of its max |x|: xi = round(x 2^(22-E))
// in (-2^22, 2^22), split into three signed bytes (hi, mid, lo).
template <int NB, class Load>
__device__ inline void quantise_input(const GemvXView& xv, const Split& sp, Load load, int nthreads) {
  using L = GemvLayout<NB>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane & 7;  // 8 lanes per (row, group) item
  const int t = sub >> 1;    // word within group
  const int hh = sub & 1;    // half word: bits 16 hh .. 16 hh + 15
  const int items = NB * sp.ng;
  const int nwarps = nthreads >> 5;
  for (int base = warp * 4; base < items; base += nwarps * 4) {
    const int item = base + (lane >> 3);
    const bool valid = item < items;
    const int b = valid ? item / sp.ng : 0;
    const int gl = valid ? item - b * sp.ng : 0;
    float v[16];
    if (valid) {
      load(b, 128 * (sp.g0 + gl) + 32 * t + 16 * hh, v);
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
    if (mx > 0.f) frexpf(mx, &E);  // mx = f 2^E, f in [0.5, 1)
    const int sf = 22 - E;
    const int sf1 = sf / 2, sf2 = sf - sf1;
    const float m1 = __uint_as_float(static_cast<uint32_t>(sf1 + 127) << 23);
    const float m2 = __uint_as_float(static_cast<uint32_t>(sf2 + 127) << 23);
    uint32_t e[16];
    uint32_t bsum = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      // bits = 0x4B400000 + round(x 2^sf) exactly, |x 2^sf| < 2^22 (1.5*2^23 trick)
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
        xv.xsum[gl * NB + b] = xs;
        xv.xf[gl * NB + b] = ldexpf(1.0f, E - 22);
      }
      const int jt_hi = (b < 4) ? 0 : 2;
      const int c_hi = 2 * (b & 3);
      const int c_lo = (L::NT == 1) ? 4 + b : (b < 4) ? 2 * b : 2 * (b - 4) + 1;
      const int ci_hi = digit_col<NB>(jt_hi, c_hi), ci_mid = digit_col<NB>(jt_hi, c_hi + 1);
      const int ci_lo = digit_col<NB>(L::NT == 1 ? 0 : 1, c_lo);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // elements r, r+4, r+8, r+12 of this lane share q = r + 4 hh
        const uint32_t e0 = e[r], e1 = e[r + 4], e2 = e[r + 8], e3 = e[r + 12];
        const uint32_t p01 = prmt(e0, e1, 0x5140u), p23 = prmt(e2, e3, 0x5140u);
        const uint32_t d0 = prmt(p01, p23, 0x5410u);
        const uint32_t d1 = prmt(p01, p23, 0x7632u);
        const uint32_t d2 = prmt(prmt(e0, e1, 0x0062u), prmt(e2, e3, 0x0062u), 0x5410u);
        const int qq = r + 4 * hh;
        const int m = qq >> 1, h = qq & 1;
        unsigned char* blk = xv.xq + (gl * 4 + m) * L::BLOCK + t * 8 + h * 4;
        *reinterpret_cast<uint32_t*>(blk + ci_hi * 32) = d2;
        *reinterpret_cast<uint32_t*>(blk + ci_mid * 32) = d1;
        *reinterpret_cast<uint32_t*>(blk + ci_lo * 32) = d0;
      }
    }
  }
}

// Stage this CTA's fp16 scales [rows_c][ng] in shared memory; loads are
// issued eight at a time before any store so their latencies overlap.
__device__ inline void stage_scales(const GemvXView& xv, const Split& sp, const uint16_t* scales, int NG,
                                    int nthreads) {
  const int total = sp.rows_c * sp.ng;
  for (int base = threadIdx.x; base < total; base += 8 * nthreads) {
    uint16_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * nthreads;
      if (i < total) {
        const int r = i / sp.ng, gl = i - r * sp.ng;
        v[u] = __ldg(scales + (sp.r_first + r) * NG + sp.g0 + gl);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * nthreads;
      if (i < total) xv.sc[i] = v[u];
    }
  }
}

// -(bit q + 4i of w) for i = 0..3 as int8 bytes (PRMT with 0x00/0xFF tables);
// w3 = w >> 3, w16 = w >> 16, w19 = w >> 19 are precomputed.
__device__ __forceinline__ uint32_t extract_q(int q, uint32_t w, uint32_t w3, uint32_t w16, uint32_t w19) {
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

// Word t of group gl, row r of a stage written by swizzled TMA boxes
// (16 rows x bw groups of 16 bytes; 16-byte chunk index XOR the swizzle row).
__device__ __forceinline__ uint32_t stage_word(const unsigned char* st, int bw, int r, int gl, int t) {
  const int box = gl / bw, c = gl - box * bw;
  const int pitch = 16 * bw;
  const int f = ((r * pitch) >> 7) & (bw - 1);
  return *reinterpret_cast<const uint32_t*>(st + box * 16 * pitch + r * pitch + ((c ^ f) << 4) + t * 4);
}

// Consumer warps: units (tile, K sub-range) round-robin; each unit's partial
// sums for its 16 rows go to xv.part[sub].  HAS_SCALES: multiply each group by
// s[row][g] (else by 1).
template <int NB, bool HAS_SCALES>
__device__ inline void consume_tiles(const GemvSmemView& v, const GemvXView& xv, const Split& sp, int bw,
                                     const unsigned char* zero16, int warp, int lane) {
  using L = GemvLayout<NB>;
  constexpr int NT = L::NT;
  const int g = lane >> 2, t = lane & 3;
  // this lane's B-fragment base per n-tile; unused columns read a zero block
  const unsigned char* boff[NT];
  int bmul[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int ci = digit_col<NB>(j, g);
    boff[j] = ci >= 0 ? xv.xq + ci * 32 + t * 8 : zero16;
    bmul[j] = ci >= 0 ? 1 : 0;
  }
  // Warp group grp (wpt warps, one per K sub-range) takes tiles grp, grp + G,
  // ...  When stages are reused (ns < tiles), G divides ns, so every use of a
  // stage is awaited by the same warp group in order: a waiter is never more
  // than one barrier phase ahead.
  int G = kConsumerWarps / sp.wpt;
  if (G < 1) G = 1;
  if (v.ns < sp.ntiles)
    while (v.ns % G) --G;
  const int grp = warp / sp.wpt, sub = warp - grp * sp.wpt;
  if (grp >= G) return;
  for (int it = grp; it < sp.ntiles; it += G) {
    const int s = it % v.ns;
    if (!mbar_wait_warp(&v.full[s], (it / v.ns) & 1)) break;
    const unsigned char* st = v.stages + s * v.stage_bytes;
    const int gl0 = (sub * sp.ng) / sp.wpt, gl1 = ((sub + 1) * sp.ng) / sp.wpt;
    const int rl0 = it * 16;
    const int rA = rl0 + g, rB = rl0 + g + 8;
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 2
    for (int gl = gl0; gl < gl1; ++gl) {
      const uint32_t wA = stage_word(st, bw, g, gl, t);
      const uint32_t wB = stage_word(st, bw, g + 8, gl, t);
      const uint32_t wA3 = wA >> 3, wA16 = wA >> 16, wA19 = wA >> 19;
      const uint32_t wB3 = wB >> 3, wB16 = wB >> 16, wB19 = wB >> 19;
      int C[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j) C[j][0] = C[j][1] = C[j][2] = C[j][3] = 0;
      const int blk = gl * 4 * L::BLOCK;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t a[4];
        a[0] = extract_q(2 * m, wA, wA3, wA16, wA19);
        a[1] = extract_q(2 * m, wB, wB3, wB16, wB19);
        a[2] = extract_q(2 * m + 1, wA, wA3, wA16, wA19);
        a[3] = extract_q(2 * m + 1, wB, wB3, wB16, wB19);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const unsigned char* bp = boff[j] + (blk + m * L::BLOCK) * bmul[j];
          const uint2 bb = *reinterpret_cast<const uint2*>(bp);
          mma_s8_16832(C[j], a, bb.x, bb.y, C[j]);
        }
      }
      float sA = 1.f, sB = 1.f;
      if (HAS_SCALES) {
        sA = (rA < sp.rows_c) ? __half2float(__ushort_as_half(xv.sc[rA * sp.ng + gl])) : 0.f;
        sB = (rB < sp.rows_c) ? __half2float(__ushort_as_half(xv.sc[rB * sp.ng + gl])) : 0.f;
      }
      if (NT == 1) {
        // lo digits of batch rows 0 and 1 sit in columns 4 and 5 (lane t = 2)
        const int src = (lane & ~3) | 2;
        const int l0 = __shfl_sync(0xFFFFFFFFu, C[0][0], src), l1 = __shfl_sync(0xFFFFFFFFu, C[0][1], src);
        const int l2 = __shfl_sync(0xFFFFFFFFu, C[0][2], src), l3 = __shfl_sync(0xFFFFFFFFu, C[0][3], src);
        if (t < NB) {
          const int X = xv.xsum[gl * NB + t];
          const float f = xv.xf[gl * NB + t];
          const int VA = X + 131072 * C[0][0] + 512 * C[0][1] + 2 * (t == 0 ? l0 : l1);
          const int VB = X + 131072 * C[0][2] + 512 * C[0][3] + 2 * (t == 0 ? l2 : l3);
          acc[0][0] = fmaf(sA * f, static_cast<float>(VA), acc[0][0]);
          acc[1][0] = fmaf(sB * f, static_cast<float>(VB), acc[1][0]);
        }
      } else {
#pragma unroll
        for (int be = 0; be < 2; ++be) {
          const int b = t + 4 * be;
          if (b < NB) {
            const int jh = (be && NT > 2) ? 2 : 0;
            const int X = xv.xsum[gl * NB + b];
            const float f = xv.xf[gl * NB + b];
            // sum (1-2 bit) x = X + 2 sum(-bit) x, digits weighted 2^16, 2^8, 1
            const int VA = X + 131072 * C[jh][0] + 512 * C[jh][1] + 2 * C[NT > 1 ? 1 : 0][be ? 1 : 0];
            const int VB = X + 131072 * C[jh][2] + 512 * C[jh][3] + 2 * C[NT > 1 ? 1 : 0][be ? 3 : 2];
            acc[0][be] = fmaf(sA * f, static_cast<float>(VA), acc[0][be]);
            acc[1][be] = fmaf(sB * f, static_cast<float>(VB), acc[1][be]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&v.empty[s]);
    float* pp = xv.part + sub * NB * xv.part_stride;
#pragma unroll
    for (int be = 0; be < 2; ++be) {
      const int b = t + 4 * be;
      if (b < NB) {
        if (rA < sp.rows_c) pp[b * xv.part_stride + rA] = acc[0][be];
        if (rB < sp.rows_c) pp[b * xv.part_stride + rB] = acc[1][be];
      }
    }
  }
}

// After a cluster barrier: this CTA sums its share of the cluster's rows over
// the wpt sub-partials of the S CTAs (fixed order, deterministic) and hands
// each sum to store(b, row, value).
template <int NB, class Store>
__device__ inline void cluster_reduce(const GemvXView& xv, const Split& sp, int S, int crank, Store store,
                                      int nthreads) {
  const int r_lo = (crank * sp.rows_c) / S;
  const int r_hi = ((crank + 1) * sp.rows_c) / S;
  const int span = r_hi - r_lo;
  const uint32_t part_base = smem_u32(xv.part);
  const int wpt = sp.wpt;
  for (int i = threadIdx.x; i < span * NB; i += nthreads) {
    const int b = i / span, r = r_lo + (i - b * span);
    float sum = 0.f;
    if (S == 1) {
      for (int sub = 0; sub < wpt; ++sub) sum += xv.part[(sub * NB + b) * xv.part_stride + r];
    } else {
      for (int sub = 0; sub < wpt; ++sub) {
        const uint32_t off = static_cast<uint32_t>(((sub * NB + b) * xv.part_stride + r) * 4);
        float vals[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) vals[c] = (c < S) ? ld_dsmem_f32(map_shared_rank(part_base + off, c)) : 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) sum += vals[c];
      }
    }
    store(b, sp.r_first + r, sum);
  }
}

}  // namespace w1

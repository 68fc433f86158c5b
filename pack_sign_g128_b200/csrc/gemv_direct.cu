// w1_gemv: the decode kernel (1 <= B <= 8).
//
//   y[b,n] = sum_g s[n,g] * sum_{k in g} (1 - 2 bit[n,k]) x[b,k]
//
// Storage format: "1-bit group-128 sign packing" (one sign bit per weight,
// LSB-first in uint32 words along K, one fp16 mean|w| scale per 128 weights).
//
// Built for latency: a decode GEMV moves a few MB, so the time of one launch is
// set by its serial chain, not by bandwidth.  The kernel therefore
//  * issues every weight byte it will need at its first instruction: each warp
//    copies its rows x K-range of sign words into shared memory with 16-byte
//    asynchronous copies (cp.async, every lane, all in flight at once) and,
//    with the W1_GEMV_STATIC_WEIGHTS flag, does so before waiting on the
//    previous kernel in the stream (programmatic dependent launch);
//  * quantises the activations of its K range once per CTA while those copies
//    are in flight, then lets every warp run alone until the final reduction;
//  * reduces the warps' partial sums with several threads per output (a
//    fixed-order butterfly), and a K split over a thread-block cluster with
//    one barrier: partial sums are stored straight into the owning CTA's
//    shared memory (DSMEM), and only the owner reads them.
// The kernel runs with 8 warps per CTA (two CTAs fit an SM, so the next
// launch's CTA can stage its weights early) or 16 (more latency hidden for
// large K ranges and B >= 4); the dispatcher times both.
//
// Arithmetic (exact up to the fp32 fold):
//  * Activations -> fixed point.  Per (batch row, group) x is scaled by
//    2^(22-E) (E from the group max), rounded to a 23-bit integer and split
//    into three signed int8 digits hi/mid/lo.  Error <= 2^(E-23) per element.
//  * Signs -> int8 {0, -1} with one PRMT per 4 weights (a byte table keyed on
//    bit 0, 1 or 2 of each selector nibble; bit 3 via w >> 3; upper half via
//    w >> 16), so  sum (1-2b) n = X + 2 * sum (-b) n  with X = sum n.
//  * int8 mma.sync m16n8k32, A = sign bytes (16 weight rows: two 8-row
//    n-tiles), B = activation digits (column 3b + p for batch row b and digit
//    p; columns past 3B are zero), s32 accumulators.  Four MMAs cover one
//    group of 16 rows (2048 weights), and each group is folded once:
//    acc += s * (f*W_p * D_p + [p = hi] f*X),  W = {2^17, 2^9, 2}, f = 2^(E-22).
// K order inside one MMA is free as long as A and B agree: k-slot 4c+i+16h of
// MMA q of a group holds bit q + 4i + 16h of the group's word c, which is the
// order the PRMT extraction produces.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cuda_fp16.h>
#include <mutex>
#include <type_traits>

#include "w1_common.cuh"

namespace w1 {

namespace gd {
constexpr int kWarps = 8;           // warps per CTA (the GEMV kernel also runs with 16)
constexpr int kThreads = kWarps * 32;
constexpr int kMaxTw = 4;        // 8-row n-tiles per warp
constexpr int kMaxTp = (kMaxTw + 1) / 2;  // 16-row MMA tiles per warp
constexpr int kDigitStride = 34;  // words per digit row of the activation scratch (bank spread)
constexpr int kMaxSets = 64;      // sets (of G groups) per CTA

template <int NB>
struct Cfg {
  static constexpr int G = 1;                      // groups per set
  static constexpr int NCOL = 3 * NB;              // digit columns: 3 per batch row
  static constexpr int NN = (NCOL + 7) / 8;        // 8-column MMA n-tiles
  static constexpr int ROWS = NCOL;                // digit rows of the activation scratch
  static constexpr int SCR = ROWS * kDigitStride + 2 * ROWS;  // scratch words: digits, f*W_p, f*X
  static constexpr int RED = 8 * NCOL;             // reduction floats per warp and n-tile
};

// Reduction buffer: per (warp block along sets, CTA n-tile) 8 rows x NCOL
// columns, plus one float of padding per warp block (bank spread).
template <int NB, int NW = kWarps>
__host__ __device__ inline int gd_red_bytes(int Tw) {
  return ((NW * Tw * Cfg<NB>::RED + NW) * 4 + 15) / 16 * 16;
}
}  // namespace gd

struct GdParams {
  const uint32_t* signs;
  const uint16_t* scales;  // fp16 group scales, or nullptr (every s = 1)
  const void* x;           // [B][K] bf16, or fp32 with x_f32
  const uint16_t* cdiag;   // fp16 [K] multiplied into x (bf16 x only), or nullptr
  const uint16_t* rdiag;   // fp16 [N] multiplied into y, or nullptr
  const int* xrows;        // batch row b reads row xrows[b] of x (nullptr: row b)
  float* y;                // [B][N]
  int x_f32;
  int N, K, NG;
  int S;      // CTAs per cluster (K split)
  int Q;      // clusters
  int NT;     // 8-row n-tiles in total
  int Wn, Wg;  // warps along n-tiles x along sets (Wn * Wg = warps per CTA)
  int Tw;     // n-tiles per warp (max)
  int NSw;    // sets per warp (max)
  int P;      // bytes per staged weight row
  int chunk;  // rows owned per CTA in the cluster reduction
  int NSc;    // sets per CTA (max)
  int lgS, lgWg;  // log2 of S and Wg
  int lgGw;   // log2 of the power-of-two stride >= NSw * G (staging loops)
  int tq, tr;  // NT = Q * tq + tr
  int early;  // read weights before the grid dependency wait
  int alias_red;  // the reduction buffer overlays the activation scratch (plans that need the room)
};

struct GdSmem {
  int warp_bytes, wts, scl, xs, red, part, total;
};

// Per warp: staged sign words (8*Tw rows of P bytes), scales (float,
// [group][row]).  Per CTA: activation scratch (nsc sets of SCR words), the
// reduction buffer and (cluster) the owner partials.
// With alias_red the reduction buffer starts at the activation scratch (it is
// written only after every warp has finished its products).  The cluster
// inbox never overlays anything: other CTAs may write it at any time.
template <int NB, int NW = gd::kWarps>
__host__ __device__ inline GdSmem gd_layout(int Tw, int NSw, int P, int S, int chunk, int nsc,
                                            bool alias_red = false) {
  using C = gd::Cfg<NB>;
  GdSmem L;
  L.wts = 0;
  L.scl = L.wts + 8 * Tw * P;
  L.warp_bytes = (L.scl + NSw * C::G * 8 * Tw * 4 + 15) / 16 * 16;
  L.xs = NW * L.warp_bytes;
  const int xs_bytes = (nsc * C::SCR * 4 + 15) / 16 * 16;
  const int red_bytes = gd::gd_red_bytes<NB, NW>(Tw);
  L.red = alias_red ? L.xs : L.xs + xs_bytes;
  L.part = alias_red ? L.xs + (xs_bytes > red_bytes ? xs_bytes : red_bytes) : L.red + red_bytes;
  L.total = L.part + (S > 1 ? S * NB * chunk * 4 : 0);
  return L;
}

// -(bit q + 4i of w), i = 0..3, as int8 bytes; q in 0..7 (4..7: upper half).
template <int Q>
__device__ __forceinline__ uint32_t sign_bytes(uint32_t w) {
  if constexpr (Q == 0) return prmt(0xFF00FF00u, 0xFF00FF00u, w);
  else if constexpr (Q == 1) return prmt(0xFFFF0000u, 0xFFFF0000u, w);
  else if constexpr (Q == 2) return prmt(0x00000000u, 0xFFFFFFFFu, w);
  else if constexpr (Q == 3) return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 3);
  else if constexpr (Q == 4) return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 16);
  else if constexpr (Q == 5) return prmt(0xFFFF0000u, 0xFFFF0000u, w >> 16);
  else if constexpr (Q == 6) return prmt(0x00000000u, 0xFFFFFFFFu, w >> 16);
  else return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 19);
}

__device__ __forceinline__ void mma_s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Quantise one 16-element activation item and store its digit words and
// (lane 0 of the item) the fold factors.  `v` holds x[k0 .. k0+15].
template <int NB>
__device__ __forceinline__ void quantise_item(const float (&v)[16], bool valid, int it, uint32_t* scr) {
  using C = gd::Cfg<NB>;
  float m8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m8[i] = fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1]));
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m8[i] = fmaxf(m8[i], m8[i + w]);
  float mx = m8[0];
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
  int E = 0;
  if (mx > 0.f) frexpf(mx, &E);  // mx = f 2^E, f in [0.5, 1): |x 2^(22-E)| < 2^22
  const int sf = 22 - E, sf1 = sf / 2, sf2 = sf - sf1;
  const float m1 = __uint_as_float(static_cast<uint32_t>(sf1 + 127) << 23);
  const float m2 = __uint_as_float(static_cast<uint32_t>(sf2 + 127) << 23);
  uint32_t e[16], bs[8];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    // 0x4B400000 + round(x 2^sf): exact rounding to an integer for |x 2^sf| < 2^22
    const uint32_t bits = __float_as_uint(fmaf(v[i] * m1, m2, 12582912.0f));
    if (i & 1) bs[i >> 1] += bits;
    else bs[i >> 1] = bits;
    e[i] = (bits - 0x4ABF7F80u) ^ 0x00808080u;  // bytes: signed digits lo, mid, hi
  }
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) bs[i] += bs[i + w];
  int xs = static_cast<int>(bs[0] - 16u * 0x4B400000u);
  xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 1);
  xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 2);
  xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 4);
  if (!valid) return;
  const int sub = it & 7, wi = sub >> 1, hh = sub & 1, gb = it >> 3;
  const int r0 = 3 * gb;  // digit rows r0 (hi), r0+1 (mid), r0+2 (lo)
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    // elements q, q+4, q+8, q+12 are bits q + 4i + 16 hh of word wi
    const uint32_t e0 = e[q], e1 = e[q + 4], e2 = e[q + 8], e3 = e[q + 12];
    const uint32_t p01 = prmt(e0, e1, 0x5140u), p23 = prmt(e2, e3, 0x5140u);
    const uint32_t dlo = prmt(p01, p23, 0x5410u);
    const uint32_t dmid = prmt(p01, p23, 0x7632u);
    const uint32_t dhi = prmt(prmt(e0, e1, 0x0062u), prmt(e2, e3, 0x0062u), 0x5410u);
    const int off = wi * 8 + q * 2 + hh;
    scr[(r0 + 0) * gd::kDigitStride + off] = dhi;
    scr[(r0 + 1) * gd::kDigitStride + off] = dmid;
    scr[(r0 + 2) * gd::kDigitStride + off] = dlo;
  }
  if (sub == 0) {
    const float f = ldexpf(1.0f, E - 22);
    float* fw = reinterpret_cast<float*>(scr + C::ROWS * gd::kDigitStride);
    float* cx = fw + C::ROWS;
    fw[r0 + 0] = f * 131072.0f;
    fw[r0 + 1] = f * 512.0f;
    fw[r0 + 2] = f * 2.0f;
    cx[r0 + 0] = f * static_cast<float>(xs);
    cx[r0 + 1] = 0.f;
    cx[r0 + 2] = 0.f;
  }
}

// One warp's products over its n-tiles (TW of them, a compile-time count so that
// no MMA sits under a per-tile branch) and its sets (one group each).  An MMA
// takes n-tiles 2tp and 2tp+1 as its A rows 0-7 and 8-15.  Returns the fp32
// partial sums in acc[tp][nn][e] (C-fragment order: weight row lane/4 of n-tile
// 2tp + (e>>1), digit column 8nn + 2(lane&3) + (e&1)).
template <int NB, int TW>
__device__ __forceinline__ void gd_compute(const unsigned char* wts, int P, const float* scl, int sstride,
                                           const uint32_t* xs, int nsw, int lane,
                                           float (&acc)[gd::kMaxTp][gd::Cfg<NB>::NN][4]) {
  using C = gd::Cfg<NB>;
  constexpr int NN = C::NN, NCOL = C::NCOL, TP = (TW + 1) / 2;
  const int r1 = lane >> 2, cq = lane & 3;
  // B-fragment source of this lane: digit column 8nn + lane/4, word lane&3
  int bofs[NN];
  bool bact[NN];
#pragma unroll
  for (int nn = 0; nn < NN; ++nn) {
    const int n = 8 * nn + r1;
    bact[nn] = n < NCOL;
    bofs[nn] = n * gd::kDigitStride + cq * 8;
  }
  // A-fragment source: word lane&3 of the group in weight rows lane/4 (+8)
  const unsigned char* wrow = wts + r1 * P + cq * 4;
  for (int si = 0; si < nsw; ++si) {
    const uint32_t* scr = xs + si * C::SCR;
    uint32_t W0[TP], W1[TP];
#pragma unroll
    for (int tp = 0; tp < TP; ++tp) {
      W0[tp] = *reinterpret_cast<const uint32_t*>(wrow + 16 * tp * P + si * 16);
      W1[tp] = (2 * tp + 1 < TW) ? *reinterpret_cast<const uint32_t*>(wrow + (16 * tp + 8) * P + si * 16) : 0u;
    }
    int Cacc[TP][NN][4];
#pragma unroll
    for (int tp = 0; tp < TP; ++tp)
#pragma unroll
      for (int nn = 0; nn < NN; ++nn)
#pragma unroll
        for (int e = 0; e < 4; ++e) Cacc[tp][nn][e] = 0;
    auto step = [&](auto qc) {
      constexpr int qq = decltype(qc)::value;
      uint32_t B0[NN], B1[NN];
#pragma unroll
      for (int nn = 0; nn < NN; ++nn) {
        uint2 u = make_uint2(0, 0);
        if (bact[nn]) u = *reinterpret_cast<const uint2*>(scr + bofs[nn] + qq * 2);
        B0[nn] = u.x;
        B1[nn] = u.y;
      }
#pragma unroll
      for (int tp = 0; tp < TP; ++tp) {
        const uint32_t A[4] = {sign_bytes<qq>(W0[tp]), sign_bytes<qq>(W1[tp]), sign_bytes<qq + 4>(W0[tp]),
                               sign_bytes<qq + 4>(W1[tp])};
#pragma unroll
        for (int nn = 0; nn < NN; ++nn) mma_s8(Cacc[tp][nn], A, B0[nn], B1[nn]);
      }
    };
    step(std::integral_constant<int, 0>{});
    step(std::integral_constant<int, 1>{});
    step(std::integral_constant<int, 2>{});
    step(std::integral_constant<int, 3>{});
    // fold: acc += s[row, group] * (f W_p D + [hi] f X)
    const float* fwv = reinterpret_cast<const float*>(scr + C::ROWS * gd::kDigitStride);
    float fw[NN][2], cx[NN][2];
#pragma unroll
    for (int nn = 0; nn < NN; ++nn)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = 8 * nn + 2 * cq + c;
        fw[nn][c] = n < NCOL ? fwv[n] : 0.f;
        cx[nn][c] = n < NCOL ? fwv[C::ROWS + n] : 0.f;
      }
    const float* sset = scl + si * sstride + r1;
#pragma unroll
    for (int tp = 0; tp < TP; ++tp) {
      const float s0 = sset[16 * tp];
      const float s1 = (2 * tp + 1 < TW) ? sset[16 * tp + 8] : 0.f;
#pragma unroll
      for (int nn = 0; nn < NN; ++nn)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          acc[tp][nn][c] = fmaf(s0, fmaf(fw[nn][c], static_cast<float>(Cacc[tp][nn][c]), cx[nn][c]), acc[tp][nn][c]);
          acc[tp][nn][2 + c] =
              fmaf(s1, fmaf(fw[nn][c], static_cast<float>(Cacc[tp][nn][2 + c]), cx[nn][c]), acc[tp][nn][2 + c]);
        }
    }
  }
}

// ---- one product, split into device steps (the GEMV kernel runs one, the
// DBF chain kernel two, with a grid barrier between them)

// This CTA's share (cluster q's n-tiles, K sets [cs0, cs0 + nsc)) and this
// warp's block of both.
struct GdGeom {
  int crank, cs0, nsc, t0c, Tq, wn, wg, tw, ws0, nsw, row0, nrows, g0, ngw;
  bool busy;
};

template <int NB>
__device__ __forceinline__ GdGeom gd_geom(const GdParams& p, int warp) {
  constexpr int G = gd::Cfg<NB>::G;
  GdGeom g;
  const int NS = (p.NG + G - 1) / G;
  g.crank = p.S > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int q = p.S > 1 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  g.cs0 = (g.crank * NS) >> p.lgS;
  g.nsc = (((g.crank + 1) * NS) >> p.lgS) - g.cs0;
  g.t0c = q * p.tq + min(q, p.tr);  // NT = Q * tq + tr tiles, the first tr clusters one more
  g.Tq = q < p.Q ? p.tq + (q < p.tr ? 1 : 0) : 0;
  g.wn = warp >> p.lgWg;
  g.wg = warp & (p.Wg - 1);
  g.tw = max(0, min(p.Tw, g.Tq - g.wn * p.Tw));              // n-tiles of this warp
  g.ws0 = g.cs0 + ((g.wg * g.nsc) >> p.lgWg);                 // first set of this warp
  g.nsw = g.cs0 + (((g.wg + 1) * g.nsc) >> p.lgWg) - g.ws0;   // sets of this warp
  g.row0 = (g.t0c + g.wn * p.Tw) * 8;                         // first weight row of this warp
  g.nrows = max(0, min(8 * g.tw, p.N - g.row0));
  g.busy = g.tw > 0 && g.nsw > 0;
  g.g0 = g.ws0 * G;                                           // first group of this warp
  g.ngw = g.busy ? min(g.nsw * G, p.NG - g.g0) : 0;           // real groups of this warp
  return g;
}

// This warp's sign words -> shared memory: 16-byte asynchronous copies, every
// lane, one commit group.
template <int NB>
__device__ __forceinline__ void gd_stage(const GdParams& p, const GdGeom& g, unsigned char* wts, int lane) {
  const int lgw = p.lgGw, gmask = (1 << lgw) - 1;  // power-of-two stride over a row's groups
  const int KW = p.K >> 5;
  const int n = g.nrows << lgw;
  for (int i = lane; i < n; i += 32) {
    const int r = i >> lgw, gg = i & gmask;
    if (gg < g.ngw)
      cp_async16(wts + r * p.P + gg * 16, p.signs + static_cast<int64_t>(g.row0 + r) * KW + 4 * (g.g0 + gg));
  }
  cp_async_commit();
}

// Scales: plain loads into registers (issued early), converted and stored to
// scl[group][row] later.  Without scales every value is 1.
constexpr int kGdSpl = 8;
template <int NB>
__device__ __forceinline__ void gd_load_scales(const GdParams& p, const GdGeom& g, int base, int lane,
                                               uint16_t (&sreg)[kGdSpl]) {
  constexpr int G = gd::Cfg<NB>::G;
  const int lgw = p.lgGw, gmask = (1 << lgw) - 1;
  const int nscl = g.busy ? (8 * g.tw) << lgw : 0;
#pragma unroll
  for (int j = 0; j < kGdSpl; ++j) {
    const int i = base + lane + 32 * j;
    const int rl = i >> lgw, gl = i & gmask;
    sreg[j] = 0;
    if (i < nscl && gl < g.nsw * G && g.row0 + rl < p.N && g.g0 + gl < p.NG)
      sreg[j] = p.scales ? __ldg(p.scales + static_cast<int64_t>(g.row0 + rl) * p.NG + g.g0 + gl)
                         : static_cast<uint16_t>(0x3C00u);
  }
}
template <int NB>
__device__ __forceinline__ void gd_store_scales(const GdParams& p, const GdGeom& g, int base, int lane,
                                                const uint16_t (&sreg)[kGdSpl], float* scl) {
  constexpr int G = gd::Cfg<NB>::G;
  const int lgw = p.lgGw, gmask = (1 << lgw) - 1;
  const int nscl = g.busy ? (8 * g.tw) << lgw : 0;
  const int sstride = 8 * p.Tw;
#pragma unroll
  for (int j = 0; j < kGdSpl; ++j) {
    const int i = base + lane + 32 * j;
    const int rl = i >> lgw, gl = i & gmask;
    if (i < nscl && gl < g.nsw * G) scl[gl * sstride + rl] = __half2float(__ushort_as_half(sreg[j]));
  }
}
// The first register batch is stored; longer K ranges load and store the rest.
template <int NB>
__device__ __forceinline__ void gd_finish_scales(const GdParams& p, const GdGeom& g, int lane,
                                                 const uint16_t (&sreg)[kGdSpl], float* scl) {
  if (!g.busy) return;
  gd_store_scales<NB>(p, g, 0, lane, sreg, scl);
  const int nscl = (8 * g.tw) << p.lgGw;
  for (int base = 32 * kGdSpl; base < nscl; base += 32 * kGdSpl) {
    uint16_t r2[kGdSpl];
    gd_load_scales<NB>(p, g, base, lane, r2);
    gd_store_scales<NB>(p, g, base, lane, r2, scl);
  }
}

// The CTA's activations -> digit scratch.  Unit = (set, group j, batch b):
// 8 lanes x 16 elements; 4 units per warp per pass, two passes in flight.
// bf16 x (optionally times the fp16 column diagonal, exact in fp32) or fp32 x
// (read through L2: it may have been written by other CTAs of this grid).
// Unit u of this CTA -> this lane's 16 values (+ diagonal); zeros past the end.
template <int NB, bool XF32>
__device__ __forceinline__ void gd_load_unit(const GdParams& p, const GdGeom& g, int u, int sub, uint4 (&r)[4]) {
  constexpr int G = gd::Cfg<NB>::G;
  const int units = g.nsc * G * NB;
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] = make_uint4(0, 0, 0, 0);
  if (u < units) {
    const int sl = u / (G * NB), gb = u - sl * (G * NB);
    const int gj = gb / NB, b = gb - gj * NB;
    const int gi = (g.cs0 + sl) * G + gj;
    if (gi < p.NG) {
      const int64_t k0 = static_cast<int64_t>(gi) * 128 + sub * 16;
      const int64_t xr = p.xrows ? p.xrows[b] : b;
      if (XF32) {
        const uint4* src =
            reinterpret_cast<const uint4*>(static_cast<const float*>(p.x) + xr * p.K + k0);
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] = __ldcg(src + i);
      } else {
        const uint4* src =
            reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + xr * p.K + k0);
        r[0] = __ldg(src);
        r[1] = __ldg(src + 1);
        if (p.cdiag) {
          const uint4* dg = reinterpret_cast<const uint4*>(p.cdiag + k0);
          r[2] = __ldg(dg);
          r[3] = __ldg(dg + 1);
        }
      }
    }
  }
}

// The loads of this warp's first unit (split from the loop so that a caller
// can place them among its other copies).
template <int NB, bool XF32>
__device__ __forceinline__ void gd_x_first(const GdParams& p, const GdGeom& g, int warp, int lane, uint4 (&xa)[4]) {
  gd_load_unit<NB, XF32>(p, g, warp * 4 + (lane >> 3), lane & 7, xa);
}

// xa: this lane's first unit, from gd_x_first.
template <int NB, bool XF32, int NW = gd::kWarps>
__device__ __forceinline__ void gd_prep_x(const GdParams& p, const GdGeom& g, uint32_t* xs, int warp, int lane,
                                          uint4 (&xa)[4]) {
  using C = gd::Cfg<NB>;
  constexpr int G = C::G;
  const int units = g.nsc * G * NB;
  const int sub = lane & 7;
  auto load_unit = [&](int u, uint4 (&r)[4]) { gd_load_unit<NB, XF32>(p, g, u, sub, r); };
  auto process = [&](const uint4 (&r)[4], int u) {
    float v[16];
    if (XF32) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[4 * i] = __uint_as_float(r[i].x);
        v[4 * i + 1] = __uint_as_float(r[i].y);
        v[4 * i + 2] = __uint_as_float(r[i].z);
        v[4 * i + 3] = __uint_as_float(r[i].w);
      }
    } else {
      const uint32_t w[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
      if (p.cdiag) {
        const uint32_t d[8] = {r[2].x, r[2].y, r[2].z, r[2].w, r[3].x, r[3].y, r[3].z, r[3].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&d[i]));
          v[2 * i] *= f.x;  // bf16 x fp16: exact in fp32
          v[2 * i + 1] *= f.y;
        }
      }
    }
    const int sl = u / (G * NB);
    const int it = (u - sl * (G * NB)) * 8 + sub;  // item index within the set
    quantise_item<NB>(v, u < units, it, xs + sl * C::SCR);
  };
  constexpr int kPass = 4 * NW;  // units per pass of the CTA
  const int u0 = warp * 4 + (lane >> 3);
  uint4 xb[4];
  for (int u = u0; u - u0 < units; u += 2 * kPass) {  // trip count uniform over the CTA
    load_unit(u + kPass, xb);
    process(xa, u);
    if (u - u0 + kPass >= units) break;
    load_unit(u + 2 * kPass, xa);
    process(xb, u + kPass);
  }
}

// Products, CTA reduction, cluster reduction and output:
// y[b][row] = rdiag[row] * sum.  Call after the weights, scales and digits are
// in shared memory (and a __syncthreads).  `wait_cluster`: wait on the
// cluster barrier arrived at kernel entry before the first remote store.
template <int NB, int NW = gd::kWarps>
__device__ __forceinline__ void gd_finish(const GdParams& p, const GdGeom& g, const unsigned char* wts,
                                          const float* scl, const uint32_t* xs, float* red, float* part, int warp,
                                          int lane, bool wait_cluster) {
  using C = gd::Cfg<NB>;
  constexpr int NN = C::NN, NCOL = C::NCOL;
  const int sstride = 8 * p.Tw;
  float acc[gd::kMaxTp][NN][4];
#pragma unroll
  for (int tp = 0; tp < gd::kMaxTp; ++tp)
#pragma unroll
    for (int nn = 0; nn < NN; ++nn)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tp][nn][e] = 0.f;
  if (g.busy) {
    const uint32_t* xw = xs + (g.ws0 - g.cs0) * C::SCR;
    switch (g.tw) {  // warp-uniform
      case 1: gd_compute<NB, 1>(wts, p.P, scl, sstride, xw, g.nsw, lane, acc); break;
      case 2: gd_compute<NB, 2>(wts, p.P, scl, sstride, xw, g.nsw, lane, acc); break;
      case 3: gd_compute<NB, 3>(wts, p.P, scl, sstride, xw, g.nsw, lane, acc); break;
      default: gd_compute<NB, 4>(wts, p.P, scl, sstride, xw, g.nsw, lane, acc); break;
    }
  }
  // ---- CTA reduction buffer: red[wg * GS + (tile * 8 + row) * NCOL + column],
  // tile = wn * Tw + t (CTA-local); GS is odd so that the warp blocks spread
  // over the banks.
  const int r1 = lane >> 2, cq = lane & 3;
  const int GS = p.Wn * p.Tw * C::RED + 1;
  if (p.alias_red) __syncthreads();  // every warp is done reading the activation scratch
  {
    float* wr = red + g.wg * GS + (g.wn * p.Tw * 8 + r1) * NCOL;
#pragma unroll
    for (int tp = 0; tp < gd::kMaxTp; ++tp)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 2 * tp + (e >> 1);
        if (t < g.tw) {
#pragma unroll
          for (int nn = 0; nn < NN; ++nn) {
            const int n = 8 * nn + 2 * cq + (e & 1);
            if (n < NCOL) wr[t * 8 * NCOL + n] = acc[tp][nn][e];
          }
        }
      }
  }
  __syncthreads();
  // Output o = (row rl of this cluster, batch b), o = rl * NB + b: T threads
  // each sum the three digit columns of b over every T-th warp block (fixed
  // order; blocks without sets wrote nothing and are skipped), then a T-lane
  // butterfly.  The sum goes to the owning CTA (or straight to y when S = 1).
  const int R8 = 8 * g.Tq, O = NB * R8;
  int lgT = 0;
  while (lgT < p.lgWg && (O << (lgT + 1)) <= NW * 32) ++lgT;
  const int T = 1 << lgT, j = threadIdx.x & (T - 1);
  if (p.S > 1 && wait_cluster) cluster_wait();  // every CTA of the cluster has started
  for (int o0 = 0; o0 < O; o0 += NW * 32 >> lgT) {  // trip count uniform over the CTA
    const int o = o0 + (threadIdx.x >> lgT);
    const int rl = o / NB, b = o - rl * NB;
    float sum = 0.f;
    if (o < O) {
      const float* rp = red + rl * NCOL + 3 * b;
      for (int g2 = j; g2 < p.Wg; g2 += T) {
        if ((((g2 + 1) * g.nsc) >> p.lgWg) <= ((g2 * g.nsc) >> p.lgWg)) continue;
        const float* q = rp + g2 * GS;
        sum += (q[0] + q[1]) + q[2];
      }
    }
    for (int m = 1; m < T; m <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, m);
    if (o < O && j == 0) {
      const int row = g.t0c * 8 + rl;
      if (p.S == 1) {
        if (row < p.N)
          p.y[static_cast<int64_t>(b) * p.N + row] = p.rdiag ? __half2float(__ushort_as_half(p.rdiag[row])) * sum : sum;
      } else {
        int owner = 0;
        while (owner + 1 < p.S && rl >= (owner + 1) * p.chunk) ++owner;
        const uint32_t local = smem_u32(part + (g.crank * NB + b) * p.chunk + (rl - owner * p.chunk));
        st_dsmem_f32(map_shared_rank(local, static_cast<uint32_t>(owner)), sum);
      }
    }
  }
  if (p.S > 1) {
    cluster_sync();
    const int lo = g.crank * p.chunk, cnt = max(0, min(R8, lo + p.chunk) - lo);
    for (int i = threadIdx.x; i < NB * cnt; i += NW * 32) {
      const int ro = i / NB, b = i - ro * NB;
      float sum = 0.f;
      for (int c = 0; c < p.S; ++c) sum += part[(c * NB + b) * p.chunk + ro];
      const int row = g.t0c * 8 + lo + ro;
      if (row < p.N)
        p.y[static_cast<int64_t>(b) * p.N + row] = p.rdiag ? __half2float(__ushort_as_half(p.rdiag[row])) * sum : sum;
    }
  }
}

template <int NB, int NW>
__global__ void __launch_bounds__(NW * 32, 1) gemv_direct_kernel(const GdParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const GdSmem L = gd_layout<NB, NW>(p.Tw, p.NSw, p.P, p.S, p.chunk, p.NSc, p.alias_red != 0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wreg = smem + warp * L.warp_bytes;
  unsigned char* wts = wreg + L.wts;
  float* scl = reinterpret_cast<float*>(wreg + L.scl);
  uint32_t* xs = reinterpret_cast<uint32_t*>(smem + L.xs);
  if (p.S > 1) cluster_arrive_relaxed();  // matched by the wait before the first remote store
  const GdGeom g = gd_geom<NB>(p, warp);
  uint16_t sreg[kGdSpl];
  if (p.early) {
    if (g.busy) gd_stage<NB>(p, g, wts, lane);
    gd_load_scales<NB>(p, g, 0, lane, sreg);
  }
  pdl_wait();
  pdl_launch_dependents();
  if (!p.early) {
    if (g.busy) gd_stage<NB>(p, g, wts, lane);
    gd_load_scales<NB>(p, g, 0, lane, sreg);
  }
  uint4 xa[4];  // after the weight copies: the weights are the longer path
  if (p.x_f32) gd_x_first<NB, true>(p, g, warp, lane, xa);
  else gd_x_first<NB, false>(p, g, warp, lane, xa);
  if (p.x_f32) gd_prep_x<NB, true, NW>(p, g, xs, warp, lane, xa);
  else gd_prep_x<NB, false, NW>(p, g, xs, warp, lane, xa);
  gd_finish_scales<NB>(p, g, lane, sreg, scl);
  cp_async_wait_all();
  __syncthreads();
  gd_finish<NB, NW>(p, g, wts, scl, xs, reinterpret_cast<float*>(smem + L.red),
                    reinterpret_cast<float*>(smem + L.part), warp, lane, true);
}

// ------------------------------------------------------------------ host side

template <int NB, int NW>
static int gd_max_clusters(int S, int smem_bytes) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(S * 64));
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S > 1 ? 1 : 0;
  int n = 0;
  if (ensure_dyn_smem(reinterpret_cast<const void*>(gemv_direct_kernel<NB, NW>), smem_bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (S > 1) {
    if (cudaOccupancyMaxActiveClusters(&n, gemv_direct_kernel<NB, NW>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return n;
  }
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_direct_kernel<NB, NW>, NW * 32, smem_bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;  // per SM
}

struct GdPlan {
  int S, Q, Wn, Wg, Tw, NSw, NSc, P, chunk, smem, alias_red;
  double cost;
};

// Instruction-count model per SM (lane instructions / 128 per clock):
// activation quantisation ~24 per element of the CTA's K range (its chain is
// latency-bound; fitted to measured K splits), weights ~c_w
// per weight, CTAs per SM rounded up, plus a fixed charge for a cluster
// barrier.
template <int NB, int NW>
static bool gd_plan_for(int N, int NG, int S, int num_sms, int smem_cap, GdPlan* out) {
  using C = gd::Cfg<NB>;
  const int NT = (N + 7) / 8;
  const int NS = (NG + C::G - 1) / C::G;
  if (S > 1 && S > NS) return false;
  const int nsc = (NS + S - 1) / S;
  if (nsc > gd::kMaxSets) return false;
  int Q = std::max(1, std::min(NT, num_sms / S));
  for (int iter = 0; iter < 8; ++iter) {
    const int Tmax = (NT + Q - 1) / Q;
    int Wn = 0;
    for (int w = 1; w <= NW; w *= 2)
      if ((Tmax + w - 1) / w <= gd::kMaxTw) {
        Wn = w;
        break;
      }
    if (Wn == 0) {  // more rows per cluster than the warps' n-tiles: more clusters
      Q = (NT + NW * gd::kMaxTw - 1) / (NW * gd::kMaxTw);
      continue;
    }
    const int Wg = NW / Wn;
    const int Tw = (Tmax + Wn - 1) / Wn;
    const int NSw = (nsc + Wg - 1) / Wg;
    const int span = NSw * 16 * C::G;
    const int P = ((span / (16 * C::G)) & 1) ? span : span + 16 * C::G;  // odd multiple: bank spread
    const int chunk = (8 * Tmax + S - 1) / S;
    GdSmem L = gd_layout<NB, NW>(Tw, NSw, P, S, chunk, nsc);
    int alias_red = 0;
    if (L.total > smem_cap) {  // first the reduction buffer over the activation scratch
      L = gd_layout<NB, NW>(Tw, NSw, P, S, chunk, nsc, true);
      alias_red = 1;
    }
    if (L.total > smem_cap) {
      if (Q >= NT) return false;
      Q = std::min(NT, Q * 2);  // fewer rows per CTA
      continue;
    }
    const int occ = gd_max_clusters<NB, NW>(S, L.total);
    if (occ <= 0) return false;
    const double cw = NB <= 2 ? 0.35 : (NB <= 5 ? 1.0 : 1.2);
    const double xprep = 24.0 * NB * 128.0 * C::G * nsc;          // per CTA
    const double wts = 8.0 * Tmax * 128.0 * C::G * nsc * cw;      // per CTA
    const double ctas_per_sm = std::ceil(static_cast<double>(Q) * S / num_sms);
    const double cost = (xprep + wts) / 128.0 * ctas_per_sm + (S > 1 ? 800.0 : 0.0);
    *out = GdPlan{S, Q, Wn, Wg, Tw, NSw, nsc, P, chunk, L.total, alias_red, cost};
    return true;
  }
  return false;
}

struct GdPlanEntry {
  int N, NG, NB, NW, sms, dev, force;
  bool ok;
  GdPlan plan;
};
static GdPlanEntry g_gd_cache[64];
static int g_gd_count = 0;
static std::mutex g_gd_mu;

template <int NB, int NW>
static bool gd_cached_plan(int N, int NG, int num_sms, int smem_cap, int force_s, GdPlan* out) {
  int force = force_s;
  if (!force)
    force = knob(kKnobGemvSplit);  // tuning knob: force the K split
  if (force != 1 && force != 2 && force != 4 && force != 8) force = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(g_gd_mu);
    for (int i = 0; i < g_gd_count; ++i) {
      const GdPlanEntry& e = g_gd_cache[i];
      if (e.N == N && e.NG == NG && e.NB == NB && e.NW == NW && e.sms == num_sms && e.dev == dev &&
          e.force == force) {
        *out = e.plan;
        return e.ok;
      }
    }
  }
  GdPlan best = {};
  bool ok = false;
  for (int S = 1; S <= 8; S *= 2) {
    if (force && S != force) continue;
    GdPlan pl;
    if (gd_plan_for<NB, NW>(N, NG, S, num_sms, smem_cap, &pl) && (!ok || pl.cost < best.cost)) {
      best = pl;
      ok = true;
    }
  }
  std::lock_guard<std::mutex> lock(g_gd_mu);
  const int i = g_gd_count < 64 ? g_gd_count++ : (N + NG + NB) & 63;
  g_gd_cache[i] = GdPlanEntry{N, NG, NB, NW, num_sms, dev, force, ok, best};
  *out = best;
  return ok;
}

template <int NB, int NW>
static cudaError_t launch_gemv_direct_nb(const GdParams& base, cudaStream_t stream, int num_sms, int smem_cap,
                                         int force_s) {
  GdPlan plan;
  if (!gd_cached_plan<NB, NW>(base.N, base.NG, num_sms, smem_cap, force_s, &plan)) return cudaErrorNotSupported;
  if (knob(kKnobVerbose))
    fprintf(stderr,
            "w1_gemv(direct) plan: N=%d NG=%d B=%d warps=%d -> clusters=%d split=%d warps=%dx%d tiles/warp=%d "
            "sets/warp=%d smem=%d\n",
            base.N, base.NG, NB, NW, plan.Q, plan.S, plan.Wn, plan.Wg, plan.Tw, plan.NSw, plan.smem);

  GdParams p = base;
  p.S = plan.S;
  p.Q = plan.Q;
  p.NT = (base.N + 7) / 8;
  p.Wn = plan.Wn;
  p.Wg = plan.Wg;
  p.Tw = plan.Tw;
  p.NSw = plan.NSw;
  p.P = plan.P;
  p.chunk = plan.chunk;
  p.NSc = plan.NSc;
  p.alias_red = plan.alias_red;
  auto lg2 = [](int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
  };
  p.lgS = lg2(plan.S);
  p.lgWg = lg2(plan.Wg);
  p.lgGw = lg2(plan.NSw * gd::Cfg<NB>::G);
  p.tq = p.NT / plan.Q;
  p.tr = p.NT - p.tq * plan.Q;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(gemv_direct_kernel<NB, NW>), plan.smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.Q * plan.S));
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (plan.S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(plan.S);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, gemv_direct_kernel<NB, NW>, p);
}

// Returns cudaErrorNotSupported when the shape is outside this kernel's plan
// (or outside the plan with the forced K split force_s; 0 = planner's choice).
// warps: 8 or 16 per CTA.
template <int NW>
static cudaError_t launch_gemv_direct_nw(const GdParams& p, int B, cudaStream_t stream, int num_sms, int smem_cap,
                                         int force_s) {
  switch (B) {
    case 1: return launch_gemv_direct_nb<1, NW>(p, stream, num_sms, smem_cap, force_s);
    case 2: return launch_gemv_direct_nb<2, NW>(p, stream, num_sms, smem_cap, force_s);
    case 3: return launch_gemv_direct_nb<3, NW>(p, stream, num_sms, smem_cap, force_s);
    case 4: return launch_gemv_direct_nb<4, NW>(p, stream, num_sms, smem_cap, force_s);
    case 5: return launch_gemv_direct_nb<5, NW>(p, stream, num_sms, smem_cap, force_s);
    case 6: return launch_gemv_direct_nb<6, NW>(p, stream, num_sms, smem_cap, force_s);
    case 7: return launch_gemv_direct_nb<7, NW>(p, stream, num_sms, smem_cap, force_s);
    default: return launch_gemv_direct_nb<8, NW>(p, stream, num_sms, smem_cap, force_s);
  }
}

// x is bf16 [B][K], or fp32 [B][K] when x_f32.
cudaError_t launch_gemv_direct(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                               const void* x, bool x_f32, int B, float* y, bool static_weights,
                               cudaStream_t stream, int num_sms, int smem_cap, int force_s, int warps) {
  if (N > (int64_t)1 << 30 || K > (int64_t)1 << 30) return cudaErrorNotSupported;
  GdParams p = {};
  p.signs = signs;
  p.scales = scales;
  p.x = x;
  p.y = y;
  p.x_f32 = x_f32 ? 1 : 0;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.NG = static_cast<int>(K / 128);
  p.early = static_weights ? 1 : 0;
  // A 16-warp CTA never shares an SM with the next launch's CTA (registers),
  // so its plans may use up to twice the shared memory cap of 8-warp plans.
  if (warps == 16)
    return launch_gemv_direct_nw<16>(p, B, stream, num_sms, std::min(2 * smem_cap, 200 * 1024), force_s);
  return launch_gemv_direct_nw<8>(p, B, stream, num_sms, smem_cap, force_s);
}

// One product with diagonals and no group scales (a step of the DBF chain):
// y[b][row] = rdiag[row] * sum_k s(row, k) * cdiag[k] * x[b][k], cdiag only
// for bf16 x (nullptr: none).  early: the sign words were not written by the
// kernel this launch follows (they may be read before its grid dependency
// wait).  force_s: CTAs per cluster splitting K (0 = planner).  Same
// planning and kernels as launch_gemv_direct.
cudaError_t launch_gemv_direct_diag(const uint32_t* signs, int64_t N, int64_t K, const void* x, bool x_f32,
                                    const uint16_t* cdiag, const uint16_t* rdiag, int B, float* y, bool early,
                                    cudaStream_t stream, int num_sms, int smem_cap, int warps, int force_s) {
  if (N > (int64_t)1 << 30 || K > (int64_t)1 << 30 || (x_f32 && cdiag)) return cudaErrorNotSupported;
  GdParams p = {};
  p.signs = signs;
  p.scales = nullptr;
  p.x = x;
  p.y = y;
  p.x_f32 = x_f32 ? 1 : 0;
  p.cdiag = cdiag;
  p.rdiag = rdiag;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.NG = static_cast<int>(K / 128);
  p.early = early ? 1 : 0;
  if (warps == 16)
    return launch_gemv_direct_nw<16>(p, B, stream, num_sms, std::min(2 * smem_cap, 200 * 1024), force_s);
  return launch_gemv_direct_nw<8>(p, B, stream, num_sms, smem_cap, force_s);
}

}  // namespace w1

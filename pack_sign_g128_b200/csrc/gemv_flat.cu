// w1_gemv, the register-fed decode kernel (bf16 activations, 1 <= B <= 8).
//
//   y[b,n] = sum_g s[n,g] * sum_{k in g} (1 - 2 bit[n,k]) x[b,k]
//
// Storage format: "1-bit group-128 sign packing" (one sign bit per weight,
// LSB-first in uint32 words along K, one fp16 mean|w| scale per 128 weights);
// generation multiplies one vector (or a few) by every weight once ("LLM
// binarization episode 01: DBF", section 4), so the kernel is built around
// the latency of one pass over the packed bytes.
//
// On this GPU a warp-level MMA (mma.sync) runs at its issue rate only when its
// operands come from registers: fed from shared memory at every MMA it is
// several times slower.  And many small per-lane loads of the sign words
// exhaust the SM's outstanding-request capacity.  So the sign words arrive
// by a few 2-D TMA boxes per CTA (8 groups x R rows each, 128-byte swizzle,
// each on its own mbarrier, issued right after the grid dependency wait, or
// before it with W1_GEMV_STATIC_WEIGHTS), and each warp then copies exactly
// the words its MMA fragments need into registers in one batch (the swizzle
// makes those reads bank-conflict free) and expands them there.
//
// Work split.  A CTA (one per SM) owns R = 16 T consecutive weight rows and a
// K range (all of K, or 1/S of it when S CTAs of a thread-block cluster split
// K and meet in distributed shared memory).  Its warps split that K range by
// groups; every warp runs all R rows over its groups, and no warp waits for
// another until the final reduction.  A warp loads (and, for B <= 2,
// quantises) its activations while the boxes land, then runs its groups in
// order; the T tiles of a group are independent accumulator chains.
//
// Two arithmetic forms, chosen by the batch size (both exact up to the f32
// accumulation and fold):
//  * B <= 2, int8: the activations of each (batch row, group) become 23-bit
//    fixed point (scaled by 2^(22-E), E from the group maximum) in three
//    signed 8-bit digits; the weights are the bytes -bit (0 or -1), one PRMT
//    per 4 weights; mma.sync m16n8k32 s8 with the digit columns 3b + d; per
//    group  sum (1-2 bit) q = X + 2 sum_d W_d C_d  (W = 2^16, 2^8, 1; X =
//    sum q) is folded with the scale.  Quantisation error <= 2^(E-23) per
//    element, far inside the 1e-3 * sum |s x| tolerance.
//  * B >= 3, bf16: the batch rows are the MMA columns (one 8-column n-tile),
//    the activations enter unchanged, the weights become bf16 +-1 pairs
//    (one shift and one LOP3 per two weights); mma.sync m16n8k16 bf16 -> f32;
//    the group scale multiplies each group's f32 partial sums.
// The diagonal form (a step of the DBF chain: fp32 or diagonal-scaled input,
// no group scales, a row diagonal on the outputs) feeds the int8 digits from
// the fp32 values for B <= 2, and for B = 3, 4 splits each fp32 value into
// bf16 high and low parts, two MMA columns per batch row (error 2^-17 |v|).
// K order inside one MMA is free as long as A and B agree; the activation
// values are placed in the order the sign-bit extraction produces, and the
// canonical weight bytes are read unchanged.
#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <mutex>
#include <type_traits>

#include "w1_common.cuh"

namespace w1 {

namespace fl {
constexpr int kMaxBox = 48;  // TMA boxes (8 groups each) per CTA
constexpr int kBoxG = 8;     // groups per box (128 bytes of sign words per row)
template <int NB, bool DIAG = false>
struct Cfg {
  static constexpr bool BF = NB >= 3;  // bf16 products, batch rows as the MMA columns
  // result columns per row: int8 digits 3 per batch row; bf16 one per batch
  // row, or two (the bf16 high and low parts of an fp32 input) in the diagonal form
  static constexpr int NCOL = BF ? (DIAG ? 2 * NB : NB) : 3 * NB;
  static_assert(NCOL <= 8, "one 8-column n-tile");
  static constexpr int MAXT = 8;                 // 16-row tiles per CTA (R <= 128)
  static constexpr int UPL = 2;                  // int8 form: activation units per lane and pass
  static constexpr int GW = BF ? 0 : 4 * 64;     // int8 form: digit words per group (4 MMAs x 32 lanes x 2)
};
}  // namespace fl

struct FlParams {
  const uint32_t* signs;   // [N][K/32]
  const uint16_t* scales;  // fp16 [N][NG]
  const uint16_t* x;       // bf16 [B][K]
  float* y;                // [B][N]
  int N, K, NG;
  int S;      // CTAs per cluster (K split)
  int R, T;   // rows per CTA (16 T)
  int G;      // groups per CTA (the last CTA of a cluster may have fewer)
  int gw;     // max groups per warp
  int chunk;  // rows owned per CTA in the cluster reduction
  int early;  // read weights before the grid dependency wait
  // diagonal form (a step of the DBF chain; no group scales):
  // y[b][n] = rdiag[n] * sum_k s(n, k) * (cdiag[k] *) x[b][k]
  const uint16_t* cdiag;  // fp16 [K], bf16 x only, or nullptr
  const uint16_t* rdiag;  // fp16 [N], or nullptr
  int x_f32;              // x is fp32 [B][K]
};

struct FlSmem {
  int wts, dig, red, scl, fold, inbox, total;
};

// Shared memory from a 1024-byte aligned base: the swizzled sign boxes, the
// digit buffers (int8 form; the reduction buffer overlays them), the scales,
// the fold factors, the cluster inbox.
template <int NB, int NW, bool DIAG>
__host__ __device__ inline FlSmem fl_layout(int R, int G, int gw, int NG, int S, int chunk) {
  using C = fl::Cfg<NB, DIAG>;
  FlSmem L;
  const int nbox = (G + fl::kBoxG - 1) / fl::kBoxG;
  const int dig_bytes = NW * gw * C::GW * 4;
  const int red_bytes = NW * R * C::NCOL * 4;
  L.wts = 0;  // boxes of R x 128 bytes (R a multiple of 16: each box stays 1024-byte aligned)
  L.dig = nbox * R * 128;
  L.red = L.dig;  // the reduction buffer overlays the digits (written after every warp's last MMA)
  L.scl = L.dig + ((dig_bytes > red_bytes ? dig_bytes : red_bytes) + 15) / 16 * 16;  // [R][NG] fp16
  L.fold = L.scl + ((R * NG * 2 + 15) / 16) * 16;
  L.inbox = L.fold + (C::BF ? 0 : NW * gw * NB * 4 * 4);
  L.total = L.inbox + (S > 1 ? S * NB * chunk * 4 : 0);
  return L;
}

// -(bit q + 4i of w), i = 0..3, as int8 bytes (0 or -1); q in 0..7 (4..7: upper half).
template <int Q>
__device__ __forceinline__ uint32_t fl_sign_s8(uint32_t w) {
  if constexpr (Q == 0) return prmt(0xFF00FF00u, 0xFF00FF00u, w);
  else if constexpr (Q == 1) return prmt(0xFFFF0000u, 0xFFFF0000u, w);
  else if constexpr (Q == 2) return prmt(0x00000000u, 0xFFFFFFFFu, w);
  else if constexpr (Q == 3) return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 3);
  else if constexpr (Q == 4) return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 16);
  else if constexpr (Q == 5) return prmt(0xFFFF0000u, 0xFFFF0000u, w >> 16);
  else if constexpr (Q == 6) return prmt(0x00000000u, 0xFFFFFFFFu, w >> 16);
  else return prmt(0xFF00FF00u, 0xFF00FF00u, w >> 19);
}

// bf16 +-1 pair: bit 15 - SHL of w -> sign of the low half, bit 31 - SHL ->
// sign of the high half (bit = 1 means -1).
template <int SHL>
__device__ __forceinline__ uint32_t fl_sign_bf16(uint32_t w) {
  return ((w << SHL) & 0x80008000u) | 0x3F803F80u;
}

__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bounded mbarrier wait of a whole warp (all lanes leave together).
__device__ __forceinline__ bool fl_wait(uint64_t* bar) { return mbar_wait_warp(bar, 0); }

// int8 form: one activation unit -- 16 consecutive bf16 values (elements 16h
// .. 16h+15 of word cq of a group) of batch row b -- to digit words.  For each
// MMA q the digit words of k-slots 4cq + i + 16h (elements q + 4i of the unit)
// go to column 3b + d (d = 0 hi, 1 mid, 2 lo) of the group's B fragments.
// Lanes of the 8-lane set of one (group, batch row) share the group maximum;
// lane (cq, h) == (0, 0) writes the fold factors f1, f2 (2^(E-22) = f1 f2)
// and X f (X = the sum of the group's 23-bit integers).
__device__ __forceinline__ void fl_quantise_values(const float (&v)[16], bool store, uint32_t* dig, float* fold,
                                                   int b, int cq, int h) {
  float m8[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) m8[j] = fmaxf(fabsf(v[2 * j]), fabsf(v[2 * j + 1]));
#pragma unroll
  for (int s = 4; s >= 1; s >>= 1)
#pragma unroll
    for (int j = 0; j < s; ++j) m8[j] = fmaxf(m8[j], m8[j + s]);
  float mx = m8[0];
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
  int E = 0;
  if (mx > 0.f) frexpf(mx, &E);  // mx = f 2^E, f in [0.5, 1): |x 2^(22-E)| < 2^22
  const int sf = 22 - E, sf1 = sf / 2, sf2 = sf - sf1;
  const float m1 = __uint_as_float(static_cast<uint32_t>(sf1 + 127) << 23);
  const float m2 = __uint_as_float(static_cast<uint32_t>(sf2 + 127) << 23);
  uint32_t e[16];
  int xs = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    // 0x4B400000 + round(x 2^sf): exact rounding to an integer for |x 2^sf| < 2^22
    const uint32_t bits = __float_as_uint(fmaf(v[i] * m1, m2, 12582912.0f));
    xs += static_cast<int>(bits - 0x4B400000u);
    e[i] = (bits - 0x4ABF7F80u) ^ 0x00808080u;  // bytes: signed digits lo, mid, hi
  }
  xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 1);
  xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 2);
  xs += __shfl_xor_sync(0xFFFFFFFFu, xs, 4);
  if (!store) return;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    // elements q, q+4, q+8, q+12 -> bytes 0..3 of the digit words
    const uint32_t e0 = e[q], e1 = e[q + 4], e2 = e[q + 8], e3 = e[q + 12];
    const uint32_t p01 = prmt(e0, e1, 0x5140u), p23 = prmt(e2, e3, 0x5140u);
    const uint32_t dlo = prmt(p01, p23, 0x5410u);
    const uint32_t dmid = prmt(p01, p23, 0x7632u);
    const uint32_t dhi = prmt(prmt(e0, e1, 0x0062u), prmt(e2, e3, 0x0062u), 0x5410u);
    uint32_t* base = dig + q * 64 + (3 * b * 4 + cq) * 2 + h;  // column 3b + d, word cq, half h
    base[0] = dhi;
    base[8] = dmid;
    base[16] = dlo;
  }
  if (cq == 0 && h == 0) {
    const float f1 = __uint_as_float(static_cast<uint32_t>(127 - sf1) << 23);
    const float f2 = __uint_as_float(static_cast<uint32_t>(127 - sf2) << 23);
    fold[b * 4 + 0] = f1;
    fold[b * 4 + 1] = f2;
    fold[b * 4 + 2] = (static_cast<float>(xs) * f1) * f2;
  }
}
__device__ __forceinline__ void fl_quantise_unit(const uint4 (&r)[2], bool store, uint32_t* dig, float* fold, int b,
                                                 int cq, int h) {
  const uint32_t w[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
  float v[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
  fl_quantise_values(v, store, dig, fold, b, cq, h);
}

// The warp's products over its groups for all T tiles of the CTA's rows,
// then (after a CTA barrier: the reduction buffer overlays the fragment
// buffers) its partial sums into red[warp][row][col].
//  1. int8 form: the activations of all the warp's groups are quantised into
//     its digit buffer in MMA fragment order.
//  2. Groups run GI at a time (GI T <= 8 accumulator chains), MMA steps
//     outermost, so consecutive MMAs never depend on each other; the bf16
//     form builds its B pairs from activations held in registers, the next
//     block's loads in flight.
// acc[t][e][c]: partial sum of row 16 t + lane/4 + 8 e, result column
// 2 (lane%4) + c (int8: digit column 3b + d, bf16: batch row).
// `prologue` is the grid dependency wait and what must follow it.
template <int NB, int NW, int T, bool DIAG, class Prologue>
__device__ __forceinline__ void fl_products(const FlParams& p, int row0, int g0, int G, int wg0, int nwg,
                                            const unsigned char* wts, uint64_t* bars, int nbox, uint32_t* dig,
                                            float* fold, const uint16_t* scl, uint64_t* sbar, int lane, float* red,
                                            Prologue&& prologue) {
  using C = fl::Cfg<NB, DIAG>;
  constexpr int STEPS = C::BF ? 8 : 4;            // MMAs per group and tile
  // groups per block: GI T <= 8 accumulator chains; the bf16 form also holds
  // two blocks' activations in registers (16 words per group), so it takes at
  // most 2 groups, 1 with 16 warps
  constexpr int GI0 = 8 / T >= 4 ? 4 : (8 / T >= 2 ? 2 : 1);
  constexpr int GI = C::BF ? (NW == 16 ? 1 : (GI0 > 2 ? 2 : GI0)) : GI0;
  float acc[T][2][2];
#pragma unroll
  for (int t = 0; t < T; ++t) acc[t][0][0] = acc[t][0][1] = acc[t][1][0] = acc[t][1][1] = 0.f;
  bool ok = true;
  const int r1 = lane >> 2, cq = lane & 3;
  prologue();
  // ---- 1. int8 form: activations -> digit fragments in shared memory
  if constexpr (DIAG && !C::BF) {
    // fp32 x (read through L2: the preceding launch wrote it), or bf16 x
    // times the column diagonal (exact in fp32)
    const int U = nwg * NB * 8;
    for (int u = lane; u - lane < U; u += 32) {  // trip count uniform over the warp
      const int gl = u / (8 * NB), b = (u >> 3) % NB, ucq = (u >> 1) & 3, h = u & 1;
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.f;
      if (u < U) {
        const int64_t k0 = static_cast<int64_t>(g0 + wg0 + gl) * 128 + 32 * ucq + 16 * h;
        if (p.x_f32) {
          const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.x) +
                                                              static_cast<int64_t>(b) * p.K + k0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 f = __ldcg(src + i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
          }
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(b) * p.K + k0);
          const uint4 r0 = __ldg(src), r1x = __ldg(src + 1);
          const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1x.x, r1x.y, r1x.z, r1x.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
          }
          if (p.cdiag) {
            const uint4* dg = reinterpret_cast<const uint4*>(p.cdiag + k0);
            const uint4 d0 = __ldg(dg), d1 = __ldg(dg + 1);
            const uint32_t dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&dd[j]));
              v[2 * j] *= f.x;  // bf16 x fp16: exact in fp32
              v[2 * j + 1] *= f.y;
            }
          }
        }
      }
      fl_quantise_values(v, u < U, dig + gl * C::GW, fold + gl * NB * 4, b, ucq, h);
    }
  } else if constexpr (!C::BF) {
    const int U = nwg * NB * 8;
    constexpr int UPL = C::UPL;
    uint4 xr[UPL][2];
    for (int u0 = 0; u0 < U; u0 += 32 * UPL) {  // trip count uniform over the warp
#pragma unroll
      for (int i = 0; i < UPL; ++i) {
        const int u = u0 + lane + 32 * i;
        const int gl = u / (8 * NB), b = (u >> 3) % NB, ucq = (u >> 1) & 3, h = u & 1;
        xr[i][0] = xr[i][1] = make_uint4(0, 0, 0, 0);
        if (u < U) {
          const uint4* src = reinterpret_cast<const uint4*>(
              p.x + static_cast<int64_t>(b) * p.K + static_cast<int64_t>(g0 + wg0 + gl) * 128 + 32 * ucq + 16 * h);
          xr[i][0] = __ldg(src);
          xr[i][1] = __ldg(src + 1);
        }
      }
#pragma unroll
      for (int i = 0; i < UPL; ++i) {
        if (u0 + 32 * i >= U) break;  // uniform: no lane of this slot has a unit
        const int u = u0 + lane + 32 * i;
        const int gl = u / (8 * NB), b = (u >> 3) % NB, ucq = (u >> 1) & 3, h = u & 1;
        fl_quantise_unit(xr[i], u < U, dig + gl * C::GW, fold + gl * NB * 4, b, ucq, h);
      }
    }
  }
  __syncwarp();  // fragment buffer and fold factors stored
  if (!(nwg == 0 || fl_wait(sbar))) ok = false;

  // int8 form: this lane's result columns 2cq + c are digit column 3b + d
  int cb[2], cd[2];
  float cw[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int col = 2 * cq + c;
    cb[c] = col < 3 * NB ? col / 3 : 0;
    cd[c] = col < 3 * NB ? col - 3 * cb[c] : 3;
    cw[c] = cd[c] == 0 ? 131072.f : (cd[c] == 1 ? 512.f : (cd[c] == 2 ? 2.f : 0.f));  // 2 W_d
  }
  // ---- 2. products, GI groups at a time
  // bf16 form: lane (r1, cq) holds batch row r1's 32 elements of word cq of
  // each group of a block (16 bf16x2 words), the next block's loads in flight.
  // Diagonal form: column r1 = 2 b + part holds the high (part 0) or low
  // (part 1) bf16 part of batch row b's fp32 input v = fp32 x or bf16 x times
  // the column diagonal: hi = bf16(v), lo = bf16(v - hi) (v - hi exact), so
  // hi + lo = v to 2^-17 |v|.
  auto load_x = [&](int gb, uint4 (&xv)[GI][4]) {
#pragma unroll
    for (int g = 0; g < GI; ++g) {
#pragma unroll
      for (int i = 0; i < 4; ++i) xv[g][i] = make_uint4(0, 0, 0, 0);
      if constexpr (C::BF && DIAG) {
        const int b = r1 >> 1;
        if (b < NB && gb + g < nwg) {
          const int64_t k0 = static_cast<int64_t>(g0 + wg0 + gb + g) * 128 + 32 * cq;
          float v[32];
          if (p.x_f32) {
            const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.x) +
                                                                static_cast<int64_t>(b) * p.K + k0);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 f = __ldcg(src + i);
              v[4 * i] = f.x;
              v[4 * i + 1] = f.y;
              v[4 * i + 2] = f.z;
              v[4 * i + 3] = f.w;
            }
          } else {
            const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(b) * p.K + k0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 u = __ldg(src + i);
              const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
              }
            }
            if (p.cdiag) {
              const uint4* dg = reinterpret_cast<const uint4*>(p.cdiag + k0);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint4 u = __ldg(dg + i);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
                  v[8 * i + 2 * j] *= f.x;  // bf16 x fp16: exact in fp32
                  v[8 * i + 2 * j + 1] *= f.y;
                }
              }
            }
          }
          const bool low = r1 & 1;
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float e[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float hi = __bfloat162float(__float2bfloat16_rn(v[2 * j + h]));
              e[h] = low ? v[2 * j + h] - hi : hi;
            }
            const __nv_bfloat162 pr = __floats2bfloat162_rn(e[0], e[1]);
            o[j] = *reinterpret_cast<const uint32_t*>(&pr);
          }
          xv[g][0] = make_uint4(o[0], o[1], o[2], o[3]);
          xv[g][1] = make_uint4(o[4], o[5], o[6], o[7]);
          xv[g][2] = make_uint4(o[8], o[9], o[10], o[11]);
          xv[g][3] = make_uint4(o[12], o[13], o[14], o[15]);
        }
      } else if (C::BF && r1 < NB && gb + g < nwg) {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.x + static_cast<int64_t>(r1) * p.K + static_cast<int64_t>(g0 + wg0 + gb + g) * 128 + 32 * cq);
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[g][i] = __ldg(src + i);
      }
    }
  };
  uint4 xcur[GI][4], xnext[GI][4];
  if constexpr (C::BF) load_x(0, xcur);
  int waited = -1;  // highest box this warp has waited for
  for (int gb = 0; gb < nwg; gb += GI) {
    // sign words of the block's groups: rows 16 t + r1 (+8), word cq, from the
    // swizzled boxes (each box waited for once)
    uint32_t W[GI][T][2];
#pragma unroll
    for (int g = 0; g < GI; ++g) {
      const int j = wg0 + gb + (gb + g < nwg ? g : 0);  // CTA-local group
      const int bx = min(j / fl::kBoxG, nbox - 1);
      while (waited < bx) {
        ++waited;
        if (!fl_wait(&bars[waited])) ok = false;
      }
      const int jj = j - (G >= fl::kBoxG ? min(bx * fl::kBoxG, G - fl::kBoxG) : 0);
      const unsigned char* wrow = wts + bx * p.R * 128 + r1 * 128 + ((jj ^ r1) << 4) + (cq << 2);
#pragma unroll
      for (int t = 0; t < T; ++t) {
        W[g][t][0] = *reinterpret_cast<const uint32_t*>(wrow + 16 * t * 128);
        W[g][t][1] = *reinterpret_cast<const uint32_t*>(wrow + (16 * t + 8) * 128);
      }
    }
    const int ng = min(GI, nwg - gb);
    if constexpr (C::BF) load_x(gb + GI, xnext);
    using Acc = typename std::conditional<C::BF, float, int>::type;
    Acc cc[GI][T][4];
#pragma unroll
    for (int g = 0; g < GI; ++g)
#pragma unroll
      for (int t = 0; t < T; ++t) cc[g][t][0] = cc[g][t][1] = cc[g][t][2] = cc[g][t][3] = 0;
    auto step = [&](auto mc) {
      constexpr int m = decltype(mc)::value;
      uint2 bb[GI];
#pragma unroll
      for (int g = 0; g < GI; ++g) {
        if constexpr (C::BF) {
          // elements (m, m+16) and (m+8, m+24) of the lane's word as the B pairs
          const uint32_t X[16] = {xcur[g][0].x, xcur[g][0].y, xcur[g][0].z, xcur[g][0].w,
                                  xcur[g][1].x, xcur[g][1].y, xcur[g][1].z, xcur[g][1].w,
                                  xcur[g][2].x, xcur[g][2].y, xcur[g][2].z, xcur[g][2].w,
                                  xcur[g][3].x, xcur[g][3].y, xcur[g][3].z, xcur[g][3].w};
          constexpr uint32_t sel = (m & 1) ? 0x7632u : 0x5410u;
          bb[g] = make_uint2(prmt(X[m / 2], X[8 + m / 2], sel), prmt(X[4 + m / 2], X[12 + m / 2], sel));
        } else {
          bb[g] = g < ng ? reinterpret_cast<const uint2*>(dig + (gb + g) * C::GW)[m * 32 + lane] : make_uint2(0, 0);
        }
      }
#pragma unroll
      for (int g = 0; g < GI; ++g)
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const uint32_t w0 = W[g][t][0], w1 = W[g][t][1];
          if constexpr (C::BF)
            mma_bf16(cc[g][t], fl_sign_bf16<15 - m>(w0), fl_sign_bf16<15 - m>(w1), fl_sign_bf16<7 - m>(w0),
                     fl_sign_bf16<7 - m>(w1), bb[g].x, bb[g].y);
          else
            mma_s8(cc[g][t], fl_sign_s8<m>(w0), fl_sign_s8<m>(w1), fl_sign_s8<m + 4>(w0), fl_sign_s8<m + 4>(w1),
                   bb[g].x, bb[g].y);
        }
    };
    step(std::integral_constant<int, 0>{});
    step(std::integral_constant<int, 1>{});
    step(std::integral_constant<int, 2>{});
    step(std::integral_constant<int, 3>{});
    if constexpr (C::BF) {
      step(std::integral_constant<int, 4>{});
      step(std::integral_constant<int, 5>{});
      step(std::integral_constant<int, 6>{});
      step(std::integral_constant<int, 7>{});
    }
    // fold
#pragma unroll
    for (int g = 0; g < GI; ++g) {
      if (g >= ng) break;
      const int gl = gb + g;
      const uint16_t* sg = scl + r1 * p.NG + g0 + wg0 + gl;
      if constexpr (C::BF) {
        // acc += s * C
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const float s0 = DIAG ? 1.f : __half2float(__ushort_as_half(sg[16 * t * p.NG]));
          const float s1 = DIAG ? 1.f : __half2float(__ushort_as_half(sg[(16 * t + 8) * p.NG]));
          acc[t][0][0] = fmaf(s0, cc[g][t][0], acc[t][0][0]);
          acc[t][0][1] = fmaf(s0, cc[g][t][1], acc[t][0][1]);
          acc[t][1][0] = fmaf(s1, cc[g][t][2], acc[t][1][0]);
          acc[t][1][1] = fmaf(s1, cc[g][t][3], acc[t][1][1]);
        }
      } else {
        // acc += s * (f1 f2 2 W_d C + [d = hi] f X)   (s = 1 in the diagonal form)
        float f1[2], f2[2], fx[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float* fb = fold + (gl * NB + cb[c]) * 4;
          f1[c] = fb[0];
          f2[c] = fb[1];
          fx[c] = cd[c] == 0 ? fb[2] : 0.f;
        }
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const float s0 = DIAG ? 1.f : __half2float(__ushort_as_half(sg[16 * t * p.NG]));
          const float s1 = DIAG ? 1.f : __half2float(__ushort_as_half(sg[(16 * t + 8) * p.NG]));
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            acc[t][0][c] = fmaf(s0, (cw[c] * static_cast<float>(cc[g][t][c]) * f1[c]) * f2[c] + fx[c], acc[t][0][c]);
            acc[t][1][c] =
                fmaf(s1, (cw[c] * static_cast<float>(cc[g][t][2 + c]) * f1[c]) * f2[c] + fx[c], acc[t][1][c]);
          }
        }
      }
    }
    if constexpr (C::BF) {
#pragma unroll
      for (int g = 0; g < GI; ++g)
#pragma unroll
        for (int k = 0; k < 4; ++k) xcur[g][k] = xnext[g][k];
    }
  }
  if (threadIdx.x < 32 && nwg == 0) fl_wait(sbar);  // the copy completes inside the CTA's lifetime
  __syncthreads();  // every warp is done with the fragment buffers the reduction overlays
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int col = 2 * cq + c;
      if (col < C::NCOL) {
        red[(warp * p.R + 16 * t + r1) * C::NCOL + col] = ok ? acc[t][0][c] : 0.f;
        red[(warp * p.R + 16 * t + r1 + 8) * C::NCOL + col] = ok ? acc[t][1][c] : 0.f;
      }
    }
}

template <int NB, int NW, bool DIAG = false>
__global__ void __launch_bounds__(NW * 32, 1) gemv_flat_kernel(const __grid_constant__ CUtensorMap tmap,
                                                               const FlParams p) {
  using C = fl::Cfg<NB, DIAG>;
  constexpr int NCOL = C::NCOL;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[fl::kMaxBox];  // the sign boxes
  __shared__ __align__(8) uint64_t sbar;               // the scales' bulk copy
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r1 = lane >> 2, cq = lane & 3;
  const int crank = p.S > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int q = p.S > 1 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int row0 = q * p.R;
  const int g0 = crank * p.G;
  const int G = max(0, min(p.NG, g0 + p.G) - g0);  // this CTA's groups
  const int rows = max(0, min(p.R, p.N - row0));   // this CTA's rows inside N
  const int nbox = (G + fl::kBoxG - 1) / fl::kBoxG;
  const FlSmem L = fl_layout<NB, NW, DIAG>(p.R, p.G, p.gw, p.NG, p.S, p.chunk);
  const unsigned char* wts = smem + L.wts;
  uint16_t* scl = reinterpret_cast<uint16_t*>(smem + L.scl);
  if (p.S > 1) cluster_arrive_relaxed();  // matched by the wait before the first remote store
  if (threadIdx.x == 0) {
    for (int b = 0; b < nbox; ++b) mbar_init(&bars[b], 1);
    mbar_init(&sbar, 1);
    fence_mbarrier_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap) : "memory");
  }
  __syncthreads();
  // The weight copies.  Box b holds CTA-local groups [bs, bs + 8), bs =
  // min(8 b, G - 8) (the last box overlaps its neighbour rather than reaching
  // past the CTA's range).  The scale block [rows][NG] is contiguous: one bulk
  // copy (a tail under 16 bytes, when rows * NG is not a multiple of 8, with
  // plain loads before the barrier arrival).
  auto issue = [&]() {
    if (threadIdx.x == 0) {
      for (int b = 0; b < nbox; ++b) {
        const int bs = G >= fl::kBoxG ? min(b * fl::kBoxG, G - fl::kBoxG) : 0;
        mbar_arrive_expect_tx(&bars[b], static_cast<uint32_t>(p.R * 128));
        tma_load_2d(smem + L.wts + b * p.R * 128, &tmap, (g0 + bs) * 4, row0, &bars[b]);
      }
      if (DIAG) {
        mbar_arrive(&sbar);  // no group scales
      } else {
        const uint32_t sbytes = static_cast<uint32_t>(rows) * p.NG * 2;
        const uint32_t sbulk = sbytes & ~15u;
        const uint16_t* ssrc = p.scales + static_cast<int64_t>(row0) * p.NG;
        for (uint32_t i = sbulk / 2; i < sbytes / 2; ++i) scl[i] = __ldg(ssrc + i);
        mbar_arrive_expect_tx(&sbar, sbulk);
        for (uint32_t off = 0; off < sbulk; off += 32768)
          bulk_g2s(reinterpret_cast<unsigned char*>(scl) + off, reinterpret_cast<const unsigned char*>(ssrc) + off,
                   min(32768u, sbulk - off), &sbar);
      }
    }
  };
  // The next launch in the stream may start now: its own grid dependency wait
  // orders everything it reads or writes after this grid.
  pdl_launch_dependents();
  if (p.early) issue();
  auto prologue = [&]() {
    pdl_wait();
    if (!p.early) issue();
  };
  // ---- this warp's groups [wg0, wg1) of the CTA's range
  const int wg0 = (warp * G) / NW, wg1 = ((warp + 1) * G) / NW, nwg = wg1 - wg0;
  uint32_t* dig = reinterpret_cast<uint32_t*>(smem + L.dig) + warp * p.gw * C::GW;
  float* fold = reinterpret_cast<float*>(smem + L.fold) + warp * p.gw * NB * 4;
  float* red = reinterpret_cast<float*>(smem + L.red);
  switch (p.T) {  // uniform over the grid
#define W1_FL_CASE(TV) \
  case TV:                                                                                                \
    fl_products<NB, NW, TV, DIAG>(p, row0, g0, G, wg0, nwg, wts, bars, nbox, dig, fold, scl, &sbar, lane, red, \
                                  prologue);                                                                   \
    break;
    W1_FL_CASE(1)
    W1_FL_CASE(2)
    W1_FL_CASE(3)
    W1_FL_CASE(4)
    W1_FL_CASE(5)
    W1_FL_CASE(6)
    W1_FL_CASE(7)
    W1_FL_CASE(8)
#undef W1_FL_CASE
    default:
      prologue();
      if (threadIdx.x < 32) {
        fl_wait(&sbar);
        for (int b = 0; b < nbox; ++b) fl_wait(&bars[b]);
      }
      __syncthreads();
      break;
  }
  __syncthreads();
  const int O = p.R * NB;
  float* inbox = reinterpret_cast<float*>(smem + L.inbox);
  if (p.S > 1) cluster_wait();  // every CTA of the cluster has started (its inbox exists)
  for (int o = threadIdx.x; o < O; o += NW * 32) {
    const int r = o / NB, b = o - r * NB;
    float sum = 0.f;
    if constexpr (C::BF && DIAG) {
#pragma unroll 4
      for (int w = 0; w < NW; ++w) {
        const float* rp = red + (w * p.R + r) * NCOL + 2 * b;
        sum += rp[0] + rp[1];
      }
    } else if constexpr (C::BF) {
#pragma unroll 4
      for (int w = 0; w < NW; ++w) sum += red[(w * p.R + r) * NCOL + b];
    } else {
#pragma unroll 4
      for (int w = 0; w < NW; ++w) {
        const float* rp = red + (w * p.R + r) * NCOL + 3 * b;
        sum += (rp[0] + rp[1]) + rp[2];
      }
    }
    if (p.S == 1) {
      // (with a K split the owner applies the row diagonal to the cluster's sum)
      if (DIAG && p.rdiag && row0 + r < p.N) sum *= __half2float(__ushort_as_half(p.rdiag[row0 + r]));
      if (row0 + r < p.N) p.y[static_cast<int64_t>(b) * p.N + row0 + r] = sum;
    } else {
      const int owner = r / p.chunk;
      const uint32_t local = smem_u32(inbox + (crank * NB + b) * p.chunk + (r - owner * p.chunk));
      st_dsmem_f32(map_shared_rank(local, static_cast<uint32_t>(owner)), sum);
    }
  }
  if (p.S > 1) {
    cluster_sync();
    const int lo = crank * p.chunk, cnt = max(0, min(p.R, lo + p.chunk) - lo);
    for (int i = threadIdx.x; i < NB * cnt; i += NW * 32) {
      const int ro = i / NB, b = i - ro * NB;
      float sum = 0.f;
      for (int c = 0; c < p.S; ++c) sum += inbox[(c * NB + b) * p.chunk + ro];
      const int row = row0 + lo + ro;
      if (DIAG && p.rdiag && row < p.N) sum *= __half2float(__ushort_as_half(p.rdiag[row]));
      if (row < p.N) p.y[static_cast<int64_t>(b) * p.N + row] = sum;
    }
  }
}

// ------------------------------------------------------------------ host side

// 2-D uint32 tensor map over the sign words [rows][words]: box {32 words, box_rows}
// (8 groups, 128 bytes per row), 128-byte swizzle, zero fill out of bounds.
bool make_tmap_u32_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t words, int box_rows);

struct FlPlan {
  int S, Q, R, T, G, gw, chunk, smem;
};

// Rows per CTA: the fewest 16-row tiles that cover N with at most one
// cluster of S CTAs per S SMs; groups per CTA: ceil(NG / S).
template <int NB, int NW, bool DIAG>
static bool fl_plan_for(int N, int NG, int S, int num_sms, int smem_cap, FlPlan* out) {
  using C = fl::Cfg<NB, DIAG>;
  if (S < 1 || S > 8 || S > NG) return false;
  const int tiles = (N + 15) / 16;
  const int qmax = num_sms / S;
  if (qmax < 1) return false;
  const int T = (tiles + qmax - 1) / qmax;
  if (T > C::MAXT) return false;
  const int R = 16 * T;
  const int Q = (tiles + T - 1) / T;
  const int G = (NG + S - 1) / S;
  if ((G + fl::kBoxG - 1) / fl::kBoxG > fl::kMaxBox) return false;
  const int gw = (G + NW - 1) / NW;
  const int chunk = (R + S - 1) / S;
  const FlSmem L = fl_layout<NB, NW, DIAG>(R, G, gw, NG, S, chunk);
  const int smem = L.total + 1024;  // alignment slack for the swizzled boxes
  if (smem > smem_cap) return false;
  *out = FlPlan{S, Q, R, T, G, gw, chunk, smem};
  return true;
}

template <int NB, int NW, bool DIAG = false>
static cudaError_t launch_gemv_flat_nb(const FlParams& base, cudaStream_t stream, int num_sms, int smem_cap, int S) {
  FlPlan plan;
  if (!fl_plan_for<NB, NW, DIAG>(base.N, base.NG, S, num_sms, smem_cap, &plan)) return cudaErrorNotSupported;
  if (knob(kKnobVerbose))
    fprintf(stderr, "w1_gemv(flat) plan: N=%d NG=%d B=%d warps=%d -> clusters=%d split=%d rows/CTA=%d smem=%d\n",
            base.N, base.NG, NB, NW, plan.Q, plan.S, plan.R, plan.smem);
  FlParams p = base;
  p.S = plan.S;
  p.R = plan.R;
  p.T = plan.T;
  p.G = plan.G;
  p.gw = plan.gw;
  p.chunk = plan.chunk;
  CUtensorMap tmap;
  if (!make_tmap_u32_sw128(&tmap, base.signs, base.N, base.K / 32, plan.R)) return cudaErrorInvalidValue;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(gemv_flat_kernel<NB, NW, DIAG>), plan.smem);
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
  return cudaLaunchKernelEx(&cfg, gemv_flat_kernel<NB, NW, DIAG>, tmap, p);
}

template <int NW>
static cudaError_t launch_gemv_flat_nw(const FlParams& p, int B, cudaStream_t stream, int num_sms, int smem_cap,
                                       int S) {
  switch (B) {
    case 1: return launch_gemv_flat_nb<1, NW>(p, stream, num_sms, smem_cap, S);
    case 2: return launch_gemv_flat_nb<2, NW>(p, stream, num_sms, smem_cap, S);
    case 3: return launch_gemv_flat_nb<3, NW>(p, stream, num_sms, smem_cap, S);
    case 4: return launch_gemv_flat_nb<4, NW>(p, stream, num_sms, smem_cap, S);
    case 5: return launch_gemv_flat_nb<5, NW>(p, stream, num_sms, smem_cap, S);
    case 6: return launch_gemv_flat_nb<6, NW>(p, stream, num_sms, smem_cap, S);
    case 7: return launch_gemv_flat_nb<7, NW>(p, stream, num_sms, smem_cap, S);
    default: return launch_gemv_flat_nb<8, NW>(p, stream, num_sms, smem_cap, S);
  }
}

// bf16 x [B][K] only.  split: CTAs per cluster along K (1, 2, 4 or 8; 0 = the
// smallest that fits); warps: 8 or 16 per CTA.  cudaErrorNotSupported when
// no plan fits.
cudaError_t launch_gemv_flat(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K, const uint16_t* x,
                             int B, float* y, bool static_weights, cudaStream_t stream, int num_sms, int smem_cap,
                             int split, int warps) {
  if (N > (int64_t)1 << 30 || K > (int64_t)1 << 30 || B < 1 || B > 8) return cudaErrorNotSupported;
  FlParams p = {};
  p.signs = signs;
  p.scales = scales;
  p.x = x;
  p.y = y;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.NG = static_cast<int>(K / 128);
  p.early = static_weights ? 1 : 0;
  // one CTA per SM: the plan may use up to twice the caller's cap (at most the
  // per-block opt-in maximum of an sm_100 SM)
  smem_cap = std::min(2 * smem_cap, 227 * 1024);
  for (int S = split > 0 ? split : 1; S <= 8; S *= 2) {
    const cudaError_t e = warps == 16 ? launch_gemv_flat_nw<16>(p, B, stream, num_sms, smem_cap, S)
                                      : launch_gemv_flat_nw<8>(p, B, stream, num_sms, smem_cap, S);
    if (e != cudaErrorNotSupported || split > 0) return e;
  }
  return cudaErrorNotSupported;
}

// The diagonal form (a step of the DBF chain, no group scales), 1 to 4 batch
// rows (1-2: int8 digits; 3-4: bf16 high and low parts of the fp32 input as
// two MMA columns per row): y[b][n] = rdiag[n] * sum_k s(n, k) * (cdiag[k] *) x[b][k], x bf16
// [B][K] (with the fp16 column diagonal cdiag, or nullptr) or fp32 [B][K]
// (x_f32; no cdiag); rdiag fp16 [N] or nullptr.  early: the sign words were
// not written by the kernel this launch follows.  split as for
// launch_gemv_flat; cudaErrorNotSupported when no plan fits.
cudaError_t launch_gemv_flat_diag(const uint32_t* signs, int64_t N, int64_t K, const void* x, bool x_f32,
                                  const uint16_t* cdiag, const uint16_t* rdiag, int B, float* y, bool early,
                                  cudaStream_t stream, int num_sms, int smem_cap, int split, int warps) {
  if (N > (int64_t)1 << 30 || K > (int64_t)1 << 30 || B < 1 || B > 4 || (x_f32 && cdiag))
    return cudaErrorNotSupported;
  FlParams p = {};
  p.signs = signs;
  p.scales = nullptr;
  p.x = static_cast<const uint16_t*>(x);
  p.y = y;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.NG = static_cast<int>(K / 128);
  p.early = early ? 1 : 0;
  p.cdiag = cdiag;
  p.rdiag = rdiag;
  p.x_f32 = x_f32 ? 1 : 0;
  smem_cap = std::min(2 * smem_cap, 227 * 1024);
  for (int S = split > 0 ? split : 1; S <= 8; S *= 2) {
    cudaError_t e;
    if (warps == 16) {
      switch (B) {
        case 1: e = launch_gemv_flat_nb<1, 16, true>(p, stream, num_sms, smem_cap, S); break;
        case 2: e = launch_gemv_flat_nb<2, 16, true>(p, stream, num_sms, smem_cap, S); break;
        case 3: e = launch_gemv_flat_nb<3, 16, true>(p, stream, num_sms, smem_cap, S); break;
        default: e = launch_gemv_flat_nb<4, 16, true>(p, stream, num_sms, smem_cap, S); break;
      }
    } else {
      switch (B) {
        case 1: e = launch_gemv_flat_nb<1, 8, true>(p, stream, num_sms, smem_cap, S); break;
        case 2: e = launch_gemv_flat_nb<2, 8, true>(p, stream, num_sms, smem_cap, S); break;
        case 3: e = launch_gemv_flat_nb<3, 8, true>(p, stream, num_sms, smem_cap, S); break;
        default: e = launch_gemv_flat_nb<4, 8, true>(p, stream, num_sms, smem_cap, S); break;
      }
    }
    if (e != cudaErrorNotSupported || split > 0) return e;
  }
  return cudaErrorNotSupported;
}

}  // namespace w1

// w1_moe_grouped: routed SwiGLU expert layer with 1-bit group-128 experts.
//
// For every token t: p = softmax(logits[t]) over E experts, the top_k
// experts by probability (ties to the lower index) are its routes; each route
// (t, e) computes h = silu(G_e x_t) * (U_e x_t) and out[t] += p_e * D_e h, the
// slot terms added in slot order.  "LLM binarization episode 01: DBF",
// section 4: every (token, slot) route carries an expert identity and a route
// weight; gate/up consume one hidden state shared by the selected experts,
// down consumes route-specific intermediates; section 5 items 8 and 10:
// expert-major compaction of route-specific inputs, shared gate/up inputs
// kept un-duplicated, fused SwiGLU, skipped empty tiles.
//
// Up to 8 tokens (the decode regime) the layer runs as per-route products:
// gate/up + SwiGLU (up to 4 tokens with the routing computed in each CTA,
// else after the router kernel) and down with the slot-ordered combine (see
// "decode regime" below); from 9 to 16 tokens as products grouped by expert
// (see "decode regime, grouped by expert").  Larger batches take the
// expert-sorted tile pipeline.
//
// Seven launches on one stream (programmatic dependent launch between them):
//  1. route_kernel     warp per token: fp32 softmax, top-k by logit, weights,
//                      and the token's fp16 multiplier (a power of two).
//  2. sort_kernel      one CTA: stable counting sort of the routes by expert
//                      (deterministic), route -> sorted position map, and the
//                      tile lists of the two grouped GEMMs (no empty tiles).
//  3. gather_kernel    x rows in expert-sorted route order as fp16, scaled by
//                      the token's power of two (max |x| in [2^14, 2^15)).
//  4. moe_gemm<GATEUP> tcgen05 grouped GEMM, swap-AB as in w1_gemm: the gate
//                      and up rows of expert e as +-s fp16 (the group scale
//                      with the weight's sign, exact) times the expert's
//                      contiguous route rows; each accumulates all of K in
//                      TMEM; the epilogue applies the route scale, SiLU(g) * u
//                      and stores h (bf16) in sorted order.
//  5. hprep_kernel     h -> fp16 with a power of two per route.
//  6. moe_gemm<DOWN>   the down rows of expert e times those rows; epilogue
//                      multiplies by the route scale and the route weight and
//                      stores the route output (fp32, sorted order).
//  7. combine_kernel   out[t] = sum over slots, in slot order.
// MMA N (routes per tile) is set per tile from the expert's route count
// (rounded up to 16), so partially filled tiles cost only what they hold.
// On B200 x is duplicated once per route (top_k copies, fp16): one plain TMA
// box per pipeline stage replaces 32 row gathers, for a few MB of traffic.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "w1_common.cuh"

namespace w1 {

bool make_tmap_bf16_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows);

namespace moe {
constexpr int TN_GU = 128;   // routes per gate/up tile
constexpr int TN_D = 128;    // routes per down tile
constexpr int kMaxE = 256;
constexpr int kMaxTopK = 32;
constexpr int kExpWarps = 8;                 // expander warps: 2 threads per weight row
constexpr int kThreads = (6 + kExpWarps) * 32;  // producer, MMA, expanders, 4 epilogue warps

struct Tile {
  int e, rt, start, count;  // expert, 128-row tile, first sorted route, routes
};

struct Workspace {
  size_t hdr, ids, wts, pos, sroute, stok, offsets, tiles_gu, tiles_d, h, rout, xs, xscale, hs, hscale, xcs, total;
  int max_tiles_gu, max_tiles_d;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline Workspace workspace_layout(int64_t T, int64_t H, int64_t I, int E, int top_k) {
  Workspace w;
  const int64_t R = T * top_k;
  w.max_tiles_gu = static_cast<int>(((R + TN_GU - 1) / TN_GU + E) * (I / 128));
  w.max_tiles_d = static_cast<int>(((R + TN_D - 1) / TN_D + E) * (H / 128));
  size_t off = 0;
  w.hdr = off;
  off += 256;
  w.ids = off;
  off = align_up(off + 4 * R, 256);
  w.wts = off;
  off = align_up(off + 4 * R, 256);
  w.pos = off;
  off = align_up(off + 4 * R, 256);
  w.sroute = off;
  off = align_up(off + 4 * R, 256);
  w.stok = off;
  off = align_up(off + 4 * R, 256);
  w.offsets = off;
  off = align_up(off + 4 * (E + 1), 256);
  w.tiles_gu = off;
  off = align_up(off + sizeof(Tile) * w.max_tiles_gu, 256);
  w.tiles_d = off;
  off = align_up(off + sizeof(Tile) * w.max_tiles_d, 256);
  w.h = off;
  off = align_up(off + 2 * static_cast<size_t>(R) * I, 1024);
  w.rout = off;
  off = align_up(off + 4 * static_cast<size_t>(R) * H, 1024);
  w.xs = off;
  off = align_up(off + 2 * static_cast<size_t>(R) * H, 1024);
  w.xscale = off;
  off = align_up(off + 4 * static_cast<size_t>(R), 1024);
  w.hs = off;
  off = align_up(off + 2 * static_cast<size_t>(R) * I, 1024);
  w.hscale = off;
  off = align_up(off + 4 * static_cast<size_t>(R), 256);
  w.xcs = off;
  off = align_up(off + 4 * static_cast<size_t>(T), 256);
  w.total = off;
  return w;
}
}  // namespace moe

// ------------------------------------------------------------------ fp16 operand rows

// Exponent c with max * 2^c in [2^14, 2^15) (0 for an all-zero row), at most
// 126 so that 2^c and 2^-c stay normal floats.  Scaling a bf16 row by 2^c
// keeps every value exact in fp16 (8 significant bits, no overflow).
__device__ __forceinline__ int moe_pow2_exp(float mx) {
  int c = 0;
  if (mx > 0.f) {
    int E;
    frexpf(mx, &E);  // mx < 2^E
    c = 15 - E;
  }
  return c < 126 ? c : 126;
}

__device__ __forceinline__ float bf16x8_absmax(const uint4& u, float mx) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q)
    mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w[q] << 16)), fabsf(__uint_as_float(w[q] & 0xFFFF0000u))));
  return mx;
}

__device__ __forceinline__ uint4 bf16x8_to_f16(const uint4& u, float cs) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __half2 h2 = __floats2half2_rn(__uint_as_float(w[q] << 16) * cs, __uint_as_float(w[q] & 0xFFFF0000u) * cs);
    o[q] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// ------------------------------------------------------------------ 1. router

// One warp routes one token from its E logits: fp32 softmax, the top_k
// experts by logit (the softmax is monotone, so this is selection by
// probability without rounding ties; ties to the lower index); lane 0 writes
// ids[s], wts[s] for s < top_k.
__device__ __forceinline__ void moe_route_token(const float* __restrict__ lp, int E, int top_k, int lane,
                                                int* ids, float* wts) {
  constexpr int PER = moe::kMaxE / 32;
  float z[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    z[j] = (e < E) ? lp[e] : -INFINITY;
  }
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < PER; ++j) mx = fmaxf(mx, z[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j) sum += (lane + 32 * j < E) ? expf(z[j] - mx) : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  for (int s = 0; s < top_k; ++s) {
    // lane-local best: largest logit, lowest index on ties
    float bz = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane + 32 * j;
      if (e < E && (z[j] > bz || (z[j] == bz && e < be))) {
        bz = z[j];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float oz = __shfl_xor_sync(0xFFFFFFFFu, bz, o);
      const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, o);
      if (oz > bz || (oz == bz && oe < be)) {
        bz = oz;
        be = oe;
      }
    }
    if (lane == 0) {
      ids[s] = be;
      wts[s] = expf(bz - mx) / sum;
    }
    if ((be & 31) == lane) z[be >> 5] = -INFINITY;  // taken
  }
}

// One warp per token: routing, and the token's fp16 multiplier 2^c for the
// gate/up operand (xcs[t]), once per token instead of once per route.
__global__ void __launch_bounds__(256) moe_route_kernel(const float* __restrict__ logits, int T, int E, int top_k,
                                                        int* __restrict__ ids, float* __restrict__ wts,
                                                        const uint16_t* __restrict__ x, int H,
                                                        float* __restrict__ xcs) {
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp < T) {
    moe_route_token(logits + static_cast<int64_t>(warp) * E, E, top_k, lane, ids + warp * top_k,
                    wts + warp * top_k);
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(warp) * H);
    float m = 0.f;
#pragma unroll 4
    for (int i = lane; i < (H >> 3); i += 32) m = bf16x8_absmax(__ldg(xr + i), m);
    m = warp_max(m);
    if (lane == 0) xcs[warp] = ldexpf(1.f, moe_pow2_exp(m));
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ 2. sort + tiles

struct SortArgs {
  const int* ids;
  int R, E, top_k, rt_gu, rt_d;  // routes, experts, k, row tiles of gate/up (I/128) and down (H/128)
  int* offsets;
  int* sroute;
  int* stok;
  int* pos;
  moe::Tile* tiles_gu;
  moe::Tile* tiles_d;
  int* hdr;
  int stage;  // sorted routes staged in dynamic shared memory (R ints), written out coalesced
};

// Lanes of this warp holding the same expert id as this lane (ids in
// [0, kMaxE), -1 for none): one ballot per id bit and one for validity.
// Deterministic, and far cheaper than __match_any_sync on this part.
__device__ __forceinline__ unsigned same_id_lanes(int e) {
  static_assert(moe::kMaxE <= 256, "8 id bits");
  const bool valid = e >= 0;
  const unsigned vb = __ballot_sync(0xFFFFFFFFu, valid);
  unsigned m = valid ? vb : ~vb;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const bool bit = (e >> b) & 1;
    const unsigned bb = __ballot_sync(0xFFFFFFFFu, bit);
    m &= bit ? bb : ~bb;
  }
  return m;
}

// One CTA of 1024 threads.  Warp w owns the contiguous route segment
// [w L, (w+1) L); positions inside an expert follow route order (stable).
__global__ void __launch_bounds__(1024) moe_sort_kernel(const SortArgs a) {
  extern __shared__ int sorted[];  // a.stage: sorted position -> route
  __shared__ int cnt[moe::kMaxE];
  __shared__ int tbl[32][moe::kMaxE];  // per (segment, expert): count, then exclusive prefix
  __shared__ int offs[moe::kMaxE + 1];
  __shared__ int pgu[moe::kMaxE + 1], pd[moe::kMaxE + 1];  // tile-list prefixes per expert
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * moe::kMaxE; i += blockDim.x) (&tbl[0][0])[i] = 0;
  const int L = (a.R + 31) / 32;
  const int s0 = warp * L, s1 = min(a.R, s0 + L);
  // this warp's expert ids: the first kPre rounds loaded at once (independent
  // loads), later rounds (R > 32 * 32 * kPre) read in the loops
  constexpr int kPre = 8;
  int pre[kPre];
#pragma unroll
  for (int it = 0; it < kPre; ++it) {
    const int r = s0 + 32 * it + lane;
    pre[it] = (r < s1) ? a.ids[r] : -1;
  }
  auto id_of = [&](int it) {
    int e = -1;
#pragma unroll
    for (int j = 0; j < kPre; ++j)
      if (it == j) e = pre[j];
    if (it >= kPre) {
      const int r = s0 + 32 * it + lane;
      e = (r < s1) ? a.ids[r] : -1;
    }
    return e;
  };
  const int rounds = (s1 - s0 + 31) / 32;  // uniform over the warp
  __syncthreads();
  // per-(segment, expert) counts (order-free: shared-memory atomics)
  for (int it = 0; it < rounds; ++it) {
    const int e = id_of(it);
    if (e >= 0) atomicAdd(&tbl[warp][e], 1);
  }
  __syncthreads();
  // per expert: exclusive prefix over the segments (warp j takes experts j,
  // j + 32, ...; lane = segment) and the expert's total
  for (int e = warp; e < a.E; e += 32) {
    const int v = tbl[lane][e];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += t;
    }
    tbl[lane][e] = incl - v;
    if (lane == 31) cnt[e] = incl;
  }
  __syncthreads();
  // expert offsets and tile-list prefixes: one warp, lane l takes experts
  // [l EPL, (l+1) EPL) in order, then a warp scan of the lane totals
  if (warp == 0) {
    const int EPL = (a.E + 31) / 32;
    int c0 = 0, g0 = 0, d0 = 0;
    for (int k = 0; k < EPL; ++k) {
      const int e = lane * EPL + k;
      if (e < a.E) {
        const int c = cnt[e];
        c0 += c;
        g0 += (c + moe::TN_GU - 1) / moe::TN_GU * a.rt_gu;
        d0 += (c + moe::TN_D - 1) / moe::TN_D * a.rt_d;
      }
    }
    int ci = c0, gi = g0, di = d0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tc = __shfl_up_sync(0xFFFFFFFFu, ci, o);
      const int tg = __shfl_up_sync(0xFFFFFFFFu, gi, o);
      const int td = __shfl_up_sync(0xFFFFFFFFu, di, o);
      if (lane >= o) {
        ci += tc;
        gi += tg;
        di += td;
      }
    }
    int cb = ci - c0, gb = gi - g0, db = di - d0;
    for (int k = 0; k < EPL; ++k) {
      const int e = lane * EPL + k;
      if (e < a.E) {
        const int c = cnt[e];
        offs[e] = cb;
        pgu[e] = gb;
        pd[e] = db;
        cb += c;
        gb += (c + moe::TN_GU - 1) / moe::TN_GU * a.rt_gu;
        db += (c + moe::TN_D - 1) / moe::TN_D * a.rt_d;
      }
    }
    if (lane == 31) {
      offs[a.E] = ci;
      pgu[a.E] = gi;
      pd[a.E] = di;
    }
  }
  __syncthreads();
  if (threadIdx.x <= a.E) a.offsets[threadIdx.x] = offs[threadIdx.x];
  // stable scatter
  for (int it = 0; it < rounds; ++it) {
    const int r = s0 + 32 * it + lane;
    const int e = id_of(it);
    const unsigned peers = same_id_lanes(e);
    if (e >= 0) {
      const int p = offs[e] + tbl[warp][e] + __popc(peers & ((1u << lane) - 1u));
      if (a.stage) {
        sorted[p] = r;
      } else {
        a.sroute[p] = r;
        a.stok[p] = r / a.top_k;
      }
      a.pos[r] = p;
    }
    __syncwarp();
    if (e >= 0 && (__ffs(peers) - 1) == lane) tbl[warp][e] += __popc(peers);
    __syncwarp();
  }
  // tile lists, expert-major (route tile, then row tile), one tile per thread
  auto expert_of = [&](const int* pre_e, int i) {  // largest e with pre_e[e] <= i
    int lo = 0, hi = a.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre_e[mid] <= i) lo = mid;
      else hi = mid - 1;
    }
    return lo;
  };
  for (int i = threadIdx.x; i < pgu[a.E]; i += blockDim.x) {
    const int e = expert_of(pgu, i), loc = i - pgu[e];
    const int j = loc / a.rt_gu, rt = loc - j * a.rt_gu;
    a.tiles_gu[i] = moe::Tile{e, rt, offs[e] + j * moe::TN_GU, min(moe::TN_GU, cnt[e] - j * moe::TN_GU)};
  }
  for (int i = threadIdx.x; i < pd[a.E]; i += blockDim.x) {
    const int e = expert_of(pd, i), loc = i - pd[e];
    const int j = loc / a.rt_d, rt = loc - j * a.rt_d;
    a.tiles_d[i] = moe::Tile{e, rt, offs[e] + j * moe::TN_D, min(moe::TN_D, cnt[e] - j * moe::TN_D)};
  }
  if (threadIdx.x == 0) {
    a.hdr[0] = pgu[a.E];
    a.hdr[1] = pd[a.E];
  }
  if (a.stage) {  // sorted route order out, coalesced
    __syncthreads();
    for (int i = threadIdx.x; i < a.R; i += blockDim.x) {
      const int r = sorted[i];
      a.sroute[i] = r;
      a.stok[i] = r / a.top_k;
    }
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ 3/4. grouped GEMMs

struct MoeGemmParams {
  // weights of the A side: [E][rows][K/32] signs, [E][rows][K/128] scales
  const uint32_t* a_signs;
  const uint16_t* a_scales;
  const uint32_t* u_signs;   // gate/up only: the up matrix (a_* is gate)
  const uint16_t* u_scales;
  const moe::Tile* tiles;
  const int* hdr;            // hdr[0] gate/up tiles, hdr[1] down tiles
  const int* stok;           // sorted position -> token (gather rows)
  const int* sroute;         // sorted position -> route
  const float* wts;          // route weights
  const float* rscale;       // per sorted route: 2^-c of the fp16 B rows
  __nv_bfloat16* h;          // gate/up output [R][I]
  float* rout;               // down output [R][H]
  int rows;                  // rows of each expert matrix (I for gate/up, H for down)
  int K;                     // contracted size (H for gate/up, I for down)
  int out_ld;                // leading dimension of the output
};

template <bool GATEUP>
struct MoeCfg {
  static constexpr int TN = GATEUP ? moe::TN_GU : moe::TN_D;  // routes per tile (max MMA N)
  static constexpr int NMAT = GATEUP ? 2 : 1;                 // weight matrices per tile
  // K per pipeline stage: one scale group, two 64-wide (128-byte) swizzle
  // atoms; long stages amortise the MMA issuer's barrier wait over 8 x NMAT MMAs
  static constexpr int BKS = 128;
  static constexpr int NS = GATEUP ? 2 : 3;                   // stages (192 KB either way)
  static constexpr int XATOM = TN * 128;                      // bytes of one 64-wide atom of B
  static constexpr int XSTAGE = 2 * XATOM;                    // bytes of one B stage (fp16)
  static constexpr int AATOM = 128 * 128;                     // bytes of one 64-wide atom of A
  static constexpr int ASTAGE = 2 * AATOM;                    // bytes of one weight matrix stage
  static constexpr uint32_t kTmemCols = GATEUP ? 512 : 256;   // two accumulator sets
};

template <bool GATEUP>
struct MoeSmem {
  alignas(1024) unsigned char x[MoeCfg<GATEUP>::NS][MoeCfg<GATEUP>::XSTAGE];
  alignas(1024) unsigned char a[MoeCfg<GATEUP>::NS][MoeCfg<GATEUP>::NMAT][MoeCfg<GATEUP>::ASTAGE];
  uint64_t full[MoeCfg<GATEUP>::NS], empty[MoeCfg<GATEUP>::NS];
  uint64_t full_c[2], empty_c[2];
  uint32_t tmem_base;
};

__device__ __forceinline__ void moe_st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Warp roles: 0 TMA producer (route rows of B), 1 MMA issuer, 2-9 expanders
// (two threads per weight row: sign words + the group scale -> fp16 pairs +-s
// in the 128B-swizzled K-major layout; gate/up: one matrix each, down: one
// word pair of the stage each), 10-13 epilogue (thread = TMEM lane).  One
// 128-wide K stage: NMAT x 8 MMAs (M = 128, N = the tile's route count rounded
// up to 16, K = 16), all of K into one accumulator per matrix per tile; two
// accumulator sets alternate between tiles.
template <bool GATEUP>
__global__ void __launch_bounds__(moe::kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const MoeGemmParams p) {
  using C = MoeCfg<GATEUP>;
  extern __shared__ unsigned char smem_raw[];
  MoeSmem<GATEUP>& sm =
      *reinterpret_cast<MoeSmem<GATEUP>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      // one barrier per stage: the expanders' arrivals plus the producer's
      // arrival with the activation tile's transaction bytes
      mbar_init(&sm.full[i], 32 * moe::kExpWarps + 1);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.full_c[i], 1);
      mbar_init(&sm.empty_c[i], 128);
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_b) : "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();
  const int ntiles = p.hdr[GATEUP ? 0 : 1];
  const int NG = p.K >> 7;          // scale groups per row
  const int NKS = p.K / C::BKS;     // stages per tile

  if (warp == 0) {
    if (lane == 0) {
      uint32_t c = 0;
      for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
        const moe::Tile tl = p.tiles[ti];
        for (int ks = 0; ks < NKS; ++ks, ++c) {
          const int s = c % C::NS;
          if (!mbar_wait(&sm.empty[s], ((c / C::NS) & 1) ^ 1)) goto done_prod;
          mbar_arrive_expect_tx(&sm.full[s], C::XSTAGE);
          tma_load_2d(sm.x[s], &tmap_b, ks * C::BKS, tl.start, &sm.full[s]);
          tma_load_2d(sm.x[s] + C::XATOM, &tmap_b, ks * C::BKS + 64, tl.start, &sm.full[s]);
        }
      }
    done_prod:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t c = 0, tli = 0;
      for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x, ++tli) {
        const moe::Tile tl = p.tiles[ti];
        const int n_mma = ((tl.count + 15) >> 4) << 4;
        const uint32_t idesc = idesc_f16(128, n_mma, 0, 0);  // fp16 x fp16 -> fp32
        const int cb = tli & 1;
        if (!mbar_wait(&sm.empty_c[cb], ((tli >> 1) & 1) ^ 1)) goto done_mma;
        tc_fence_after();
        for (int ks = 0; ks < NKS; ++ks, ++c) {
          const int s = c % C::NS;
          if (!mbar_wait(&sm.full[s], (c / C::NS) & 1)) goto done_mma;
          tc_fence_after();
          const uint32_t xbase = smem_u32(sm.x[s]);
#pragma unroll
          for (int mat = 0; mat < C::NMAT; ++mat) {
            const uint32_t d = tmem + (cb * C::NMAT + mat) * C::TN;
            const uint32_t abase = smem_u32(sm.a[s][mat]);
#pragma unroll
            for (int kk = 0; kk < C::BKS / 16; ++kk) {
              const uint32_t ao = (kk >> 2) * C::AATOM + (kk & 3) * 32, xo = (kk >> 2) * C::XATOM + (kk & 3) * 32;
              tc_mma_ss(d, smem_desc_sw128(abase + ao), smem_desc_sw128(xbase + xo), idesc,
                        (ks > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(&sm.empty[s]);
        }
        tc_commit(&sm.full_c[cb]);
      }
    done_mma:;
    }
  } else if (warp < 2 + moe::kExpWarps) {
    // expanders: two threads per weight row of the tile's 128-row block.
    // gate/up: half h expands matrix h (gate, up), all four sign words of a
    // 128-wide stage; down: half h expands words 2h, 2h+1 (swizzle atom h).
    constexpr int kPf = 4;
    constexpr int NW = GATEUP ? 4 : 2;  // sign words per thread per stage
    const int et = (warp - 2) * 32 + lane;
    const int rl = et & 127, half = et >> 7;
    const int mat = GATEUP ? half : 0;
    const int w0 = GATEUP ? 0 : 2 * half;  // first word of the stage this thread expands
    const int64_t wrow = p.K >> 5;
    // the stream's current tile: row pointers cached in registers, the tile
    // descriptor read once per tile (not once per stage)
    int ld_ti = blockIdx.x, ld_ks = 0;
    const uint32_t* wp = nullptr;
    const uint16_t* sp = nullptr;
    bool ld_valid = false;
    auto load_tile = [&]() {
      ld_valid = false;
      if (ld_ti < ntiles) {
        const moe::Tile tl = p.tiles[ld_ti];
        const int row = tl.rt * 128 + rl;
        ld_valid = row < p.rows;
        const int64_t ridx = static_cast<int64_t>(tl.e) * p.rows + (ld_valid ? row : 0);
        wp = (mat ? p.u_signs : p.a_signs) + ridx * wrow + w0;
        sp = (mat ? p.u_scales : p.a_scales) + ridx * NG;
      }
    };
    load_tile();
    auto fetch = [&](uint32_t (&w)[NW], uint32_t& sc) {
#pragma unroll
      for (int i = 0; i < NW; ++i) w[i] = 0;
      sc = 0x3C00u;
      if (ld_ti < ntiles) {
        if (ld_valid) {
          if constexpr (NW == 4) {  // a row's words are 16-byte aligned (K % 128 == 0)
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(wp) + ld_ks);
            w[0] = u.x;
            w[1 % NW] = u.y;
            w[2 % NW] = u.z;
            w[3 % NW] = u.w;
          } else {
            const uint2 u = __ldg(reinterpret_cast<const uint2*>(wp + 4 * ld_ks));
            w[0] = u.x;
            w[1 % NW] = u.y;
          }
          sc = __ldg(sp + ld_ks);  // one scale group per stage
        }
        if (++ld_ks == NKS) {
          ld_ks = 0;
          ld_ti += gridDim.x;
          load_tile();
        }
      }
    };
    uint32_t wr[kPf][NW];
    uint32_t sr[kPf];
#pragma unroll
    for (int j = 0; j < kPf; ++j) fetch(wr[j], sr[j]);
    const int my_tiles = (ntiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                         static_cast<int>(gridDim.x);
    const int my_stages = (my_tiles > 0 ? my_tiles : 0) * NKS;
    const uint32_t row_off = static_cast<uint32_t>(rl) * 128u;
    const uint32_t swz = static_cast<uint32_t>(rl & 7);
    uint32_t c = 0;
    for (int c0 = 0; c0 < my_stages; c0 += kPf) {
#pragma unroll
      for (int j = 0; j < kPf; ++j) {
        if (c0 + j >= my_stages) break;
        uint32_t cur[NW];
#pragma unroll
        for (int i = 0; i < NW; ++i) cur[i] = wr[j][i];
        const uint32_t ss = sr[j] * 0x00010001u;  // the scale in both fp16 halves
        fetch(wr[j], sr[j]);
        const int s = c % C::NS;
        if (!mbar_wait_warp(&sm.empty[s], ((c / C::NS) & 1) ^ 1)) goto done_exp;
        const uint32_t abase = smem_u32(sm.a[s][mat]) + row_off;  // + atom offset per word pair
#pragma unroll
        for (int wi = 0; wi < NW; ++wi) {
          const uint32_t w = cur[wi];
          uint32_t rr[16];
#pragma unroll
          for (int pp = 0; pp < 16; ++pp) {
            const uint32_t src = (pp < 8) ? w : (w >> 16);
            const int b = 2 * (pp & 7);
            const uint32_t m = src & (3u << b);
            const uint32_t tt = m * (0x40008000u >> b);
            rr[pp] = (tt & 0x80008000u) | ss;
          }
          const int gw = w0 + wi;  // word of the stage: atom gw / 2, chunks 4 (gw % 2) + q
          const uint32_t ab = abase + static_cast<uint32_t>((gw >> 1) * C::AATOM);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t chunk = static_cast<uint32_t>((gw & 1) * 4 + q);
            moe_st_shared_v4(ab + ((chunk ^ swz) << 4), rr[4 * q], rr[4 * q + 1], rr[4 * q + 2], rr[4 * q + 3]);
          }
        }
        fence_async_shared();
        mbar_arrive(&sm.full[s]);
        ++c;
      }
    }
  done_exp:;
  } else {
    // epilogue: thread = weight row (TMEM lane)
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t tli = 0;
    for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x, ++tli) {
      const moe::Tile tl = p.tiles[ti];
      const int row = tl.rt * 128 + rl;
      const bool valid = row < p.rows;
      const int cb = tli & 1;
      if (!mbar_wait_warp(&sm.full_c[cb], (tli >> 1) & 1)) goto done_epi;
      tc_fence_after();
#pragma unroll 1
      for (int q4 = 0; q4 < C::TN / 32; ++q4) {
        if (q4 * 32 >= tl.count) break;
        uint32_t rg[32];
        tmem_ld32(tmem + lane_addr + (cb * C::NMAT) * C::TN + q4 * 32, rg);
        if (GATEUP) {
          uint32_t ru[32];
          tmem_ld32(tmem + lane_addr + (cb * C::NMAT + C::NMAT - 1) * C::TN + q4 * 32, ru);
          tc_wait_ld();
          if (valid) {
            __nv_bfloat16* hp = p.h + static_cast<int64_t>(tl.start) * p.out_ld + row;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int jj = q4 * 32 + j;
              if (jj < tl.count) {
                const float rs = __ldg(p.rscale + tl.start + jj);
                const float g = __uint_as_float(rg[j]) * rs;
                const float u = __uint_as_float(ru[j]) * rs;
                const float hv = g / (1.0f + expf(-g)) * u;
                hp[static_cast<int64_t>(jj) * p.out_ld] = __float2bfloat16_rn(hv);
              }
            }
          }
        } else {
          tc_wait_ld();
          if (valid) {
            float* op = p.rout + static_cast<int64_t>(tl.start) * p.out_ld + row;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int jj = q4 * 32 + j;
              if (jj < tl.count) {
                const float wgt = __ldg(p.wts + __ldg(p.sroute + tl.start + jj)) * __ldg(p.rscale + tl.start + jj);
                __stcs(op + static_cast<int64_t>(jj) * p.out_ld, wgt * __uint_as_float(rg[j]));
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
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ gather x rows (sorted, fp16)

// One warp per sorted route p: xs[p] = fp16(x[t] * 2^c_t) for t = stok[p], with
// the token's multiplier from the router (max |x_t| * 2^c_t in [2^14, 2^15):
// exact for every bf16 value), xscale[p] = 2^-c_t.  A plain streaming copy:
// 16-byte loads and stores, no reduction.
__global__ void __launch_bounds__(256) moe_gather_kernel(const uint16_t* __restrict__ x, const int* __restrict__ stok,
                                                         const float* __restrict__ xcs, int R, int H,
                                                         __half* __restrict__ xs, float* __restrict__ xscale) {
  pdl_wait();
  const int p = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (p < R) {
    const int t = __ldg(stok + p);
    const float cs = __ldg(xcs + t);
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * H);
    uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<int64_t>(p) * H);
#pragma unroll 4
    for (int i = lane; i < (H >> 3); i += 32) dst[i] = bf16x8_to_f16(__ldg(src + i), cs);
    if (lane == 0) xscale[p] = 1.f / cs;  // exact: cs is a normal power of two
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ h rows -> fp16

// One warp per sorted route p: hs[p] = fp16(h[p] * 2^c) with max |h[p]| * 2^c
// in [2^14, 2^15), hscale[p] = 2^-c.  The row stays in registers between the
// max and the conversion when I <= 32 * 8 * kKeep, longer rows are re-read.
__global__ void __launch_bounds__(256) moe_hprep_kernel(const uint16_t* __restrict__ h, int R, int I,
                                                        __half* __restrict__ hs, float* __restrict__ hscale) {
  constexpr int kKeep = 8;
  pdl_wait();
  const int p = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (p < R) {
    const uint4* src = reinterpret_cast<const uint4*>(h + static_cast<int64_t>(p) * I);
    uint4* dst = reinterpret_cast<uint4*>(hs + static_cast<int64_t>(p) * I);
    const int nv = I >> 3;
    uint4 keep[kKeep];
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < kKeep; ++j) {
      const int i = lane + 32 * j;
      keep[j] = i < nv ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      m = bf16x8_absmax(keep[j], m);
    }
    for (int i = lane + 32 * kKeep; i < nv; i += 32) m = bf16x8_absmax(__ldg(src + i), m);
    const int c = moe_pow2_exp(warp_max(m));
    const float cs = ldexpf(1.f, c);
#pragma unroll
    for (int j = 0; j < kKeep; ++j) {
      const int i = lane + 32 * j;
      if (i < nv) dst[i] = bf16x8_to_f16(keep[j], cs);
    }
    for (int i = lane + 32 * kKeep; i < nv; i += 32) dst[i] = bf16x8_to_f16(__ldg(src + i), cs);
    if (lane == 0) hscale[p] = ldexpf(1.f, -c);
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ decode regime (T <= kDecodeMaxT = 16)

// With a handful of tokens every expert sees about one route, so the tile
// pipeline's 128-route MMA tiles would be almost empty.  Instead each route is
// a batch-1 product on the direct GEMV steps (gemv_direct.cu): exact
// fixed-point activation digits, int8 mma.sync on the sign bytes, one fold
// per group.  Gate/up: a CTA takes one route and 64 output rows; warps 0-3
// own 16 rows each of G_e and warps 4-7 the same rows of U_e, each over all of
// K (no cross-warp reduction), and h = bf16(silu(g) u) is formed through
// shared memory.  Down + combine: moe_decode_down_kernel below.
namespace moed {
constexpr int kWarps = 8;
constexpr int kTw = 2;                   // 8-row n-tiles per warp
constexpr int kRowsGu = 4 * 8 * kTw;     // gate/up rows per CTA (of each matrix)
constexpr int kSmemCap = 220 * 1024;     // dynamic shared memory the decode kernels may use
}  // namespace moed

struct MoeDecParams {
  const float* logits;       // gate/up with self_route: router logits [T][E]
  int E;
  int self_route;            // gate/up: each CTA routes its token (else ids come from the router kernel)
  int* ids;                  // [R] expert per route (written by gate/up, read by down)
  float* wts;                // [R] route weight
  const uint16_t* x;         // gate/up: tokens [T][H] bf16; down: h [R][I] bf16
  const uint32_t* signs0;    // gate/up: G, down: D   [E][rows][K/32]
  const uint16_t* scales0;
  const uint32_t* signs1;    // gate/up: U
  const uint16_t* scales1;
  __nv_bfloat16* h;          // gate/up output [R][I]
  int* pos;                  // gate/up: route -> its row of h (identity here)
  int R, top_k, rows, K, NG, P, lgGw;
};

__host__ __device__ inline GdSmem moed_layout(const MoeDecParams& q, int tw = moed::kTw) {
  return gd_layout<1, moed::kWarps>(tw, q.NG, q.P, 1, 0, q.NG);
}

// TWG 8-row n-tiles per warp: 2 (16 rows of G or U per warp, 64 per CTA) or
// 4 (32 per warp, 128 per CTA: half the CTAs, each activation fragment and
// fold shared by two MMA tiles, the token's x quantised half as often).
template <int TWG>
__global__ void __launch_bounds__(moed::kWarps * 32, 1) moe_decode_gateup_kernel(const MoeDecParams q) {
  constexpr int kRows = 4 * 8 * TWG;  // rows of each matrix per CTA
  constexpr int TP = (TWG + 1) / 2;   // 16-row MMA tiles per warp
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float gu[2][kRows];
  const GdSmem L = moed_layout(q, TWG);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int sid[moe::kMaxTopK];
  __shared__ float swt[moe::kMaxTopK];
  const int r = blockIdx.y, t = r / q.top_k, slot = r - t * q.top_k;
  pdl_wait();
  pdl_launch_dependents();
  // self_route: the token's routing, computed by every CTA of the token from
  // the router kernel's routine; the route's first row block records it
  int e;
  if (q.self_route) {
    if (warp == 0) moe_route_token(q.logits + static_cast<int64_t>(t) * q.E, q.E, q.top_k, lane, sid, swt);
    __syncthreads();
    e = sid[slot];
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      q.ids[r] = e;
      q.wts[r] = swt[slot];
    }
  } else {
    e = q.ids[r];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) q.pos[r] = r;
  // this warp's matrix (0: G, 1: U) and rows
  const int mat = warp >> 2;
  const int row0 = blockIdx.x * kRows + (warp & 3) * 8 * TWG;
  GdParams p = {};
  const int64_t mrow = static_cast<int64_t>(e) * q.rows;  // the expert's first row
  p.signs = (mat ? q.signs1 : q.signs0) + mrow * (q.K >> 5);
  p.scales = (mat ? q.scales1 : q.scales0) + mrow * q.NG;
  p.x = q.x + static_cast<int64_t>(t) * q.K;
  p.N = q.rows;
  p.K = q.K;
  p.NG = q.NG;
  p.Tw = TWG;
  p.NSw = q.NG;
  p.P = q.P;
  p.lgGw = q.lgGw;
  GdGeom g = {};
  g.nsc = q.NG;
  g.tw = TWG;
  g.nsw = q.NG;
  g.row0 = row0;
  g.nrows = max(0, min(8 * TWG, q.rows - row0));
  g.busy = g.nrows > 0;
  g.ngw = q.NG;
  unsigned char* wreg = smem + warp * L.warp_bytes;
  unsigned char* wts = wreg + L.wts;
  float* scl = reinterpret_cast<float*>(wreg + L.scl);
  uint32_t* xs = reinterpret_cast<uint32_t*>(smem + L.xs);
  uint16_t sreg[kGdSpl];
  if (g.busy) gd_stage<1>(p, g, wts, lane);
  else cp_async_commit();
  gd_load_scales<1>(p, g, 0, lane, sreg);
  uint4 xa[4];
  gd_x_first<1, false>(p, g, warp, lane, xa);
  gd_prep_x<1, false, moed::kWarps>(p, g, xs, warp, lane, xa);
  gd_finish_scales<1>(p, g, lane, sreg, scl);
  cp_async_wait_all();
  __syncthreads();
  float acc[gd::kMaxTp][gd::Cfg<1>::NN][4];
#pragma unroll
  for (int tp = 0; tp < gd::kMaxTp; ++tp)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[tp][0][i] = 0.f;
  if (g.busy) gd_compute<1, TWG>(wts, p.P, scl, 8 * TWG, xs, q.NG, lane, acc);
  // digit columns -> row sums: a lane holds columns 2(lane&3), +1 of rows
  // 16 tp + lane/4 and 16 tp + lane/4 + 8 of each MMA tile tp; columns past
  // the three digits are zero, so the quad sum is the row's value
  const int rl = lane >> 2;
  const int base = (warp & 3) * 8 * TWG;
#pragma unroll
  for (int tp = 0; tp < TP; ++tp) {
    float v0 = acc[tp][0][0] + acc[tp][0][1], v1 = acc[tp][0][2] + acc[tp][0][3];
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, o);
      v1 += __shfl_xor_sync(0xFFFFFFFFu, v1, o);
    }
    if ((lane & 3) == 0) {
      gu[mat][base + 16 * tp + rl] = v0;
      if (16 * tp + 8 < 8 * TWG) gu[mat][base + 16 * tp + 8 + rl] = v1;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRows; i += blockDim.x) {
    const int row = blockIdx.x * kRows + i;
    if (row < q.rows) {
      const float gv = gu[0][i], uv = gu[1][i];
      q.h[static_cast<int64_t>(r) * q.rows + row] = __float2bfloat16_rn(gv / (1.0f + expf(-gv)) * uv);
    }
  }
}

// ------------------------------------------------------------------ 5. combine

__global__ void __launch_bounds__(256) moe_combine_kernel(const float* __restrict__ rout, const int* __restrict__ pos,
                                                          int T, int H, int top_k, float* __restrict__ out) {
  pdl_wait();
  const int64_t total4 = static_cast<int64_t>(T) * (H / 4);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / (H / 4));
    const int c4 = static_cast<int>(i - static_cast<int64_t>(t) * (H / 4));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < top_k; ++s) {
      const int p = __ldg(pos + t * top_k + s);
      const float4 v = __ldcs(reinterpret_cast<const float4*>(rout + static_cast<int64_t>(p) * H) + c4);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    reinterpret_cast<float4*>(out + static_cast<int64_t>(t) * H)[c4] = acc;
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ host side

size_t moe_workspace_bytes(int64_t T, int64_t H, int64_t I, int E, int top_k) {
  return moe::workspace_layout(T, H, I, E, top_k).total;
}

template <class Kern, class... Args>
static cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Down products and the slot-ordered combine of the decode regime, fused:
// one CTA per (token, RB output rows), RB = 16 x tokens (at most 128), so a
// route's h is quantised by as many CTAs as there are row blocks, whatever
// the batch.  Warp w takes slots w, w + 8, ...: it quantises that route's h
// into its own digit scratch, stages RB rows of D_e at once and forms their
// products 32 rows at a time (the direct GEMV steps at batch 1).  The slots'
// partial sums (times the route weight) meet in shared memory, and RB
// threads add them in slot order (deterministic) straight into out.
struct MoeDownLayout {
  int RB, P, wts, scl, xs, warp_bytes, part, total;
};
__host__ __device__ inline MoeDownLayout moe_down_layout(int NG, int RB) {
  MoeDownLayout L;
  L.RB = RB;
  L.P = ((NG & 1) ? NG : NG + 1) * 16;  // odd multiple of 16 bytes per staged row: bank spread
  L.wts = 0;
  L.scl = (L.wts + RB * L.P + 15) / 16 * 16;
  L.xs = (L.scl + NG * RB * 4 + 15) / 16 * 16;
  L.warp_bytes = (L.xs + NG * gd::Cfg<1>::SCR * 4 + 15) / 16 * 16;
  L.part = moed::kWarps * L.warp_bytes;
  L.total = L.part + moe::kMaxTopK * RB * 4;
  return L;
}

__global__ void __launch_bounds__(moed::kWarps * 32, 1) moe_decode_down_kernel(const MoeDecParams q, int RB,
                                                                             float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const MoeDownLayout L = moe_down_layout(q.NG, RB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.y, row0 = blockIdx.x * RB;
  unsigned char* wreg = smem + warp * L.warp_bytes;
  unsigned char* wts = wreg + L.wts;
  float* scl = reinterpret_cast<float*>(wreg + L.scl);  // [group][RB rows]
  uint32_t* xs = reinterpret_cast<uint32_t*>(wreg + L.xs);
  float* part = reinterpret_cast<float*>(smem + L.part);  // [slot][RB rows]
  pdl_wait();
  pdl_launch_dependents();
  for (int s = warp; s < q.top_k; s += moed::kWarps) {  // warp-uniform
    const int r = t * q.top_k + s;
    const int e = q.ids[r];
    GdParams p = {};
    const int64_t mrow = static_cast<int64_t>(e) * q.rows;
    p.signs = q.signs0 + mrow * (q.K >> 5);
    p.scales = q.scales0 + mrow * q.NG;
    p.N = q.rows;
    p.K = q.K;
    p.NG = q.NG;
    p.Tw = RB / 8;  // scale rows stride RB
    p.NSw = q.NG;
    p.P = L.P;
    p.lgGw = q.lgGw;
    GdGeom g = {};
    g.nsc = q.NG;
    g.tw = RB / 8;
    g.nsw = q.NG;
    g.row0 = row0;
    g.nrows = max(0, min(RB, q.rows - row0));
    g.busy = g.nrows > 0;
    g.ngw = q.NG;
    uint16_t sreg[kGdSpl];
    if (g.busy) gd_stage<1>(p, g, wts, lane);
    gd_load_scales<1>(p, g, 0, lane, sreg);
    // this route's h -> digit scratch: a unit is one group (8 lanes x 16
    // values), four units per pass of the warp
    const uint16_t* hr = q.x + static_cast<int64_t>(r) * q.K;
    for (int g0 = 0; g0 < q.NG; g0 += 4) {
      const int gi = g0 + (lane >> 3), sub = lane & 7;
      float v[16];
      uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
      if (gi < q.NG) {
        const uint4* src = reinterpret_cast<const uint4*>(hr + gi * 128 + sub * 16);
        u0 = src[0];
        u1 = src[1];
      }
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
      quantise_item<1>(v, gi < q.NG, sub, xs + (gi < q.NG ? gi : 0) * gd::Cfg<1>::SCR);
    }
    gd_finish_scales<1>(p, g, lane, sreg, scl);
    cp_async_wait_all();
    __syncwarp();
    const float wt = q.wts[r];
    for (int c0 = 0; c0 < RB; c0 += 32) {  // 32 rows (4 n-tiles) or the last 16
      float acc[gd::kMaxTp][gd::Cfg<1>::NN][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[0][0][i] = acc[1][0][i] = 0.f;
      const unsigned char* wc = wts + c0 * L.P;
      const float* sc = scl + c0;
      if (g.busy) {
        if (RB - c0 >= 32) gd_compute<1, 4>(wc, L.P, sc, RB, xs, q.NG, lane, acc);
        else gd_compute<1, 2>(wc, L.P, sc, RB, xs, q.NG, lane, acc);
      }
      // quad sums: rows lane/4 + {0, 8} (pair 0) and + {16, 24} (pair 1)
      float v[4] = {acc[0][0][0] + acc[0][0][1], acc[0][0][2] + acc[0][0][3], acc[1][0][0] + acc[1][0][1],
                    acc[1][0][2] + acc[1][0][3]};
#pragma unroll
      for (int o = 1; o < 4; o <<= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] += __shfl_xor_sync(0xFFFFFFFFu, v[i], o);
      if ((lane & 3) == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = c0 + 8 * i + (lane >> 2);
          if (rr < RB) part[s * RB + rr] = wt * v[i];
        }
      }
    }
    __syncwarp();  // this warp's buffers are reused by its next slot
  }
  __syncthreads();
  for (int i = threadIdx.x; i < RB; i += blockDim.x) {
    if (row0 + i < q.rows) {
      float sum = 0.f;
      for (int s = 0; s < q.top_k; ++s) sum += part[s * RB + i];
      out[static_cast<int64_t>(t) * q.rows + row0 + i] = sum;
    }
  }
}

// ------------------------------------------------------------------ decode regime, grouped by expert
// "LLM binarization episode 01: DBF", section 7 item 1: with a few tokens,
// products specialised to the observed expert counts, so that the tokens
// routed to one expert read its packed weights once.  The list kernel routes
// the tokens and groups the routes by expert (route order within an expert);
// then one CTA per (expert, row block) stages the expert's rows once and runs
// the direct GEMV steps with the expert's routes as its batch rows -- a
// 1..4-row product chosen by the route count, 4 routes at a time above (the
// rows stay staged) -- for gate/up (+ SwiGLU) and for down (x the route
// weight); the combine adds each token's slots in slot order.  Batches of at
// most 4 rows keep a CTA within half an SM (registers and shared memory), so
// two CTAs share each SM.
namespace moeg {
constexpr int kMaxT = 16;                     // tokens of the grouped decode path
constexpr int kMaxR = kMaxT * moe::kMaxTopK;  // routes
constexpr int kRowsD = 16 * moed::kWarps;     // down rows per CTA (16 per warp)
constexpr int kBatch = 4;                     // routes per product batch
constexpr int kRedCols = 3 * kBatch;          // digit columns of a batch
}  // namespace moeg

struct MoeGroupList {
  int* nexp;       // [1] experts with at least one route
  int* exp_id;     // [E] expert of list slot i (ascending)
  int* exp_cnt;    // [E] its route count
  int* exp_start;  // [E] its first position in sroute
  int* sroute;     // [R] routes grouped by expert, route order within an expert
};

// One CTA: warp t routes token t (the router's routine), then the routes are
// counted per expert and listed.  pos[r] = r (the combine reads route rows).
__global__ void __launch_bounds__(512) moe_decode_list_kernel(const float* __restrict__ logits, int T, int E,
                                                              int top_k, int* __restrict__ ids,
                                                              float* __restrict__ wts, int* __restrict__ pos,
                                                              MoeGroupList gl) {
  __shared__ int sid[moeg::kMaxR];
  __shared__ float swt[moeg::kMaxR];
  __shared__ int cnt[moe::kMaxE], start[moe::kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = T * top_k;
  pdl_wait();
  if (warp < T)
    moe_route_token(logits + static_cast<int64_t>(warp) * E, E, top_k, lane, sid + warp * top_k, swt + warp * top_k);
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    ids[r] = sid[r];
    wts[r] = swt[r];
    pos[r] = r;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
    for (int r = 0; r < R; ++r) c += sid[r] == e;
    cnt[e] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int st = 0, nl = 0;
    for (int e = 0; e < E; ++e) {
      start[e] = st;
      if (cnt[e]) {
        gl.exp_id[nl] = e;
        gl.exp_cnt[nl] = cnt[e];
        gl.exp_start[nl] = st;
        ++nl;
      }
      st += cnt[e];
    }
    gl.nexp[0] = nl;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (!cnt[e]) continue;
    int j = start[e];
    for (int r = 0; r < R; ++r)
      if (sid[r] == e) gl.sroute[j++] = r;
  }
  pdl_launch_dependents();
}

// Shared memory of the grouped kernels: per-warp staged rows and scales (as
// the batch-1 decode kernels), the activation digits for 8 batch rows, the
// per-warp digit-column partials.
struct MoeGroupLayout {
  int warp_bytes, xs, red, total;
};
__host__ __device__ inline MoeGroupLayout moeg_layout(int NG, int P) {
  const GdSmem L = gd_layout<1, moed::kWarps>(moed::kTw, NG, P, 1, 0, NG);
  MoeGroupLayout M;
  M.warp_bytes = L.warp_bytes;
  M.xs = moed::kWarps * L.warp_bytes;
  M.red = M.xs + (NG * gd::Cfg<moeg::kBatch>::SCR * 4 + 15) / 16 * 16;
  M.total = M.red + moed::kWarps * 16 * moeg::kRedCols * 4;
  return M;
}

// One batch of NB routes of the CTA's expert: digits of the NB input rows
// (p.xrows), every warp's products over its 16 rows and all of K, the digit
// columns of each (row, route) summed -> emit(row in CTA, b, value).
template <int NB, class Emit>
__device__ __forceinline__ void moeg_batch(const GdParams& p, const GdGeom& g, const unsigned char* wts,
                                           const float* scl, uint32_t* xs, float* red, int warp, int lane,
                                           int rows_cta, Emit&& emit) {
  using C = gd::Cfg<NB>;
  uint4 xa[4];
  gd_x_first<NB, false>(p, g, warp, lane, xa);
  gd_prep_x<NB, false, moed::kWarps>(p, g, xs, warp, lane, xa);
  __syncthreads();  // every unit's digits stored
  float acc[gd::kMaxTp][C::NN][4];
#pragma unroll
  for (int tp = 0; tp < gd::kMaxTp; ++tp)
#pragma unroll
    for (int nn = 0; nn < C::NN; ++nn)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tp][nn][e] = 0.f;
  if (g.busy) gd_compute<NB, moed::kTw>(wts, p.P, scl, 8 * moed::kTw, xs, p.NG, lane, acc);
  const int r1 = lane >> 2, cq = lane & 3;
  float* rw = red + warp * 16 * moeg::kRedCols;
#pragma unroll
  for (int nn = 0; nn < C::NN; ++nn)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int col = 8 * nn + 2 * cq + c;
      if (col < C::NCOL) {
        rw[r1 * moeg::kRedCols + col] = acc[0][nn][c];
        rw[(r1 + 8) * moeg::kRedCols + col] = acc[0][nn][2 + c];
      }
    }
  __syncthreads();
  for (int o = threadIdx.x; o < rows_cta * NB; o += blockDim.x) {
    const int i = o / NB, b = o - i * NB;
    emit(i, b, red);
  }
  __syncthreads();  // digits and partials are rewritten by the next batch
}

// Rows of this warp inside the CTA's block, and its GEMV geometry.
__device__ __forceinline__ GdGeom moeg_geom(int NG, int rows, int row0) {
  GdGeom g = {};
  g.nsc = NG;
  g.tw = moed::kTw;
  g.nsw = NG;
  g.row0 = row0;
  g.nrows = max(0, min(8 * moed::kTw, rows - row0));
  g.busy = g.nrows > 0;
  g.ngw = NG;
  return g;
}

template <bool GATEUP>
__global__ void __launch_bounds__(moed::kWarps * 32, 2) moe_decode_grouped_kernel(const MoeDecParams q,
                                                                                  MoeGroupList gl,
                                                                                  float* __restrict__ rout) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int xrow[moeg::kBatch], route[moeg::kBatch];
  const MoeGroupLayout L = moeg_layout(q.NG, q.P);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  const int slot = blockIdx.y;
  if (slot >= *gl.nexp) return;  // uniform over the CTA
  const int e = gl.exp_id[slot], cnt = gl.exp_cnt[slot], st0 = gl.exp_start[slot];
  // gate/up: warps 0-3 own 16 rows each of G_e, warps 4-7 the same rows of
  // U_e (64 rows per CTA); down: warp w owns rows 16 w .. of the CTA's 128
  const int mat = GATEUP ? warp >> 2 : 0;
  const int rows_cta = GATEUP ? moed::kRowsGu : moeg::kRowsD;
  const int row0 = blockIdx.x * rows_cta + (GATEUP ? (warp & 3) : warp) * 16;
  GdParams p = {};
  const int64_t mrow = static_cast<int64_t>(e) * q.rows;
  p.signs = (mat ? q.signs1 : q.signs0) + mrow * (q.K >> 5);
  p.scales = (mat ? q.scales1 : q.scales0) + mrow * q.NG;
  p.x = q.x;
  p.xrows = xrow;
  p.N = q.rows;
  p.K = q.K;
  p.NG = q.NG;
  p.Tw = moed::kTw;
  p.NSw = q.NG;
  p.P = q.P;
  p.lgGw = q.lgGw;
  const GdGeom g = moeg_geom(q.NG, q.rows, row0);
  unsigned char* wreg = smem + warp * L.warp_bytes;
  unsigned char* wts = wreg;
  float* scl = reinterpret_cast<float*>(wreg + gd_layout<1, moed::kWarps>(moed::kTw, q.NG, q.P, 1, 0, q.NG).scl);
  uint32_t* xs = reinterpret_cast<uint32_t*>(smem + L.xs);
  float* red = reinterpret_cast<float*>(smem + L.red);
  // the expert's rows, staged once for all its routes
  uint16_t sreg[kGdSpl];
  if (g.busy) gd_stage<1>(p, g, wts, lane);
  else cp_async_commit();
  gd_load_scales<1>(p, g, 0, lane, sreg);
  gd_finish_scales<1>(p, g, lane, sreg, scl);
  cp_async_wait_all();
  for (int c0 = 0; c0 < cnt; c0 += moeg::kBatch) {
    const int nb = min(moeg::kBatch, cnt - c0);
    if (threadIdx.x < nb) {
      const int r = gl.sroute[st0 + c0 + threadIdx.x];
      route[threadIdx.x] = r;
      xrow[threadIdx.x] = GATEUP ? r / q.top_k : r;  // gate/up reads the token, down the route's h
    }
    __syncthreads();  // staged rows and scales, and the batch's rows, visible to all warps
    auto emit = [&](int i, int b, const float* rd) {
      const int row = blockIdx.x * rows_cta + i;
      if (row >= q.rows) return;
      if (GATEUP) {
        const int wg = i >> 4, rr = i & 15;
        const float* rg = rd + (wg * 16 + rr) * moeg::kRedCols + 3 * b;
        const float* ru = rd + ((wg + 4) * 16 + rr) * moeg::kRedCols + 3 * b;
        const float gv = (rg[0] + rg[1]) + rg[2], uv = (ru[0] + ru[1]) + ru[2];
        q.h[static_cast<int64_t>(route[b]) * q.rows + row] = __float2bfloat16_rn(gv / (1.0f + expf(-gv)) * uv);
      } else {
        const float* rv = rd + i * moeg::kRedCols + 3 * b;
        const int r = route[b];
        rout[static_cast<int64_t>(r) * q.rows + row] = q.wts[r] * ((rv[0] + rv[1]) + rv[2]);
      }
    };
    switch (nb) {  // uniform over the CTA
      case 1: moeg_batch<1>(p, g, wts, scl, xs, red, warp, lane, rows_cta, emit); break;
      case 2: moeg_batch<2>(p, g, wts, scl, xs, red, warp, lane, rows_cta, emit); break;
      case 3: moeg_batch<3>(p, g, wts, scl, xs, red, warp, lane, rows_cta, emit); break;
      default: moeg_batch<4>(p, g, wts, scl, xs, red, warp, lane, rows_cta, emit); break;
    }
  }
}

// The grouped decode layer: list, gate/up, down, combine (four launches).
static cudaError_t launch_moe_decode_grouped(MoeDecParams q, int T, int H, int I, MoeGroupList gl,
                                             const uint32_t* ds, const uint16_t* dc, float* rout, int* pos,
                                             float* out, cudaStream_t stream, int num_sms) {
  auto lg2 = [](int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
  };
  cudaError_t err = launch_pdl(moe_decode_list_kernel, dim3(1), dim3(512), 0, stream, q.logits, T, q.E, q.top_k,
                               q.ids, q.wts, pos, gl);
  if (err != cudaSuccess) return err;
  const unsigned slots = static_cast<unsigned>(q.E < q.R ? q.E : q.R);  // most experts a call can touch
  // gate/up (+ SwiGLU): K = H, rows = I
  MoeDecParams qg = q;
  qg.rows = I;
  qg.K = H;
  qg.NG = H / 128;
  qg.P = ((qg.NG & 1) ? qg.NG : qg.NG + 1) * 16;  // odd multiple of 16 bytes per staged row: bank spread
  qg.lgGw = lg2(qg.NG);
  int smem = moeg_layout(qg.NG, qg.P).total;
  err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_decode_grouped_kernel<true>), smem);
  if (err != cudaSuccess) return err;
  err = launch_pdl(moe_decode_grouped_kernel<true>,
                   dim3(static_cast<unsigned>((I + moed::kRowsGu - 1) / moed::kRowsGu), slots),
                   dim3(moed::kWarps * 32), static_cast<size_t>(smem), stream, qg, gl, rout);
  if (err != cudaSuccess) return err;
  // down (x the route weight): K = I, rows = H, x = h [R][I]
  MoeDecParams qd = q;
  qd.x = reinterpret_cast<const uint16_t*>(q.h);
  qd.signs0 = ds;
  qd.scales0 = dc;
  qd.signs1 = nullptr;
  qd.scales1 = nullptr;
  qd.rows = H;
  qd.K = I;
  qd.NG = I / 128;
  qd.P = ((qd.NG & 1) ? qd.NG : qd.NG + 1) * 16;
  qd.lgGw = lg2(qd.NG);
  smem = moeg_layout(qd.NG, qd.P).total;
  err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_decode_grouped_kernel<false>), smem);
  if (err != cudaSuccess) return err;
  err = launch_pdl(moe_decode_grouped_kernel<false>,
                   dim3(static_cast<unsigned>((H + moeg::kRowsD - 1) / moeg::kRowsD), slots),
                   dim3(moed::kWarps * 32), static_cast<size_t>(smem), stream, qd, gl, rout);
  if (err != cudaSuccess) return err;
  // out[t] = its slots in slot order
  const int64_t total4 = static_cast<int64_t>(T) * (H / 4);
  int64_t blocks = (total4 + 255) / 256;
  if (blocks > 8 * num_sms) blocks = 8 * num_sms;
  return launch_pdl(moe_combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                    static_cast<const float*>(rout), static_cast<const int*>(pos), T, H, q.top_k, out);
}

static cudaError_t launch_moe_decode_down(MoeDecParams q, int T, float* out, cudaStream_t stream) {
  auto lg2 = [](int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
  };
  q.lgGw = lg2(q.NG);
  // rows per CTA: 16 x (tokens rounded down to a power of two, at most 8),
  // halved while the shared memory would not fit
  int RB = 16;
  while (RB < 128 && 2 * RB <= 16 * T) RB *= 2;
  while (RB > 16 && moe_down_layout(q.NG, RB).total > moed::kSmemCap) RB /= 2;
  const int smem = moe_down_layout(q.NG, RB).total;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_decode_down_kernel), smem);
  if (err != cudaSuccess) return err;
  const dim3 grid(static_cast<unsigned>((q.rows + RB - 1) / RB), static_cast<unsigned>(T));
  return launch_pdl(moe_decode_down_kernel, grid, dim3(moed::kWarps * 32), static_cast<size_t>(smem), stream, q,
                    RB, out);
}

static cudaError_t launch_moe_decode_gateup(MoeDecParams q, cudaStream_t stream, int num_sms) {
  auto lg2 = [](int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
  };
  q.P = ((q.NG & 1) ? q.NG : q.NG + 1) * 16;  // odd multiple of 16 bytes per staged row: bank spread
  q.lgGw = lg2(q.NG);
  // 128 rows per CTA where that gives between one and two CTAs per SM, else
  // 64 (moe_tw knob: 2 or 4 n-tiles per warp).  Measured on the OLMoE-like
  // layer (us per layer, 64 / 128 rows): 2 tokens 24.6 / 26.1 (64 CTAs of
  // 128 rows), 4 tokens 36.9 / 34.8 (256), 8 tokens 54.3 / 56.3 (512).
  const int tk = knob(kKnobMoeTw);
  const int64_t ctas128 = static_cast<int64_t>((q.rows + 127) / 128) * q.R;
  const bool wide = tk ? tk == 4
                       : ctas128 >= num_sms && ctas128 < 2 * static_cast<int64_t>(num_sms) &&
                             moed_layout(q, 4).total <= moed::kSmemCap;
  if (wide) {
    const int smem = moed_layout(q, 4).total;
    cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_decode_gateup_kernel<4>), smem);
    if (err != cudaSuccess) return err;
    const dim3 grid(static_cast<unsigned>((q.rows + 127) / 128), static_cast<unsigned>(q.R));
    return launch_pdl(moe_decode_gateup_kernel<4>, grid, dim3(moed::kWarps * 32), static_cast<size_t>(smem), stream, q);
  }
  const int smem = moed_layout(q).total;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_decode_gateup_kernel<moed::kTw>), smem);
  if (err != cudaSuccess) return err;
  const dim3 grid(static_cast<unsigned>((q.rows + moed::kRowsGu - 1) / moed::kRowsGu), static_cast<unsigned>(q.R));
  return launch_pdl(moe_decode_gateup_kernel<moed::kTw>, grid, dim3(moed::kWarps * 32), static_cast<size_t>(smem),
                    stream, q);
}

cudaError_t launch_moe(const uint16_t* x, const float* logits, int64_t T, int64_t H, int64_t I, int E, int top_k,
                       const uint32_t* gs, const uint16_t* gc, const uint32_t* us, const uint16_t* uc,
                       const uint32_t* ds, const uint16_t* dc, float* out, void* workspace, cudaStream_t stream,
                       int num_sms) {
  const moe::Workspace L = moe::workspace_layout(T, H, I, E, top_k);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int* hdr = reinterpret_cast<int*>(ws + L.hdr);
  int* ids = reinterpret_cast<int*>(ws + L.ids);
  float* wts = reinterpret_cast<float*>(ws + L.wts);
  int* pos = reinterpret_cast<int*>(ws + L.pos);
  int* sroute = reinterpret_cast<int*>(ws + L.sroute);
  int* stok = reinterpret_cast<int*>(ws + L.stok);
  int* offsets = reinterpret_cast<int*>(ws + L.offsets);
  moe::Tile* tiles_gu = reinterpret_cast<moe::Tile*>(ws + L.tiles_gu);
  moe::Tile* tiles_d = reinterpret_cast<moe::Tile*>(ws + L.tiles_d);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  float* rout = reinterpret_cast<float*>(ws + L.rout);
  const int R = static_cast<int>(T * top_k);

  cudaError_t err;
  // Decode regime: a few tokens, about one route per expert -> per-route
  // products on the direct GEMV steps: gate/up (with the routing up to 4
  // tokens), down with the combine.  Measured on the OLMoE-like layer: about 2x faster
  // than the tile pipeline up to 8 tokens, still ahead at 16.
  // The moe_path knob (tiles | decode) forces a path for testing.
  constexpr int64_t kDecodeMaxT = 16;
  const int mpath = knob(kKnobMoePath);
  bool decode = (mpath ? (mpath == 2 || mpath == 3) : T <= kDecodeMaxT) && H / 128 <= gd::kMaxSets &&
                I / 128 <= gd::kMaxSets;
  if (decode) {  // both decode kernels' shared memory must fit
    MoeDecParams qg = {};
    qg.NG = static_cast<int>(H / 128);
    qg.P = ((qg.NG & 1) ? qg.NG : qg.NG + 1) * 16;
    decode = moed_layout(qg).total <= moed::kSmemCap &&
             moe_down_layout(static_cast<int>(I / 128), 16).total <= moed::kSmemCap;
  }
  if (decode) {
    // up to 4 tokens each CTA routes its token (one launch less); above,
    // the router kernel does it once per token.  From 9 tokens the grouped
    // form (one product per touched expert, its routes as the batch rows)
    // replaces the per-route products; the moe_path knob forces either.
    constexpr int64_t kSelfRouteMaxT = 4;
    auto pad16 = [](int ng) { return ((ng & 1) ? ng : ng + 1) * 16; };
    const int ngh = static_cast<int>(H / 128), ngi = static_cast<int>(I / 128);
    // Grouped by default from 9 tokens on: measured on the OLMoE-like layer
    // (graph replays, L2 flushed), 74.8 vs 93.0 us at 16 tokens, 57.3 vs
    // 54.3 at 8, slower below (20.5 / 29.7 us at 1 token: two launches more).
    constexpr int64_t kGroupedMinT = 9;
    const bool want_grouped = mpath ? mpath == 3 : T >= kGroupedMinT;
    const bool grouped = want_grouped && T <= moeg::kMaxT && moeg_layout(ngh, pad16(ngh)).total <= moed::kSmemCap &&
                         moeg_layout(ngi, pad16(ngi)).total <= moed::kSmemCap;
    MoeDecParams q = {};
    q.logits = logits;
    q.E = E;
    q.self_route = T <= kSelfRouteMaxT && !grouped ? 1 : 0;
    if (!q.self_route && !grouped) {
      float* xcs = reinterpret_cast<float*>(ws + L.xcs);
      err = launch_pdl(moe_route_kernel, dim3(static_cast<unsigned>((T + 7) / 8)), dim3(256), 0, stream, logits,
                       static_cast<int>(T), E, top_k, ids, wts, x, static_cast<int>(H), xcs);
      if (err != cudaSuccess) return err;
    }
    q.ids = ids;
    q.wts = wts;
    q.x = x;
    q.signs0 = gs;
    q.scales0 = gc;
    q.signs1 = us;
    q.scales1 = uc;
    q.h = h;
    q.pos = pos;
    q.R = R;
    q.top_k = top_k;
    q.rows = static_cast<int>(I);
    q.K = static_cast<int>(H);
    q.NG = static_cast<int>(H / 128);
    if (grouped) {
      int* tl = reinterpret_cast<int*>(ws + L.tiles_gu);
      const MoeGroupList gl{hdr, offsets, tl, tl + E, sroute};
      return launch_moe_decode_grouped(q, static_cast<int>(T), static_cast<int>(H), static_cast<int>(I), gl, ds, dc,
                                       rout, pos, out, stream, num_sms);
    }
    err = launch_moe_decode_gateup(q, stream, num_sms);
    if (err != cudaSuccess) return err;
    MoeDecParams qd = q;
    qd.x = reinterpret_cast<const uint16_t*>(h);
    qd.signs0 = ds;
    qd.scales0 = dc;
    qd.signs1 = nullptr;
    qd.scales1 = nullptr;
    qd.rows = static_cast<int>(H);
    qd.K = static_cast<int>(I);
    qd.NG = static_cast<int>(I / 128);
    return launch_moe_decode_down(qd, static_cast<int>(T), out, stream);
  }
  // 1. router
  float* xcs = reinterpret_cast<float*>(ws + L.xcs);
  err = launch_pdl(moe_route_kernel, dim3(static_cast<unsigned>((T + 7) / 8)), dim3(256), 0, stream, logits,
                   static_cast<int>(T), E, top_k, ids, wts, x, static_cast<int>(H), xcs);
  if (err != cudaSuccess) return err;
  // 2. sort + tile lists
  constexpr int kStageMax = 16384;  // routes staged in shared memory (64 KB)
  SortArgs sa{ids,  R,   E,       top_k,    static_cast<int>(I / 128), static_cast<int>(H / 128), offsets, sroute,
              stok, pos, tiles_gu, tiles_d, hdr, R <= kStageMax ? 1 : 0};
  const int sort_smem = sa.stage ? 4 * R : 0;
  if (sort_smem > 0) {
    err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_sort_kernel), sort_smem);
    if (err != cudaSuccess) return err;
  }
  err = launch_pdl(moe_sort_kernel, dim3(1), dim3(1024), static_cast<size_t>(sort_smem), stream, sa);
  if (err != cudaSuccess) return err;
  __half* xs = reinterpret_cast<__half*>(ws + L.xs);
  float* xscale = reinterpret_cast<float*>(ws + L.xscale);
  __half* hs = reinterpret_cast<__half*>(ws + L.hs);
  float* hscale = reinterpret_cast<float*>(ws + L.hscale);
  // 3. x rows in sorted route order, fp16 with a power of two per route
  err = launch_pdl(moe_gather_kernel, dim3(static_cast<unsigned>((R + 7) / 8)), dim3(256), 0, stream, x, stok,
                   static_cast<const float*>(xcs), R, static_cast<int>(H), xs, xscale);
  if (err != cudaSuccess) return err;
  // 4. gate/up with fused SwiGLU
  {
    CUtensorMap tm;
    if (!make_tmap_bf16_sw128(&tm, xs, R, H, moe::TN_GU)) return cudaErrorInvalidValue;
    MoeGemmParams p = {};
    p.a_signs = gs;
    p.a_scales = gc;
    p.u_signs = us;
    p.u_scales = uc;
    p.tiles = tiles_gu;
    p.hdr = hdr;
    p.stok = stok;
    p.sroute = sroute;
    p.wts = wts;
    p.rscale = xscale;
    p.h = h;
    p.rows = static_cast<int>(I);
    p.K = static_cast<int>(H);
    p.out_ld = static_cast<int>(I);
    const size_t smem = sizeof(MoeSmem<true>) + 1024;
    err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_gemm_kernel<true>), static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = L.max_tiles_gu < num_sms ? L.max_tiles_gu : num_sms;
    err = launch_pdl(moe_gemm_kernel<true>, dim3(grid), dim3(moe::kThreads), smem, stream, tm, p);
    if (err != cudaSuccess) return err;
  }
  // 5. h -> fp16 with a power of two per route
  err = launch_pdl(moe_hprep_kernel, dim3(static_cast<unsigned>((R + 7) / 8)), dim3(256), 0, stream,
                   reinterpret_cast<const uint16_t*>(h), R, static_cast<int>(I), hs, hscale);
  if (err != cudaSuccess) return err;
  // 6. down with route weights
  {
    CUtensorMap tm;
    if (!make_tmap_bf16_sw128(&tm, hs, R, I, moe::TN_D)) return cudaErrorInvalidValue;
    MoeGemmParams p = {};
    p.a_signs = ds;
    p.a_scales = dc;
    p.tiles = tiles_d;
    p.hdr = hdr;
    p.stok = stok;
    p.sroute = sroute;
    p.wts = wts;
    p.rscale = hscale;
    p.rout = rout;
    p.rows = static_cast<int>(H);
    p.K = static_cast<int>(I);
    p.out_ld = static_cast<int>(H);
    const size_t smem = sizeof(MoeSmem<false>) + 1024;
    err = ensure_dyn_smem(reinterpret_cast<const void*>(moe_gemm_kernel<false>), static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = L.max_tiles_d < num_sms ? L.max_tiles_d : num_sms;
    err = launch_pdl(moe_gemm_kernel<false>, dim3(grid), dim3(moe::kThreads), smem, stream, tm, p);
    if (err != cudaSuccess) return err;
  }
  // 5. combine
  {
    const int64_t total4 = T * (H / 4);
    int64_t blocks = (total4 + 255) / 256;
    if (blocks > 8 * num_sms) blocks = 8 * num_sms;
    err = launch_pdl(moe_combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, rout, pos,
                     static_cast<int>(T), static_cast<int>(H), top_k, out);
  }
  return err;
}

}  // namespace w1

// ------------------------------------------------------------------ C entry points
extern "C" {

size_t w1_moe_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int64_t top_k) {
  if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || top_k <= 0 || E > w1::moe::kMaxE || top_k > E) return 0;
  return w1::moe_workspace_bytes(T, H, I, static_cast<int>(E), static_cast<int>(top_k));
}

int w1_moe_grouped(const uint16_t* x, const float* router_logits, int64_t T, int64_t H, int64_t I, int64_t E,
                   int64_t top_k, const uint32_t* gate_signs, const uint16_t* gate_scales, const uint32_t* up_signs,
                   const uint16_t* up_scales, const uint32_t* down_signs, const uint16_t* down_scales, float* out,
                   void* workspace, size_t ws_bytes, w1_stream_t stream) {
  using namespace w1;
  if (!x || !router_logits || !gate_signs || !gate_scales || !up_signs || !up_scales || !down_signs ||
      !down_scales || !out)
    return W1_ERR_NULL;
  if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || top_k <= 0 || top_k > E || E > moe::kMaxE ||
      top_k > moe::kMaxTopK || (H % 128) != 0 || (I % 128) != 0)
    return W1_ERR_SHAPE;
  if (T * top_k > (int64_t)1 << 26 || T * top_k * H > (int64_t)1 << 40) return W1_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(router_logits) || !aligned16(gate_signs) || !aligned16(gate_scales) ||
      !aligned16(up_signs) || !aligned16(up_scales) || !aligned16(down_signs) || !aligned16(down_scales) ||
      !aligned16(out))
    return W1_ERR_ALIGN;
  if (!workspace || ws_bytes < moe_workspace_bytes(T, H, I, static_cast<int>(E), static_cast<int>(top_k)))
    return W1_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 1023u) != 0) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_moe(x, router_logits, T, H, I, static_cast<int>(E), static_cast<int>(top_k),
                                  gate_signs, gate_scales, up_signs, up_scales, down_signs, down_scales, out,
                                  workspace, reinterpret_cast<cudaStream_t>(stream), d.sms));
}

}  // extern "C"

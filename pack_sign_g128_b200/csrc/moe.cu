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
// Five launches on one stream (programmatic dependent launch between them):
//  1. route_kernel     warp per token: fp32 softmax, top-k by logit, weights.
//  2. sort_kernel      one CTA: stable counting sort of the routes by expert
//                      (deterministic), route -> sorted position map, and the
//                      tile lists of the two grouped GEMMs (no empty tiles).
//  3. moe_gemm<GATEUP> tcgen05 grouped GEMM, swap-AB as in w1_gemm: the gate
//                      and up rows of expert e (TMEM, +-1 bf16) times token
//                      rows gathered from x by TMA tile::gather4 (x is never
//                      duplicated per route); the epilogue applies the group
//                      scales, SiLU(g) * u and stores h (bf16) in sorted order.
//  4. moe_gemm<DOWN>   the down rows of expert e times h rows (contiguous per
//                      expert); epilogue multiplies by the route weight and
//                      stores the route output (fp32, sorted order).
//  5. combine_kernel   out[t] = sum over slots, in slot order.
// MMA N (tokens per tile) is set per tile from the expert's route count
// (rounded up to 16), so partially filled tiles cost only what they hold.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "w1_common.cuh"

namespace w1 {

bool make_tmap_bf16_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows);

namespace moe {
constexpr int TN_GU = 64;    // routes per gate/up tile
constexpr int TN_D = 128;    // routes per down tile
constexpr int kMaxE = 256;
constexpr int kMaxTopK = 32;
constexpr int kThreads = 320;

struct Tile {
  int e, rt, start, count;  // expert, 128-row tile, first sorted route, routes
};

struct Workspace {
  size_t hdr, ids, wts, pos, sroute, stok, offsets, tiles_gu, tiles_d, h, rout, total;
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
  off = align_up(off + 4 * static_cast<size_t>(R) * H, 256);
  w.total = off;
  return w;
}
}  // namespace moe

// ------------------------------------------------------------------ 1. router

// One warp per token.  Selection is by logit (the softmax is monotone, so this
// is selection by probability without rounding ties); weights are fp32.
__global__ void __launch_bounds__(256) moe_route_kernel(const float* __restrict__ logits, int T, int E, int top_k,
                                                        int* __restrict__ ids, float* __restrict__ wts) {
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp < T) {
    constexpr int PER = moe::kMaxE / 32;
    float z[PER];
    const float* lp = logits + static_cast<int64_t>(warp) * E;
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
        ids[warp * top_k + s] = be;
        wts[warp * top_k + s] = expf(bz - mx) / sum;
      }
      if ((be & 31) == lane) z[be >> 5] = -INFINITY;  // taken
    }
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ 2. sort + tiles

// Block-wide exclusive scan of v over threads [0, n) (n <= blockDim.x <= 1024).
__device__ inline int block_exclusive_scan(int v, int* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int w = (lane < nw) ? tmp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < nw) tmp[32 + lane] = wi - w;
  }
  __syncthreads();
  const int r = incl - v + tmp[32 + warp];
  __syncthreads();
  return r;
}

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
};

// One CTA of 1024 threads.  Warp w owns the contiguous route segment
// [w L, (w+1) L); positions inside an expert follow route order (stable).
__global__ void __launch_bounds__(1024) moe_sort_kernel(const SortArgs a) {
  __shared__ int cnt[moe::kMaxE];
  __shared__ int tbl[32][moe::kMaxE];
  __shared__ int tmp[64];
  __shared__ int offs[moe::kMaxE + 1];
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * moe::kMaxE; i += blockDim.x) (&tbl[0][0])[i] = 0;
  __syncthreads();
  const int L = (a.R + 31) / 32;
  const int s0 = warp * L, s1 = min(a.R, s0 + L);
  // per-(warp, expert) counts
  for (int base = s0; base < s1; base += 32) {
    const int r = base + lane;
    const int e = (r < s1) ? a.ids[r] : -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    if (e >= 0 && (__ffs(peers) - 1) == lane) tbl[warp][e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // expert totals and offsets
  int c = 0;
  if (threadIdx.x < a.E)
    for (int w = 0; w < 32; ++w) c += tbl[w][threadIdx.x];
  const int off = block_exclusive_scan(threadIdx.x < a.E ? c : 0, tmp);
  if (threadIdx.x < a.E) {
    cnt[threadIdx.x] = c;
    offs[threadIdx.x] = off;
    a.offsets[threadIdx.x] = off;
    int run = off;
    for (int w = 0; w < 32; ++w) {
      const int t = tbl[w][threadIdx.x];
      tbl[w][threadIdx.x] = run;
      run += t;
    }
    if (threadIdx.x == a.E - 1) {
      offs[a.E] = run;
      a.offsets[a.E] = run;
    }
  }
  __syncthreads();
  // stable scatter
  for (int base = s0; base < s1; base += 32) {
    const int r = base + lane;
    const int e = (r < s1) ? a.ids[r] : -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    if (e >= 0) {
      const int p = tbl[warp][e] + __popc(peers & ((1u << lane) - 1u));
      a.sroute[p] = r;
      a.stok[p] = r / a.top_k;
      a.pos[r] = p;
    }
    __syncwarp();
    if (e >= 0 && (__ffs(peers) - 1) == lane) tbl[warp][e] += __popc(peers);
    __syncwarp();
  }
  // tile lists: expert-major, every tile holds >= 1 route
  const int e = threadIdx.x;
  const int ce = (e < a.E) ? cnt[e] : 0;
  const int ngu = (ce + moe::TN_GU - 1) / moe::TN_GU, nd = (ce + moe::TN_D - 1) / moe::TN_D;
  const int bgu = block_exclusive_scan(e < a.E ? ngu * a.rt_gu : 0, tmp);
  const int bd = block_exclusive_scan(e < a.E ? nd * a.rt_d : 0, tmp);
  if (e < a.E) {
    int k = bgu;
    for (int j = 0; j < ngu; ++j)
      for (int rt = 0; rt < a.rt_gu; ++rt)
        a.tiles_gu[k++] = moe::Tile{e, rt, offs[e] + j * moe::TN_GU, min(moe::TN_GU, ce - j * moe::TN_GU)};
    k = bd;
    for (int j = 0; j < nd; ++j)
      for (int rt = 0; rt < a.rt_d; ++rt)
        a.tiles_d[k++] = moe::Tile{e, rt, offs[e] + j * moe::TN_D, min(moe::TN_D, ce - j * moe::TN_D)};
    if (e == a.E - 1) {  // totals = last exclusive prefix + last expert's tiles
      a.hdr[0] = bgu + ngu * a.rt_gu;
      a.hdr[1] = bd + nd * a.rt_d;
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
  __nv_bfloat16* h;          // gate/up output [R][I]
  float* rout;               // down output [R][H]
  int rows;                  // rows of each expert matrix (I for gate/up, H for down)
  int K;                     // contracted size (H for gate/up, I for down)
  int out_ld;                // leading dimension of the output
};

template <bool GATEUP>
struct MoeCfg {
  static constexpr int TN = GATEUP ? moe::TN_GU : moe::TN_D;
  static constexpr int NMAT = GATEUP ? 2 : 1;                 // A matrices per tile
  static constexpr int NSX = 4;                               // X stages
  static constexpr int NSA = GATEUP ? 2 : 4;                  // A stages (64 cols per matrix)
  static constexpr int XSTAGE = TN * 128 * 2;                 // bytes of one X stage
  static constexpr uint32_t ACOL0 = 2 * NMAT * TN;            // chunk buffers first
  static constexpr uint32_t ASTRIDE = NMAT * 64;              // TMEM cols per A stage
};

template <bool GATEUP>
struct MoeSmem {
  alignas(1024) unsigned char x[MoeCfg<GATEUP>::NSX][MoeCfg<GATEUP>::XSTAGE];
  uint64_t full_x[MoeCfg<GATEUP>::NSX], empty_x[MoeCfg<GATEUP>::NSX];
  uint64_t full_a[MoeCfg<GATEUP>::NSA], empty_a[MoeCfg<GATEUP>::NSA];
  uint64_t full_c[2], empty_c[2];
  int rows_idx[MoeCfg<GATEUP>::TN];
  uint32_t tmem_base;
};

__device__ __forceinline__ void tma_gather4(void* smem_dst, const void* tmap, int32_t col, int32_t r0, int32_t r1,
                                            int32_t r2, int32_t r3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4, %5, %6}], [%7];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t expand_pair(uint32_t w, int pp) {
  // bf16 pair for columns (2pp, 2pp+1) of a 32-bit sign word: sign bits to 15 / 31
  const uint32_t src = (pp < 8) ? w : (w >> 16);
  const int b = 2 * (pp & 7);
  const uint32_t m = src & (3u << b);
  const uint32_t t = m * (0x40008000u >> b);
  return (t & 0x80008000u) | 0x3F803F80u;
}

template <bool GATEUP>
__global__ void __launch_bounds__(moe::kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const MoeGemmParams p) {
  using C = MoeCfg<GATEUP>;
  extern __shared__ unsigned char smem_raw[];
  MoeSmem<GATEUP>& sm =
      *reinterpret_cast<MoeSmem<GATEUP>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSX; ++i) {
      mbar_init(&sm.full_x[i], 1);
      mbar_init(&sm.empty_x[i], 1);
    }
    for (int i = 0; i < C::NSA; ++i) {
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
  const int ntiles = p.hdr[GATEUP ? 0 : 1];
  const int NK = p.K >> 7;

  if (warp == 0) {
    // ---------------------------------------- producer: token rows of X
    uint32_t c = 0;
    for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
      const moe::Tile tl = p.tiles[ti];
      if (GATEUP) {
        // gather indices of this tile (rows past the count repeat the first)
        __syncwarp();
        for (int j = lane; j < C::TN; j += 32) sm.rows_idx[j] = p.stok[tl.start + (j < tl.count ? j : 0)];
        __syncwarp();
      }
      for (int kc = 0; kc < NK; ++kc, ++c) {
        const int s = c % C::NSX;
        if (!mbar_wait_warp(&sm.empty_x[s], ((c / C::NSX) & 1) ^ 1)) goto done_prod;
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.full_x[s], C::XSTAGE);
          if (GATEUP) {
#pragma unroll 1
            for (int half = 0; half < 2; ++half)
#pragma unroll 1
              for (int q = 0; q < C::TN / 4; ++q)
                tma_gather4(sm.x[s] + half * (C::XSTAGE / 2) + q * 512, &tmap_b, kc * 128 + half * 64,
                            sm.rows_idx[4 * q], sm.rows_idx[4 * q + 1], sm.rows_idx[4 * q + 2],
                            sm.rows_idx[4 * q + 3], &sm.full_x[s]);
          } else {
            tma_load_2d(sm.x[s], &tmap_b, kc * 128, tl.start, &sm.full_x[s]);
            tma_load_2d(sm.x[s] + C::XSTAGE / 2, &tmap_b, kc * 128 + 64, tl.start, &sm.full_x[s]);
          }
        }
        __syncwarp();
      }
    }
  done_prod:;
  } else if (warp == 1) {
    // ---------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t c = 0;
      for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
        const moe::Tile tl = p.tiles[ti];
        const int n_mma = ((tl.count + 15) >> 4) << 4;
        const uint32_t idesc = idesc_f16(128, n_mma, 1, 1);
        for (int kc = 0; kc < NK; ++kc, ++c) {
          const int sx = c % C::NSX, sa = c % C::NSA, cb = c & 1;
          if (!mbar_wait(&sm.full_x[sx], (c / C::NSX) & 1)) goto done_mma;
          if (!mbar_wait(&sm.full_a[sa], (c / C::NSA) & 1)) goto done_mma;
          if (!mbar_wait(&sm.empty_c[cb], ((c >> 1) & 1) ^ 1)) goto done_mma;
          tc_fence_after();
          const uint32_t xbase = smem_u32(sm.x[sx]);
#pragma unroll
          for (int mat = 0; mat < C::NMAT; ++mat) {
            const uint32_t d = tmem + cb * (C::NMAT * C::TN) + mat * C::TN;
            const uint32_t a = tmem + C::ACOL0 + sa * C::ASTRIDE + mat * 64;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t baddr = xbase + (kk >> 2) * (C::XSTAGE / 2) + (kk & 3) * 32;
              tc_mma_ts(d, a + kk * 8, smem_desc_sw128(baddr), idesc, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(&sm.empty_x[sx]);
          tc_commit(&sm.empty_a[sa]);
          tc_commit(&sm.full_c[cb]);
        }
      }
    done_mma:;
    }
  } else if (warp < 6) {
    // ---------------------------------------- expanders: thread = weight row
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t wrow = p.K >> 5;
    uint32_t c = 0;
    for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
      const moe::Tile tl = p.tiles[ti];
      const int row = tl.rt * 128 + rl;
      const bool valid = row < p.rows;
      const int64_t ridx = static_cast<int64_t>(tl.e) * p.rows + (valid ? row : 0);
      const uint4* wa = reinterpret_cast<const uint4*>(p.a_signs + ridx * wrow);
      const uint4* wu = GATEUP ? reinterpret_cast<const uint4*>(p.u_signs + ridx * wrow) : wa;
      uint4 na = valid ? __ldg(wa) : make_uint4(0, 0, 0, 0);
      uint4 nu = (GATEUP && valid) ? __ldg(wu) : make_uint4(0, 0, 0, 0);
      for (int kc = 0; kc < NK; ++kc, ++c) {
        const uint4 ca = na, cu = nu;
        if (kc + 1 < NK && valid) {
          na = __ldg(wa + kc + 1);
          if (GATEUP) nu = __ldg(wu + kc + 1);
        }
        const int sa = c % C::NSA;
        if (!mbar_wait_warp(&sm.empty_a[sa], ((c / C::NSA) & 1) ^ 1)) goto done_exp;
        tc_fence_after();
#pragma unroll
        for (int mat = 0; mat < C::NMAT; ++mat) {
          const uint4 cw = mat ? cu : ca;
          const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t r[32];
#pragma unroll
            for (int wi = 0; wi < 2; ++wi)
#pragma unroll
              for (int pp = 0; pp < 16; ++pp) r[wi * 16 + pp] = expand_pair(words[half * 2 + wi], pp);
            tmem_st32(tmem + lane_addr + C::ACOL0 + sa * C::ASTRIDE + mat * 64 + half * 32, r);
          }
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.full_a[sa]);
      }
    }
  done_exp:;
  } else {
    // ---------------------------------------- promoters + epilogue: thread = weight row
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int NG = p.K >> 7;
    uint32_t c = 0;
    for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
      const moe::Tile tl = p.tiles[ti];
      const int row = tl.rt * 128 + rl;
      const bool valid = row < p.rows;
      const int64_t ridx = static_cast<int64_t>(tl.e) * p.rows + (valid ? row : 0);
      const uint16_t* sa_p = p.a_scales + ridx * NG;
      const uint16_t* su_p = GATEUP ? p.u_scales + ridx * NG : sa_p;
      float acc[C::NMAT][C::TN];
#pragma unroll
      for (int mat = 0; mat < C::NMAT; ++mat)
#pragma unroll
        for (int j = 0; j < C::TN; ++j) acc[mat][j] = 0.f;
      const int nq = (tl.count + 31) >> 5;  // 32-column pieces holding routes
      uint16_t sa_next = valid ? __ldg(sa_p) : 0, su_next = (GATEUP && valid) ? __ldg(su_p) : 0;
      for (int kc = 0; kc < NK; ++kc, ++c) {
        const float s_a = __half2float(__ushort_as_half(sa_next));
        const float s_u = __half2float(__ushort_as_half(su_next));
        if (kc + 1 < NK && valid) {
          sa_next = __ldg(sa_p + kc + 1);
          if (GATEUP) su_next = __ldg(su_p + kc + 1);
        }
        const int cb = c & 1;
        if (!mbar_wait_warp(&sm.full_c[cb], (c >> 1) & 1)) goto done_prom;
        tc_fence_after();
#pragma unroll
        for (int mat = 0; mat < C::NMAT; ++mat) {
          const float s = mat ? s_u : s_a;
#pragma unroll
          for (int q4 = 0; q4 < C::TN / 32; ++q4) {
            if (q4 < nq) {
              uint32_t r[32];
              tmem_ld32(tmem + lane_addr + cb * (C::NMAT * C::TN) + mat * C::TN + q4 * 32, r);
              tc_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) acc[mat][q4 * 32 + j] = fmaf(s, __uint_as_float(r[j]), acc[mat][q4 * 32 + j]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.empty_c[cb]);
      }
      if (valid) {
        if (GATEUP) {
          __nv_bfloat16* hp = p.h + static_cast<int64_t>(tl.start) * p.out_ld + row;
#pragma unroll
          for (int j = 0; j < C::TN; ++j) {
            if (j < tl.count) {
              const float g = acc[0][j];
              const float hv = g / (1.0f + expf(-g)) * acc[C::NMAT - 1][j];
              hp[static_cast<int64_t>(j) * p.out_ld] = __float2bfloat16_rn(hv);
            }
          }
        } else {
          float* op = p.rout + static_cast<int64_t>(tl.start) * p.out_ld + row;
#pragma unroll
          for (int j = 0; j < C::TN; ++j) {
            if (j < tl.count) {
              const float wgt = __ldg(p.wts + __ldg(p.sroute + tl.start + j));
              __stcs(op + static_cast<int64_t>(j) * p.out_ld, wgt * acc[0][j]);
            }
          }
        }
      }
    }
  done_prom:;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
  pdl_launch_dependents();
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
  // 1. router
  err = launch_pdl(moe_route_kernel, dim3(static_cast<unsigned>((T + 7) / 8)), dim3(256), 0, stream, logits,
                   static_cast<int>(T), E, top_k, ids, wts);
  if (err != cudaSuccess) return err;
  // 2. sort + tile lists
  SortArgs sa{ids, R, E, top_k, static_cast<int>(I / 128), static_cast<int>(H / 128), offsets, sroute, stok, pos,
              tiles_gu, tiles_d, hdr};
  err = launch_pdl(moe_sort_kernel, dim3(1), dim3(1024), 0, stream, sa);
  if (err != cudaSuccess) return err;
  // 3. gate/up with fused SwiGLU
  {
    CUtensorMap tm;
    if (!make_tmap_bf16_sw128(&tm, x, T, H, 1)) return cudaErrorInvalidValue;
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
    p.h = h;
    p.rows = static_cast<int>(I);
    p.K = static_cast<int>(H);
    p.out_ld = static_cast<int>(I);
    const size_t smem = sizeof(MoeSmem<true>) + 1024;
    err = cudaFuncSetAttribute(moe_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = L.max_tiles_gu < num_sms ? L.max_tiles_gu : num_sms;
    err = launch_pdl(moe_gemm_kernel<true>, dim3(grid), dim3(moe::kThreads), smem, stream, tm, p);
    if (err != cudaSuccess) return err;
  }
  // 4. down with route weights
  {
    CUtensorMap tm;
    if (!make_tmap_bf16_sw128(&tm, h, R, I, moe::TN_D)) return cudaErrorInvalidValue;
    MoeGemmParams p = {};
    p.a_signs = ds;
    p.a_scales = dc;
    p.tiles = tiles_d;
    p.hdr = hdr;
    p.stok = stok;
    p.sroute = sroute;
    p.wts = wts;
    p.rout = rout;
    p.rows = static_cast<int>(H);
    p.K = static_cast<int>(I);
    p.out_ld = static_cast<int>(H);
    const size_t smem = sizeof(MoeSmem<false>) + 1024;
    err = cudaFuncSetAttribute(moe_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
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

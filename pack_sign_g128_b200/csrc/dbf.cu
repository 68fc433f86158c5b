// dbf_apply: the Double Binary Factorization chain
//
//   y = a (.) ( B1 . ( mid (.) ( B2 . ( b (.) x ) ) ) )
//
// with B2 = V (r x n, input side) and B1 = U (m x r, output side) sign
// matrices (bit 0 -> +1, bit 1 -> -1) and fp16 diagonals a = D_out [m],
// mid = D_mid [r], b = D_in [n] ("LLM binarization episode 01: DBF",
// section 1 "The representation" and section 4: x_scaled = D_in x,
// h = V x_scaled, h_scaled = D_mid h, y_core = U h_scaled, y = D_out y_core).
//
// Small batch (B < 64, groups of up to 8 rows), two forms chosen by the group
// size:
//  * up to 4 rows: two launches of a GEMV core (the register-fed core of
//    gemv_flat.cu, or the direct core of gemv_direct.cu), h_scaled = mid (.)
//    (V . (b (.) x)) into the workspace, then y = a (.) (U . h_scaled) (its K
//    split over r is the pages' "split rank", section 5 item 5);
//  * from 5 rows: ONE kernel (the steps of the direct GEMV kernel) runs both
//    binary products -- the joint
//    V-D_mid-U kernel with a grid-wide synchronisation that the DBF post
//    (section 7, "CUDA/HIP: a starting point") proposes for CUDA.  Each CTA
//  1. issues the asynchronous copies of its slices of BOTH sign matrices at
//     once (two commit groups), so U streams in while V . (b x) is computed;
//  2. phase 1: int8-MMA product of V with b (.) x (the column diagonal applied
//     while quantising, exact in fp32), cluster reduction, h_scaled =
//     mid (.) h -> workspace (fp32);
//  3. grid barrier (bounded spin; on timeout W1_ERR_TIMEOUT, no hang);
//  4. phase 2: the same product of U with h_scaled (read through L2), y =
//     a (.) (...).
// The intermediate stays fp32 (exact to 2^-24 relative), so the only
// quantisation is the 23-bit fixed point of each product's input.
#include <cstdint>
#include <cuda_fp16.h>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "w1_common.cuh"

namespace w1 {

// Shared memory of the chain kernel: both products' per-warp regions (sign
// words, scales), then the activation scratch, reduction buffer and cluster
// inbox sized for the larger of the two.
struct DbfdSmem {
  int wb1, wb2, w1, w2, xs, red, part, total;
};

template <int NB, int NW>
__host__ __device__ inline DbfdSmem dbfd_layout(const GdParams& p1, const GdParams& p2) {
  using C = gd::Cfg<NB>;
  const GdSmem L1 = gd_layout<NB, NW>(p1.Tw, p1.NSw, p1.P, p1.S, p1.chunk, p1.NSc);
  const GdSmem L2 = gd_layout<NB, NW>(p2.Tw, p2.NSw, p2.P, p2.S, p2.chunk, p2.NSc);
  DbfdSmem M;
  M.wb1 = L1.warp_bytes;
  M.wb2 = L2.warp_bytes;
  M.w1 = 0;
  M.w2 = NW * M.wb1;
  M.xs = M.w2 + NW * M.wb2;
  const int nsc = p1.NSc > p2.NSc ? p1.NSc : p2.NSc;
  M.red = M.xs + (nsc * C::SCR * 4 + 15) / 16 * 16;
  const int tw = p1.Tw > p2.Tw ? p1.Tw : p2.Tw;
  M.part = M.red + gd::gd_red_bytes<NB, NW>(tw);
  const int chunk = p1.chunk > p2.chunk ? p1.chunk : p2.chunk;
  M.total = M.part + (p1.S > 1 ? p1.S * NB * chunk * 4 : 0);
  return M;
}

template <int NB, int NW>
__global__ void __launch_bounds__(NW * 32, 1) dbf_direct_kernel(const GdParams p1, const GdParams p2,
                                                                     unsigned int* bar) {
  extern __shared__ __align__(16) unsigned char smem[];
  const DbfdSmem M = dbfd_layout<NB, NW>(p1, p2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wr1 = smem + M.w1 + warp * M.wb1;
  unsigned char* wr2 = smem + M.w2 + warp * M.wb2;
  const GdSmem L1 = gd_layout<NB, NW>(p1.Tw, p1.NSw, p1.P, p1.S, p1.chunk, p1.NSc);
  const GdSmem L2 = gd_layout<NB, NW>(p2.Tw, p2.NSw, p2.P, p2.S, p2.chunk, p2.NSc);
  unsigned char* wts1 = wr1 + L1.wts;
  float* scl1 = reinterpret_cast<float*>(wr1 + L1.scl);
  unsigned char* wts2 = wr2 + L2.wts;
  float* scl2 = reinterpret_cast<float*>(wr2 + L2.scl);
  uint32_t* xs = reinterpret_cast<uint32_t*>(smem + M.xs);
  float* red = reinterpret_cast<float*>(smem + M.red);
  float* part = reinterpret_cast<float*>(smem + M.part);
  if (p1.S > 1) cluster_arrive_relaxed();  // matched by the wait before phase 1's first remote store
  const GdGeom g1 = gd_geom<NB>(p1, warp);
  const GdGeom g2 = gd_geom<NB>(p2, warp);
  pdl_wait();
  pdl_launch_dependents();
  // both sign matrices in flight at once: commit group 1 = V, group 2 = U
  if (g1.busy) gd_stage<NB>(p1, g1, wts1, lane);
  else cp_async_commit();
  if (g2.busy) gd_stage<NB>(p2, g2, wts2, lane);
  else cp_async_commit();
  uint4 xa[4];
  gd_x_first<NB, false>(p1, g1, warp, lane, xa);
  {
    uint16_t sreg[kGdSpl];  // no group scales: every s = 1
    gd_load_scales<NB>(p1, g1, 0, lane, sreg);
    gd_finish_scales<NB>(p1, g1, lane, sreg, scl1);
    gd_load_scales<NB>(p2, g2, 0, lane, sreg);
    gd_finish_scales<NB>(p2, g2, lane, sreg, scl2);
  }
  // ---- phase 1: h_scaled = mid (.) (V . (b (.) x))
  gd_prep_x<NB, false, NW>(p1, g1, xs, warp, lane, xa);
  asm volatile("cp.async.wait_group 1;" ::: "memory");  // V landed (U may still be in flight)
  __syncthreads();
  gd_finish<NB, NW>(p1, g1, wts1, scl1, xs, red, part, warp, lane, true);
  // ---- every CTA's h_scaled is in memory, and every reader of this CTA's
  // scratch and inbox is done with phase 1
  if (!grid_barrier(bar, gridDim.x)) {
    cp_async_wait_all();
    if (p2.S > 1) cluster_sync();  // the one cluster barrier phase 2 would have taken
    return;
  }
  // ---- phase 2: y = a (.) (U . h_scaled)
  gd_x_first<NB, true>(p2, g2, warp, lane, xa);
  gd_prep_x<NB, true, NW>(p2, g2, xs, warp, lane, xa);
  cp_async_wait_all();
  __syncthreads();
  gd_finish<NB, NW>(p2, g2, wts2, scl2, xs, red, part, warp, lane, false);
}

// ------------------------------------------------------------------ host side

// Plan of one product for a fixed cluster size S and cluster count Q (the chain
// kernel needs both products on the same grid).  False if a cluster's rows do
// not fit the warps.
template <int NB, int NW>
static bool dbfd_plan(int N, int NG, int S, int Q, GdParams* p) {
  using C = gd::Cfg<NB>;
  const int NT = (N + 7) / 8;
  const int NS = (NG + C::G - 1) / C::G;
  if (S > 1 && S > NS) return false;
  const int nsc = (NS + S - 1) / S;
  if (nsc > gd::kMaxSets) return false;
  const int Tmax = (NT + Q - 1) / Q;
  int Wn = 0;
  for (int w = 1; w <= NW; w *= 2)
    if ((Tmax + w - 1) / w <= gd::kMaxTw) {
      Wn = w;
      break;
    }
  if (Wn == 0) return false;
  auto lg2 = [](int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
  };
  p->N = N;
  p->NG = NG;
  p->K = NG * 128;
  p->S = S;
  p->Q = Q;
  p->NT = NT;
  p->Wn = Wn;
  p->Wg = NW / Wn;
  p->Tw = (Tmax + Wn - 1) / Wn;
  p->NSw = (nsc + p->Wg - 1) / p->Wg;
  const int span = p->NSw * 16 * C::G;
  p->P = ((span / (16 * C::G)) & 1) ? span : span + 16 * C::G;  // odd multiple: bank spread
  p->chunk = (8 * Tmax + S - 1) / S;
  p->NSc = nsc;
  p->lgS = lg2(S);
  p->lgWg = lg2(p->Wg);
  p->lgGw = lg2(p->NSw * C::G);
  p->tq = NT / Q;
  p->tr = NT - p->tq * Q;
  return true;
}

template <int NB, int NW>
static int dbfd_max_clusters(int S, int smem_bytes) {
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
  cfg.numAttrs = 1;
  int n = 0;
  if (ensure_dyn_smem(reinterpret_cast<const void*>(dbf_direct_kernel<NB, NW>), smem_bytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, dbf_direct_kernel<NB, NW>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// One group of up to 8 batch rows: the chain kernel on one grid whose CTAs are
// all co-resident (the grid barrier); among the K splits whose shared memory
// fits, the one with the least modelled per-CTA work (activation
// quantisation ~24 instructions per element of a CTA's K range, ~0.6-1.5 per
// weight, a fixed charge per cluster barrier; the GEMV planner's model).
template <int NB>
static double dbfd_cost(const GdParams& p) {
  using C = gd::Cfg<NB>;
  const double cw = NB <= 2 ? 0.35 : (NB <= 5 ? 1.0 : 1.2);
  const int Tmax = (p.NT + p.Q - 1) / p.Q;
  const double xprep = 24.0 * NB * 128.0 * C::G * p.NSc;
  const double wts = 8.0 * Tmax * 128.0 * C::G * p.NSc * cw;
  return (xprep + wts) / 128.0 + (p.S > 1 ? 800.0 : 0.0);
}

template <int NB, int NW>
static cudaError_t launch_dbf_small_nb(const uint16_t* a, const uint32_t* B1, const uint16_t* mid,
                                       const uint32_t* B2, const uint16_t* bd, int m, int r, int n,
                                       const uint16_t* x, float* y, float* h, unsigned int* bar,
                                       cudaStream_t stream, int num_sms, int smem_cap) {
  GdParams best1 = {}, best2 = {};
  int best_smem = 0;
  double best_cost = 0.0;
  for (int S = 1; S <= 8; S *= 2) {
    int Q = num_sms / S;
    for (int iter = 0; iter < 4; ++iter) {
      GdParams p1 = {}, p2 = {};
      if (!dbfd_plan<NB, NW>(r, n / 128, S, Q, &p1) || !dbfd_plan<NB, NW>(m, r / 128, S, Q, &p2)) break;
      const int smem = dbfd_layout<NB, NW>(p1, p2).total;
      if (smem > smem_cap) break;
      const int occ = dbfd_max_clusters<NB, NW>(S, smem);
      if (occ <= 0) break;
      if (occ < Q) {  // every CTA must be resident for the grid barrier
        Q = occ;
        continue;
      }
      const double cost = dbfd_cost<NB>(p1) + dbfd_cost<NB>(p2);
      if (best_smem == 0 || cost < best_cost) {
        best1 = p1;
        best2 = p2;
        best_smem = smem;
        best_cost = cost;
      }
      break;
    }
  }
  if (best_smem == 0) return cudaErrorNotSupported;  // no co-resident plan: the caller takes two launches
  GdParams p1 = best1, p2 = best2;
  const int smem = best_smem, S = p1.S, Q = p1.Q;
  p1.signs = B2;
  p1.x = x;
  p1.cdiag = bd;
  p1.rdiag = mid;
  p1.y = h;
  p2.signs = B1;
  p2.x = h;
  p2.x_f32 = 1;
  p2.rdiag = a;
  p2.y = y;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(dbf_direct_kernel<NB, NW>), smem);
  if (err != cudaSuccess) return err;
  if (knob(kKnobVerbose))
    fprintf(stderr, "dbf plan: B=%d warps=%d -> clusters=%d split=%d warps=%dx%d / %dx%d smem=%d\n", NB, NW, Q, S,
            p1.Wn, p1.Wg, p2.Wn, p2.Wg, smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(Q * S));
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(S);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, dbf_direct_kernel<NB, NW>, p1, p2, bar);
}

size_t dbf_tc_workspace_bytes(int64_t r, int64_t n, int64_t B);
cudaError_t launch_dbf_tc(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                          const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B, float* y,
                          void* workspace, cudaStream_t stream, int num_sms);

cudaError_t launch_gemv_direct_diag(const uint32_t* signs, int64_t N, int64_t K, const void* x, bool x_f32,
                                    const uint16_t* cdiag, const uint16_t* rdiag, int B, float* y, bool early,
                                    cudaStream_t stream, int num_sms, int smem_cap, int warps, int force_s);
cudaError_t launch_gemv_flat_diag(const uint32_t* signs, int64_t N, int64_t K, const void* x, bool x_f32,
                                  const uint16_t* cdiag, const uint16_t* rdiag, int B, float* y, bool early,
                                  cudaStream_t stream, int num_sms, int smem_cap, int split, int warps);

// Batches of at least this many rows run on the tensor-core path.
constexpr int64_t kDbfTensorMinBatch = 64;
// Groups of up to this many rows run as two GEMV launches, larger ones (up to
// 8) as the fused chain kernel.
constexpr int kDbfTwoStepMaxRows = 4;

size_t dbf_workspace_bytes(int64_t m, int64_t r, int64_t n, int64_t B) {
  (void)m;
  const int64_t rows = B < 8 ? B : 8;
  size_t bytes = static_cast<size_t>(256 + 4 * rows * r);
  if (B >= kDbfTensorMinBatch) {
    const size_t tc = dbf_tc_workspace_bytes(r, n, B);
    if (tc > bytes) bytes = tc;
  }
  return bytes;
}

cudaError_t launch_dbf(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                       const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B,
                       float* y, void* workspace, cudaStream_t stream, int num_sms, int smem_cap,
                       bool allow_tensor_path = true) {
  if (allow_tensor_path && B >= kDbfTensorMinBatch)
    return launch_dbf_tc(a, B1, mid, B2, b, m, r, n, x, B, y, workspace, stream, num_sms);
  unsigned int* bar = reinterpret_cast<unsigned int*>(workspace);
  float* h = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + 256);
  // Batches of up to 8 rows through the fused chain kernel: 8 warps per CTA
  // for groups of up to 3 rows, 16 above (as measured).  The dbf_warps knob
  // forces 8 or 16.
  const int wknob = knob(kKnobDbfWarps);
  const int pknob = knob(kKnobDbfPath);  // 0: default, 1: fused, 2: two launches
  const int im = static_cast<int>(m), ir = static_cast<int>(r), in = static_cast<int>(n);
  for (int64_t b0 = 0; b0 < B; b0 += 8) {
    const int nb = static_cast<int>((B - b0) < 8 ? (B - b0) : 8);
    const uint16_t* xg = x + b0 * n;
    float* yg = y + b0 * m;
    const bool w16 = wknob ? wknob == 16 : nb >= 4;
    cudaError_t err;
    // Default form by the measured A/B on the 4096^3 chain (graphs of
    // back-to-back calls, us per call, fused / two launches): 1 row 11.1 /
    // 8.1, 2 rows 14.5 / 10.1, 3 rows 16.2 / 13.5, 4 rows 14.9 / 12.6 (U . h
    // with r split over 2 CTAs of a cluster; 14.5 on the register-fed core),
    // 8 rows 17.8 / 19.1 (best split).  So two launches up to 4 rows, the
    // fused kernel from 5.
    const bool two = pknob ? pknob == kDbfTwoStep : nb <= kDbfTwoStepMaxRows;
    if (!two) {
      switch (nb) {
#define W1_DBF_CASE(NBV)                                                                                   \
  case NBV:                                                                                                \
    err = w16 ? launch_dbf_small_nb<NBV, 16>(a, B1, mid, B2, b, im, ir, in, xg, yg, h, bar, stream, num_sms, \
                                             smem_cap)                                                    \
              : launch_dbf_small_nb<NBV, 8>(a, B1, mid, B2, b, im, ir, in, xg, yg, h, bar, stream, num_sms,  \
                                            smem_cap);                                                    \
    break;
        W1_DBF_CASE(1)
        W1_DBF_CASE(2)
        W1_DBF_CASE(3)
        W1_DBF_CASE(4)
        W1_DBF_CASE(5)
        W1_DBF_CASE(6)
        W1_DBF_CASE(7)
        default:
          err = w16 ? launch_dbf_small_nb<8, 16>(a, B1, mid, B2, b, im, ir, in, xg, yg, h, bar, stream, num_sms,
                                                 smem_cap)
                    : launch_dbf_small_nb<8, 8>(a, B1, mid, B2, b, im, ir, in, xg, yg, h, bar, stream, num_sms,
                                                smem_cap);
          break;
#undef W1_DBF_CASE
      }
      // a chain whose two products admit no co-resident plan (very long K)
      // runs as two launches instead
      if (err != cudaErrorNotSupported) {
        if (err != cudaSuccess) return err;
        continue;
      }
    }
    // Two launches of a GEMV core ("LLM binarization episode 01: DBF",
    // section 4: x_scaled = D_in x, h = V x_scaled, h_scaled = D_mid h, then
    // y = D_out (U h_scaled)): h_scaled in fp32 through the workspace; U may
    // be read before the first launch completes (that launch writes only h).
    // The second product contracts over r: its K split is the split-rank
    // form of section 5 item 5 (r partitioned over the CTAs of a cluster,
    // partial outputs added in a fixed order through distributed shared
    // memory); dbf_rank_split forces it.  Each product on the register-fed
    // GEMV core (1-4 rows) where its plan fits and no rank split is forced,
    // else on the direct core.
    const int warps = wknob ? wknob : (nb >= 4 ? 16 : 8);
    const int rknob = knob(kKnobDbfRankSplit);
    // 4 rows: U . h on the direct core with r split over 2 CTAs by default
    const int rsplit = rknob ? rknob : (nb == 4 ? 2 : 0);
    const int cknob = knob(kKnobDbfCore);  // 0: flat where it fits, 1: flat, 2: direct
    const bool try_flat = cknob != 2 && nb <= 4;
    const int fw = wknob ? wknob : (nb <= 2 ? 8 : 16);  // the register-fed core's warps
    err = cudaErrorNotSupported;
    if (try_flat) err = launch_gemv_flat_diag(B2, r, n, xg, false, b, mid, nb, h, false, stream, num_sms, smem_cap, 0, fw);
    if (err == cudaErrorNotSupported)
      err = launch_gemv_direct_diag(B2, r, n, xg, false, b, mid, nb, h, false, stream, num_sms, smem_cap, warps, 0);
    if (err == cudaSuccess) {
      err = cudaErrorNotSupported;
      if (try_flat && rsplit == 0)
        err = launch_gemv_flat_diag(B1, m, r, h, true, nullptr, a, nb, yg, true, stream, num_sms, smem_cap, 0, fw);
      if (err == cudaErrorNotSupported)
        err = launch_gemv_direct_diag(B1, m, r, h, true, nullptr, a, nb, yg, true, stream, num_sms, smem_cap, warps,
                                      rsplit);
      if (err == cudaErrorNotSupported && rknob == 0 && rsplit != 0)  // the default split does not fit: planner
        err = launch_gemv_direct_diag(B1, m, r, h, true, nullptr, a, nb, yg, true, stream, num_sms, smem_cap, warps, 0);
    }
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}
// ------------------------------------------------------------------ static scratch
// Scratch for callers that cannot allocate device memory: a fixed array in the
// library's own device image (every GPU that loads the library holds it until
// the process exits).  Holds the barrier count (first 256 bytes) and the fp32
// intermediate for up to 8 batch rows of r <= kDbfStaticMaxR.
constexpr int64_t kDbfStaticMaxR = 16384;
constexpr size_t kDbfStaticScratchBytes = 256 + 4 * 8 * kDbfStaticMaxR;
static __device__ __align__(256) unsigned char g_dbf_static_scratch[kDbfStaticScratchBytes];

// Device address of the scratch array for the current device.  In host code
// the symbol is only a stand-in, so the address is looked up once per device
// (with that device current) and cached.
static void* dbf_static_scratch_ptr(int* status) {
  static void* ptrs[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = W1_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dbf_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      *status = W1_ERR_CUDA;
      return nullptr;
    }
    ptrs[dev] = p;
  }
  *status = W1_OK;
  return ptrs[dev];
}

}  // namespace w1

// ------------------------------------------------------------------ C entry point
using w1::aligned16;
extern "C" {

// dbf_apply without a workspace argument (see include/w1.h): same kernel, the
// scratch being the static array above.  Allocates nothing.
int dbf_apply_noalloc(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                      const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B, float* y,
                      w1_stream_t stream) {
  if (!a || !B1 || !mid || !B2 || !b || !x || !y) return W1_ERR_NULL;
  if (m <= 0 || r <= 0 || n <= 0 || B <= 0 || (r % 128) != 0 || (n % 128) != 0) return W1_ERR_SHAPE;
  if (m > (int64_t)1 << 30 || n > (int64_t)1 << 30) return W1_ERR_SHAPE;
  if (r > w1::kDbfStaticMaxR) return W1_ERR_TOO_LARGE;
  if (!aligned16(a) || !aligned16(B1) || !aligned16(mid) || !aligned16(B2) || !aligned16(b) || !aligned16(x) ||
      !aligned16(y))
    return W1_ERR_ALIGN;
  w1::DeviceInfo d;
  int st = w1::device_info(&d);
  if (st != W1_OK) return st;
  void* scratch = w1::dbf_static_scratch_ptr(&st);
  if (st != W1_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the barrier count must start at zero (a previous call may have timed out)
  if (cudaMemsetAsync(scratch, 0, 8, s) != cudaSuccess) return W1_ERR_CUDA;
  const int cap = d.smem_optin < 200 * 1024 ? d.smem_optin : 200 * 1024;
  return w1::launch_result(w1::launch_dbf(a, B1, mid, B2, b, m, r, n, x, B, y, scratch, s, d.sms, cap, false));
}

}  // extern "C"

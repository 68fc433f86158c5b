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
//  * Memory: each 16-row tile of sign words arrives by swizzled 2-D TMA boxes
//    (16 rows x 4 or 8 groups, one instruction each; all stages issued up
//    front when they fit).  Up to 16 consumer warps share a tile, each taking
//    a K sub-range, so every warp's dependency chain is short.  When B x K is
//    too large for one CTA's shared memory a cluster of S CTAs splits K; the
//    sub-range and cluster partial sums are reduced in a fixed order through
//    (distributed) shared memory: deterministic, no atomics, no workspace.
//  * Programmatic dependent launch: the kernel waits for the previous kernel
//    before touching memory and lets the next one launch right away.
#include <cstdint>
#include <cuda_fp16.h>
#include <cstdio>
#include <cstring>
#include <cstdlib>
#include <mutex>

#include "gemv_core.cuh"

namespace w1 {

struct GemvParams {
  const uint16_t* scales;
  const uint16_t* x;
  float* y;
  int64_t N;        // total rows of the matrix (row stride of y)
  int64_t K;
  int64_t row_base; // first row handled by this launch
  int rows;         // rows handled by this launch
  int NG;           // K / 128
  int S;            // cluster size (K split)
  int bw;           // groups per TMA box (4 or 8)
  int ns;           // pipeline stages
  int max_tiles;    // max 16-row tiles per cluster
  int max_ng;       // max groups per CTA
};

struct GemvSmem {
  int stages, stage_bytes, xq, zero, xsum, xf, sc, part, bars, total;
};

template <int NB>
__host__ __device__ inline GemvSmem gemv_smem_layout(int ns, int max_tiles, int max_ng, int bw) {
  using L = GemvLayout<NB>;
  GemvSmem M;
  int off = 0;
  M.stages = off;
  M.stage_bytes = ((max_ng + bw - 1) / bw) * 16 * 16 * bw;
  off += ns * M.stage_bytes;
  off = round_up(off, 128);
  M.xq = off;
  off += max_ng * 4 * L::BLOCK;
  off = round_up(off, 16);
  M.zero = off;
  off += 16;
  M.xsum = off;
  off += max_ng * NB * 4;
  M.xf = off;
  off += max_ng * NB * 4;
  off = round_up(off, 16);
  M.sc = off;
  off += max_tiles * 16 * max_ng * 2;
  off = round_up(off, 16);
  M.part = off;
  off += gemv_wpt(max_tiles) * NB * max_tiles * 16 * 4;
  off = round_up(off, 8);
  M.bars = off;
  off += 2 * ns * 8;
  M.total = round_up(off, 128) + 1024;  // + alignment slack for the 1024-aligned stages
  return M;
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
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap, const GemvParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemvSmem M = gemv_smem_layout<NB>(p.ns, p.max_tiles, p.max_ng, p.bw);
  GemvSmemView v;
  v.stages = smem + M.stages;
  v.ns = p.ns;
  v.stage_bytes = M.stage_bytes;
  v.full = reinterpret_cast<uint64_t*>(smem + M.bars);
  v.empty = v.full + p.ns;
  GemvXView xv;
  xv.xq = smem + M.xq;
  xv.xsum = reinterpret_cast<int*>(smem + M.xsum);
  xv.xf = reinterpret_cast<float*>(smem + M.xf);
  xv.sc = reinterpret_cast<uint16_t*>(smem + M.sc);
  xv.part = reinterpret_cast<float*>(smem + M.part);
  xv.part_stride = p.max_tiles * 16;
  unsigned char* zero16 = smem + M.zero;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int crank = static_cast<int>(cluster_ctarank());
  const Split sp = make_split(p.rows, p.row_base, p.NG, p.S, crank, static_cast<int>(cluster_id_x()),
                              static_cast<int>(nclusters_x()), p.bw, p.bw, p.max_tiles);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ns; ++s) {
      mbar_init(&v.full[s], 1);
      mbar_init(&v.empty[s], static_cast<uint32_t>(sp.wpt));
    }
    fence_mbarrier_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap) : "memory");
  }
  if (threadIdx.x < 4) reinterpret_cast<uint32_t*>(zero16)[threadIdx.x] = 0u;
  __syncthreads();
  pdl_wait();
  // the next kernel in the stream may launch now; it touches no memory before
  // its own dependency wait, i.e. before this grid has completed
  pdl_launch_dependents();

  int first = 0;
  if (warp == kProducerWarp && lane == 0) first = issue_first_tiles(v, sp, &tmap, p.bw);
  __syncwarp();

  // activations -> digit planes; scales of this CTA's rows and groups -> smem
  const uint16_t* xb = p.x;
  const int64_t K = p.K;
  quantise_input<NB>(xv, sp,
                     [&](int b, int k, float (&vv)[16]) { load16_bf16(xb + static_cast<int64_t>(b) * K + k, vv); },
                     kGemvThreads);
  stage_scales(xv, sp, p.scales, p.NG, kGemvThreads);
  __syncthreads();

  if (warp == kProducerWarp) {
    if (lane == 0) produce_rest(v, sp, &tmap, p.bw, first);
    __syncwarp();  // converge before the (cluster) barrier, which is .aligned
  } else {
    consume_tiles<NB, true>(v, xv, sp, p.bw, zero16, warp, lane);
  }
  if (p.S > 1) cluster_sync(); else __syncthreads();
  float* y = p.y;
  const int64_t N = p.N;
  cluster_reduce<NB>(xv, sp, p.S, crank, [&](int b, int64_t row, float val) { y[b * N + row] = val; },
                     kGemvThreads);
  if (p.S > 1) cluster_sync();
}

// ------------------------------------------------------------------ host side

bool make_tmap_u32_rows(CUtensorMap* map, const void* base, int64_t rows, int64_t words, int box_words);

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
  if (ensure_dyn_smem(reinterpret_cast<const void*>(gemv_kernel<NB>), smem_bytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, gemv_kernel<NB>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

struct GemvPlan {
  int Q, S, bw, ns, max_tiles, max_ng, smem;
};

// K split S: the smallest that keeps this CTA's activation digits within
// budget (K split only pays off when x is large); clusters Q: one resident
// wave; stages: every tile when it fits.
template <int NB>
static bool gemv_make_plan(int rows, int NG, int num_sms, int smem_cap, int force_s, GemvPlan* out) {
  using L = GemvLayout<NB>;
  const int T16 = (rows + 15) / 16;
  for (int S = 1; S <= 8; S *= 2) {
    if (force_s && S != force_s) continue;
    if (S > NG && S > 1) break;
    const int bw = (NG % (8 * S) == 0 || S == 1) ? 8 : 4;
    const int units = (NG + bw - 1) / bw;
    const int max_ng = ((units + S - 1) / S) * bw;
    if (!force_s && max_ng * 4 * L::BLOCK > 80 * 1024 && S < 8) continue;
    int Q = num_sms / S;
    if (Q > T16) Q = T16;
    if (Q < 1) Q = 1;
    for (int iter = 0; iter < 3; ++iter) {
      const int max_tiles = (T16 + Q - 1) / Q;
      const GemvSmem M0 = gemv_smem_layout<NB>(0, max_tiles, max_ng, bw);
      const int stage_bytes = ((max_ng + bw - 1) / bw) * 16 * 16 * bw;
      int ns = max_tiles;
      const int budget = smem_cap - M0.total;
      if (ns * (stage_bytes + 16) > budget) ns = budget / (stage_bytes + 16);
      if (ns < 1) return false;
      const int smem = gemv_smem_layout<NB>(ns, max_tiles, max_ng, bw).total;
      const int occ = gemv_max_clusters<NB>(S, smem);
      if (occ > 0 && occ < Q) {
        Q = occ;
        continue;
      }
      *out = GemvPlan{Q, S, bw, ns, max_tiles, max_ng, smem};
      return true;
    }
  }
  return false;
}

struct GemvPlanEntry {
  int rows, NG, NB, sms, cap, dev, force;
  GemvPlan plan;
};
static GemvPlanEntry g_plan_cache[64];
static int g_plan_count = 0;
static std::mutex g_plan_mu;

template <int NB>
static cudaError_t launch_gemv_nb(const uint32_t* signs, const GemvParams& base, cudaStream_t stream, int num_sms,
                                  int smem_cap) {
  int force = 0;
  force = knob(kKnobGemvSplit);  // tuning knob: force the K split
  if (force != 1 && force != 2 && force != 4 && force != 8) force = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  GemvPlan plan;
  bool found = false;
  {
    std::lock_guard<std::mutex> lock(g_plan_mu);
    for (int i = 0; i < g_plan_count; ++i) {
      const GemvPlanEntry& e = g_plan_cache[i];
      if (e.rows == base.rows && e.NG == base.NG && e.NB == NB && e.sms == num_sms && e.cap == smem_cap &&
          e.dev == dev && e.force == force) {
        plan = e.plan;
        found = true;
        break;
      }
    }
  }
  if (!found) {
    if (!gemv_make_plan<NB>(base.rows, base.NG, num_sms, smem_cap, force, &plan)) return cudaErrorInvalidConfiguration;
    std::lock_guard<std::mutex> lock(g_plan_mu);
    const int i = g_plan_count < 64 ? g_plan_count++ : (base.rows + base.NG + NB) & 63;
    g_plan_cache[i] = GemvPlanEntry{base.rows, base.NG, NB, num_sms, smem_cap, dev, force, plan};
  }
  if (knob(kKnobVerbose))
    fprintf(stderr, "w1_gemv plan: rows=%d NG=%d B=%d -> clusters=%d split=%d box=%d stages=%d tiles=%d smem=%d\n",
            base.rows, base.NG, NB, plan.Q, plan.S, plan.bw, plan.ns, plan.max_tiles, plan.smem);
  GemvParams p = base;
  p.S = plan.S;
  p.bw = plan.bw;
  p.ns = plan.ns;
  p.max_tiles = plan.max_tiles;
  p.max_ng = plan.max_ng;
  CUtensorMap tmap;
  if (!make_tmap_u32_rows(&tmap, signs, base.N, base.K / 32, 4 * plan.bw)) return cudaErrorInvalidValue;
  cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(gemv_kernel<NB>), plan.smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.Q * plan.S));
  cfg.blockDim = dim3(kGemvThreads);
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
  return cudaLaunchKernelEx(&cfg, gemv_kernel<NB>, tmap, p);
}

cudaError_t launch_gemv_tc(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K, const uint16_t* x,
                           int B, float* y, bool static_weights, cudaStream_t stream, int num_sms, int force_s);
cudaError_t launch_gemv_flat(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K, const uint16_t* x,
                             int B, float* y, bool static_weights, cudaStream_t stream, int num_sms, int smem_cap,
                             int split, int warps);
cudaError_t launch_gemv_direct(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                               const void* x, bool x_f32, int B, float* y, bool static_weights,
                               cudaStream_t stream, int num_sms, int smem_cap, int force_s, int warps);

// The mma.sync ring kernel over row chunks (the fallback for shapes outside
// the other two kernels' plans).
static cudaError_t launch_gemv_ring(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                                   const uint16_t* x, int B, float* y, cudaStream_t stream, int num_sms,
                                   int smem_cap) {
  const int NG = static_cast<int>(K / 128);
  // rows per launch bounded so that per-CTA scale / partial buffers fit
  const int64_t max_rows = 32768;
  for (int64_t r0 = 0; r0 < N; r0 += max_rows) {
    const int rows = static_cast<int>((N - r0) < max_rows ? (N - r0) : max_rows);
    GemvParams p = {};
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
      case 1: err = launch_gemv_nb<1>(signs, p, stream, num_sms, smem_cap); break;
      case 2: err = launch_gemv_nb<2>(signs, p, stream, num_sms, smem_cap); break;
      case 3: err = launch_gemv_nb<3>(signs, p, stream, num_sms, smem_cap); break;
      case 4: err = launch_gemv_nb<4>(signs, p, stream, num_sms, smem_cap); break;
      case 5: err = launch_gemv_nb<5>(signs, p, stream, num_sms, smem_cap); break;
      case 6: err = launch_gemv_nb<6>(signs, p, stream, num_sms, smem_cap); break;
      case 7: err = launch_gemv_nb<7>(signs, p, stream, num_sms, smem_cap); break;
      default: err = launch_gemv_nb<8>(signs, p, stream, num_sms, smem_cap); break;
    }
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

// ------------------------------------------------------------------ dispatch

// Kernel and K split per (device, N, K, B, static weights, activation type),
// chosen by timing.  fp32 activations (the rotated-activation product) are
// read only by the direct kernel, so only its candidates are timed for them.
// The first call for a shape (outside stream capture) runs each candidate --
// the direct kernel with K split 1, 2, 4, 8 at 8 and at 16 warps per CTA, the
// tcgen05 kernel, the ring kernel -- three times plainly and twelve times back
// to back as one captured CUDA graph (timed between CUDA events), on a private
// stream ordered after the caller's work, with the caller's buffers; keeps the
// fastest, and blocks the host until that finishes (a few milliseconds).
// Calls made while the stream is being captured, or with W1_GEMV_AUTOTUNE=0,
// use the static rule instead: direct for B <= 4, tcgen05 above, each only
// where its plan fits, else the ring kernel.  W1_GEMV_PATH=direct|direct16|tc|mma forces one kernel (testing
// knob; a forced kernel whose plan does not fit fails with W1_ERR_UNSUPPORTED).
namespace {
struct GemvChoice {
  char kind;  // 'f' fp8 (gemv_flat.cu), 'd' direct, 't' tcgen05, 'm' ring
  int s;      // forced K split, 0 = the kernel's planner (flat: 1)
  int w;      // flat and direct kernels: warps per CTA (8 or 16)
};
struct GemvChoiceEntry {
  int dev;
  int64_t N, K;
  int B;
  bool st;
  bool xf;  // fp32 activations (direct kernel only)
  GemvChoice c;
};
GemvChoiceEntry g_choice[256];
int g_nchoice = 0;
std::mutex g_choice_mu;
}  // namespace

// x is bf16 [B][K], or fp32 [B][K] with xf (which only the direct kernel reads).
static cudaError_t run_gemv_choice(const GemvChoice& c, const uint32_t* signs, const uint16_t* scales, int64_t N,
                                   int64_t K, const void* x, bool xf, int B, float* y, cudaStream_t stream,
                                   int num_sms, int smem_cap, bool static_weights) {
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  switch (c.kind) {
    case 'f':
      if (xf) return cudaErrorNotSupported;
      return launch_gemv_flat(signs, scales, N, K, xb, B, y, static_weights, stream, num_sms, smem_cap, c.s, c.w);
    case 'd':
      return launch_gemv_direct(signs, scales, N, K, x, xf, B, y, static_weights, stream, num_sms, smem_cap, c.s,
                                c.w);
    case 't':
      if (xf) return cudaErrorNotSupported;
      return launch_gemv_tc(signs, scales, N, K, xb, B, y, static_weights, stream, num_sms, c.s);
    default:
      if (xf) return cudaErrorNotSupported;
      return launch_gemv_ring(signs, scales, N, K, xb, B, y, stream, num_sms, smem_cap);
  }
}

// The static rule with fallbacks: bf16 activations the fp8 kernel (8 warps,
// no split), then direct or tcgen05 by batch, then ring; fp32 activations
// only the direct kernel: 8 warps, then 16.
static cudaError_t run_gemv_rule(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                                 const void* x, bool xf, int B, float* y, cudaStream_t stream, int num_sms,
                                 int smem_cap, bool static_weights) {
  if (!xf) {
    const cudaError_t ef = run_gemv_choice(GemvChoice{'f', 0, 8}, signs, scales, N, K, x, xf, B, y, stream, num_sms,
                                           smem_cap, static_weights);
    if (ef != cudaErrorNotSupported) return ef;
  }
  const GemvChoice first = (B <= 4 || xf) ? GemvChoice{'d', 0, 8} : GemvChoice{'t', 0, 0};
  const GemvChoice second = xf ? GemvChoice{'d', 0, 16} : (B <= 4 ? GemvChoice{'t', 0, 0} : GemvChoice{'d', 0, 8});
  cudaError_t e =
      run_gemv_choice(first, signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);
  if (e != cudaErrorNotSupported) return e;
  e = run_gemv_choice(second, signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);
  if (e != cudaErrorNotSupported || xf) return e;
  return launch_gemv_ring(signs, scales, N, K, static_cast<const uint16_t*>(x), B, y, stream, num_sms, smem_cap);
}

// One autotune measurement: `reps` back-to-back launches of candidate c
// captured as one CUDA graph on the private stream ts (the way a decode loop
// replays them), after three plain launches that also check that c fits.
// Returns 1 with *ms set, 0 when c does not fit or cannot be captured, -1 on
// a device error (in *err).
static int time_gemv_choice(const GemvChoice& c, const uint32_t* signs, const uint16_t* scales, int64_t N,
                            int64_t K, const void* x, bool xf, int B, float* y, cudaStream_t ts, int num_sms,
                            int smem_cap, bool static_weights, int reps, cudaEvent_t e0, cudaEvent_t e1, float* ms,
                            cudaError_t* err) {
  for (int i = 0; i < 3; ++i) {
    if (run_gemv_choice(c, signs, scales, N, K, x, xf, B, y, ts, num_sms, smem_cap, static_weights) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
  }
  cudaGraph_t g = nullptr;
  if (cudaStreamBeginCapture(ts, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaError_t le = cudaSuccess;
  for (int i = 0; i < reps && le == cudaSuccess; ++i)
    le = run_gemv_choice(c, signs, scales, N, K, x, xf, B, y, ts, num_sms, smem_cap, static_weights);
  const cudaError_t ce = cudaStreamEndCapture(ts, &g);
  cudaGraphExec_t ge = nullptr;
  const bool built = le == cudaSuccess && ce == cudaSuccess && g && cudaGraphInstantiate(&ge, g, 0) == cudaSuccess;
  if (g) cudaGraphDestroy(g);
  if (!built) {
    cudaGetLastError();
    return 0;
  }
  cudaGraphLaunch(ge, ts);  // warm
  cudaEventRecord(e0, ts);
  cudaGraphLaunch(ge, ts);
  cudaEventRecord(e1, ts);
  *err = cudaEventSynchronize(e1);
  cudaGraphExecDestroy(ge);
  if (*err != cudaSuccess) return -1;
  cudaEventElapsedTime(ms, e0, e1);
  return 1;
}

cudaError_t launch_gemv(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                        const void* x, bool xf, int B, float* y, cudaStream_t stream, int num_sms,
                        int smem_cap, bool static_weights) {
  if (const int path = knob(kKnobGemvPath)) {
    // fp32 activations run the direct kernel whatever the knob names.
    const bool direct = path == kGemvDirect8 || path == kGemvDirect16 || xf;
    const bool flat = path == kGemvFlat || path == kGemvFlat16;
    const int split = knob(kKnobGemvSplit);
    const GemvChoice c{direct ? 'd' : (flat ? 'f' : (path == kGemvTc ? 't' : 'm')), flat ? split : 0,
                       (path == kGemvDirect16 || path == kGemvFlat16) ? 16 : 8};
    return run_gemv_choice(c, signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);
  }
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(g_choice_mu);
    for (int i = 0; i < g_nchoice; ++i) {
      const GemvChoiceEntry& e = g_choice[i];
      if (e.dev == dev && e.N == N && e.K == K && e.B == B && e.st == static_weights && e.xf == xf)
        return run_gemv_choice(e.c, signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);
    }
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
    cudaGetLastError();
    cap = cudaStreamCaptureStatusActive;
  }
  if (cap != cudaStreamCaptureStatusNone || knob(kKnobGemvAutotune) == 0)
    return run_gemv_rule(signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);

  const GemvChoice cands[] = {{'f', 1, 8},  {'f', 2, 8},  {'f', 4, 8},  {'f', 1, 16}, {'f', 2, 16}, {'f', 4, 16},
                              {'d', 1, 8},  {'d', 2, 8},  {'d', 4, 8},  {'d', 8, 8},  {'d', 1, 16}, {'d', 2, 16},
                              {'d', 4, 16}, {'d', 8, 16}, {'t', 0, 0},  {'m', 0, 0}};
  constexpr int kTimed = 12;
  // A private stream, ordered after the caller's work so far, takes the
  // captures (the caller's stream is not captured or reordered).
  cudaStream_t ts = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr, ready = nullptr;
  cudaError_t setup = cudaStreamCreateWithFlags(&ts, cudaStreamNonBlocking);
  if (setup == cudaSuccess) setup = cudaEventCreate(&e0);
  if (setup == cudaSuccess) setup = cudaEventCreate(&e1);
  if (setup == cudaSuccess) setup = cudaEventCreateWithFlags(&ready, cudaEventDisableTiming);
  if (setup == cudaSuccess) setup = cudaEventRecord(ready, stream);
  if (setup == cudaSuccess) setup = cudaStreamWaitEvent(ts, ready, 0);
  auto release = [&]() {
    if (ts) {
      cudaStreamSynchronize(ts);
      cudaStreamDestroy(ts);
    }
    if (e0) cudaEventDestroy(e0);
    if (e1) cudaEventDestroy(e1);
    if (ready) cudaEventDestroy(ready);
  };
  if (setup != cudaSuccess) {
    release();
    cudaGetLastError();
    return run_gemv_rule(signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);
  }
  // The candidates run on one weight matrix that stays in L2, which flatters
  // the kernels least sensitive to memory latency; the static rule's kernel
  // is kept unless another is more than 5% faster.
  const char rule_kind = xf ? 'd' : 'f';
  GemvChoice best{0, 0, 0}, best_rule{0, 0, 0};
  float best_ms = 0.f, best_rule_ms = 0.f;
  cudaError_t fatal = cudaSuccess;
  for (const GemvChoice& c : cands) {
    float ms = 0.f;
    if (xf && c.kind != 'd') continue;
    const int r = time_gemv_choice(c, signs, scales, N, K, x, xf, B, y, ts, num_sms, smem_cap, static_weights,
                                   kTimed, e0, e1, &ms, &fatal);
    if (r < 0) break;  // a device error: report it, choose nothing
    if (r == 0) continue;
    if (knob(kKnobVerbose))
      fprintf(stderr, "w1_gemv candidate: N=%lld K=%lld B=%d %c split=%d warps=%d %.2f us\n",
              static_cast<long long>(N), static_cast<long long>(K), B, c.kind, c.s, c.w, ms * 1e3f / kTimed);
    if (best.kind == 0 || ms < best_ms) {
      best = c;
      best_ms = ms;
    }
    if (c.kind == rule_kind && (best_rule.kind == 0 || ms < best_rule_ms)) {
      best_rule = c;
      best_rule_ms = ms;
    }
  }
  if (best_rule.kind != 0 && best.kind != rule_kind && best_ms > 0.95f * best_rule_ms) {
    best = best_rule;
    best_ms = best_rule_ms;
  }
  release();
  if (fatal != cudaSuccess) return fatal;
  if (best.kind == 0)
    return run_gemv_rule(signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);
  if (knob(kKnobVerbose))
    fprintf(stderr, "w1_gemv tuned: N=%lld K=%lld B=%d static=%d -> %c split=%d warps=%d (%.2f us)\n",
            static_cast<long long>(N), static_cast<long long>(K), B, static_weights ? 1 : 0, best.kind, best.s,
            best.w, best_ms * 1e3f / kTimed);
  {
    std::lock_guard<std::mutex> lock(g_choice_mu);
    const int i = g_nchoice < 256 ? g_nchoice++ : static_cast<int>((N + K + B) & 255);
    g_choice[i] = GemvChoiceEntry{dev, N, K, B, static_weights, xf, best};
  }
  return run_gemv_choice(best, signs, scales, N, K, x, xf, B, y, stream, num_sms, smem_cap, static_weights);
}

// Name of the cached choice for a shape ("direct/2", "direct16/1", "tc/0",
// "ring/0"), or ""
// when none has been made on the current device.
static int gemv_choice_name(int64_t N, int64_t K, int B, bool st, char* out, size_t out_len) {
  int dev = 0;
  cudaGetDevice(&dev);
  GemvChoice c{0, 0, 0};
  {
    std::lock_guard<std::mutex> lock(g_choice_mu);
    for (int i = 0; i < g_nchoice; ++i) {
      const GemvChoiceEntry& e = g_choice[i];
      if (e.dev == dev && e.N == N && e.K == K && e.B == B && e.st == st && !e.xf) c = e.c;
    }
  }
  const char* kind = c.kind == 'f'   ? (c.w == 16 ? "flat16" : "flat")
                     : c.kind == 'd' ? (c.w == 16 ? "direct16" : "direct")
                                     : (c.kind == 't' ? "tc" : (c.kind == 'm' ? "ring" : ""));
  if (c.kind == 0) return snprintf(out, out_len, "%s", "");
  return snprintf(out, out_len, "%s/%d", kind, c.s);
}

// Parses "flat/<s>", "flat16/<s>", "direct/<s>", "direct16/<s>", "tc/<s>",
// "ring/<s>" (w1_gemv_choice's notation); false for anything else.
static bool parse_gemv_choice(const char* name, GemvChoice* c) {
  const char* slash = strchr(name, '/');
  if (!slash) return false;
  const size_t len = static_cast<size_t>(slash - name);
  char* end = nullptr;
  const long sp = strtol(slash + 1, &end, 10);
  if (end == slash + 1 || *end != '\0' || sp < 0 || sp > 8) return false;
  auto is = [&](const char* k) { return strlen(k) == len && strncmp(name, k, len) == 0; };
  if (is("flat") || is("flat16")) {
    if (sp != 1 && sp != 2 && sp != 4 && sp != 8) return false;
    *c = GemvChoice{'f', static_cast<int>(sp), is("flat16") ? 16 : 8};
  } else if (is("direct") || is("direct16")) {
    if (sp != 1 && sp != 2 && sp != 4 && sp != 8) return false;
    *c = GemvChoice{'d', static_cast<int>(sp), is("direct16") ? 16 : 8};
  } else if (is("tc")) {
    *c = GemvChoice{'t', static_cast<int>(sp), 0};
  } else if (is("ring")) {
    *c = GemvChoice{'m', 0, 0};
  } else {
    return false;
  }
  return true;
}

static int gemv_set_choice(int64_t N, int64_t K, int B, bool st, const GemvChoice& c) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return W1_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_choice_mu);
  for (int i = 0; i < g_nchoice; ++i) {
    GemvChoiceEntry& e = g_choice[i];
    if (e.dev == dev && e.N == N && e.K == K && e.B == B && e.st == st && !e.xf) {
      e.c = c;
      return W1_OK;
    }
  }
  const int i = g_nchoice < 256 ? g_nchoice++ : static_cast<int>((N + K + B) & 255);
  g_choice[i] = GemvChoiceEntry{dev, N, K, B, st, false, c};
  return W1_OK;
}

}  // namespace w1

extern "C" int w1_gemv_set_choice(int64_t N, int64_t K, int64_t B, uint32_t flags, const char* name) {
  if (!name) return W1_ERR_NULL;
  if (N <= 0 || K <= 0 || (K % 128) != 0 || B < 1 || B > 8) return W1_ERR_SHAPE;
  if ((flags & ~static_cast<uint32_t>(W1_GEMV_STATIC_WEIGHTS)) != 0) return W1_ERR_SHAPE;
  w1::GemvChoice c{0, 0, 0};
  if (!w1::parse_gemv_choice(name, &c)) return W1_ERR_SHAPE;
  return w1::gemv_set_choice(N, K, static_cast<int>(B), (flags & W1_GEMV_STATIC_WEIGHTS) != 0, c);
}

extern "C" int w1_gemv_choice(int64_t N, int64_t K, int64_t B, uint32_t flags, char* out, size_t out_len) {
  if (!out || out_len == 0) return W1_ERR_NULL;
  if (N <= 0 || K <= 0 || (K % 128) != 0 || B < 1 || B > 8) return W1_ERR_SHAPE;
  w1::gemv_choice_name(N, K, static_cast<int>(B), (flags & W1_GEMV_STATIC_WEIGHTS) != 0, out, out_len);
  return W1_OK;
}

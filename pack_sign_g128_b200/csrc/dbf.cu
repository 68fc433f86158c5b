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
// Small batch (B <= 8): ONE kernel runs both binary products -- the joint
// V-D_mid-U kernel with a grid-wide synchronisation that the DBF post
// (section 7, "CUDA/HIP: a starting point") proposes for CUDA.  Each CTA
//  1. bulk-copies its slices of BOTH sign matrices into shared memory at
//     once, so U streams in while V . (b x) is computed;
//  2. phase 1: cluster-split int8-MMA product (as w1_gemv, no group scales)
//     on b (.) x, cluster reduction, h_scaled = mid (.) h -> workspace (fp32);
//  3. grid barrier (bounded spin; on timeout W1_ERR_TIMEOUT, no hang);
//  4. phase 2: the same product of U with h_scaled, y = a (.) (...).
// The intermediate stays fp32 (exact to 2^-24 relative), so the only
// quantisation is the 23-bit fixed point of each product's input.
#include <cstdint>
#include <cuda_fp16.h>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "gemv_core.cuh"

namespace w1 {

struct DbfParams {
  const uint16_t* a;    // [m] fp16
  const uint16_t* mid;  // [r] fp16
  const uint16_t* b;    // [n] fp16
  const uint16_t* x;    // [B][n] bf16
  float* y;             // [B][m]
  float* h;             // [B][r] workspace: mid (.) (B2 . (b (.) x))
  unsigned int* bar;    // workspace: grid barrier {count, generation}
  int m, r, n;
  int S, bw1, bw2;
  int ns1, ns2;
  int max_tiles1, max_tiles2, max_ng1, max_ng2;
};

struct DbfSmem {
  int st1, sb1, st2, sb2, xq, zero, xsum, xf, part, bars, total;
};

template <int NB>
__host__ __device__ inline DbfSmem dbf_smem_layout(const DbfParams& p) {
  using L = GemvLayout<NB>;
  const int mng = p.max_ng1 > p.max_ng2 ? p.max_ng1 : p.max_ng2;
  const int mt = p.max_tiles1 > p.max_tiles2 ? p.max_tiles1 : p.max_tiles2;
  const int wp = gemv_wpt(p.max_tiles1) > gemv_wpt(p.max_tiles2) ? gemv_wpt(p.max_tiles1) : gemv_wpt(p.max_tiles2);
  DbfSmem M;
  int off = 0;
  M.st1 = off;
  M.sb1 = ((p.max_ng1 + p.bw1 - 1) / p.bw1) * 16 * 16 * p.bw1;
  off += p.ns1 * M.sb1;
  off = round_up(off, 1024);
  M.st2 = off;
  M.sb2 = ((p.max_ng2 + p.bw2 - 1) / p.bw2) * 16 * 16 * p.bw2;
  off += p.ns2 * M.sb2;
  off = round_up(off, 128);
  M.xq = off;
  off += mng * 4 * L::BLOCK;
  off = round_up(off, 16);
  M.zero = off;
  off += 16;
  M.xsum = off;
  off += mng * NB * 4;
  M.xf = off;
  off += mng * NB * 4;
  off = round_up(off, 16);
  M.part = off;
  off += wp * NB * mt * 16 * 4;
  off = round_up(off, 8);
  M.bars = off;
  off += 2 * (p.ns1 + p.ns2) * 8;
  M.total = round_up(off, 128) + 1024;
  return M;
}

// Grid-wide barrier over all CTAs of the launch (all co-resident by
// construction of the grid).  bar[0] counts arrivals, bar[1] is the
// generation; the last arrival resets the count, so the state is reusable by
// the next call.  Returns false (and records W1_ERR_TIMEOUT) if the other
// CTAs do not arrive within the spin limit.
__device__ inline bool grid_barrier(unsigned int* bar, unsigned int nblocks) {
  __syncthreads();
  int ok = 1;
  if (threadIdx.x == 0) {
    __threadfence();
    unsigned int gen;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(gen) : "l"(bar + 1) : "memory");
    const unsigned int arrived = atomicAdd(bar, 1u);
    if (arrived == nblocks - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      ok = 0;
      for (uint32_t i = 0; i < kSpinLimit; ++i) {
        unsigned int g;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g) : "l"(bar + 1) : "memory");
        if (g != gen) {
          ok = 1;
          break;
        }
        __nanosleep(128);
      }
      if (!ok) set_status(W1_ERR_TIMEOUT);
    }
    __threadfence();
  }
  return __syncthreads_and(ok) != 0;
}

template <int NB>
__global__ void __launch_bounds__(kGemvThreads, 1)
    dbf_small_kernel(const __grid_constant__ CUtensorMap tm2, const __grid_constant__ CUtensorMap tm1,
                     const DbfParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const DbfSmem M = dbf_smem_layout<NB>(p);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + M.bars);
  GemvSmemView v1{smem + M.st1, p.ns1, M.sb1, bars, bars + p.ns1};
  GemvSmemView v2{smem + M.st2, p.ns2, M.sb2, bars + 2 * p.ns1, bars + 2 * p.ns1 + p.ns2};
  GemvXView xv;
  xv.xq = smem + M.xq;
  xv.xsum = reinterpret_cast<int*>(smem + M.xsum);
  xv.xf = reinterpret_cast<float*>(smem + M.xf);
  xv.sc = nullptr;
  xv.part = reinterpret_cast<float*>(smem + M.part);
  xv.part_stride = (p.max_tiles1 > p.max_tiles2 ? p.max_tiles1 : p.max_tiles2) * 16;
  unsigned char* zero16 = smem + M.zero;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int crank = static_cast<int>(cluster_ctarank());
  const int q = static_cast<int>(cluster_id_x()), Q = static_cast<int>(nclusters_x());
  // rows of V with K = n, then rows of U with K = r
  const Split sp1 = make_split(p.r, 0, p.n >> 7, p.S, crank, q, Q, p.bw1, p.bw1, p.max_tiles1);
  const Split sp2 = make_split(p.m, 0, p.r >> 7, p.S, crank, q, Q, p.bw2, p.bw2, p.max_tiles2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ns1; ++s) {
      mbar_init(&v1.full[s], 1);
      mbar_init(&v1.empty[s], static_cast<uint32_t>(sp1.wpt));
    }
    for (int s = 0; s < p.ns2; ++s) {
      mbar_init(&v2.full[s], 1);
      mbar_init(&v2.empty[s], static_cast<uint32_t>(sp2.wpt));
    }
    fence_mbarrier_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm2) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm1) : "memory");
  }
  if (threadIdx.x < 4) reinterpret_cast<uint32_t*>(zero16)[threadIdx.x] = 0u;
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();

  int first1 = 0, first2 = 0;
  if (warp == kProducerWarp && lane == 0) {
    first1 = issue_first_tiles(v1, sp1, &tm2, p.bw1);
    first2 = issue_first_tiles(v2, sp2, &tm1, p.bw2);
  }
  __syncwarp();

  // ---- phase 1: h_scaled = mid (.) (V . (b (.) x))
  {
    const uint16_t* xb = p.x;
    const uint16_t* bd = p.b;
    const int n = p.n;
    quantise_input<NB>(xv, sp1,
                       [&](int bb, int k, float (&vv)[16]) {
                         load16_bf16(xb + static_cast<int64_t>(bb) * n + k, vv);
                         const uint4 d0 = *reinterpret_cast<const uint4*>(bd + k);
                         const uint4 d1 = *reinterpret_cast<const uint4*>(bd + k + 8);
                         const uint32_t dw[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                         for (int i = 0; i < 8; ++i) {
                           const __half2 hh = *reinterpret_cast<const __half2*>(&dw[i]);
                           vv[2 * i] *= __low2float(hh);
                           vv[2 * i + 1] *= __high2float(hh);
                         }
                       },
                       kGemvThreads);
    __syncthreads();
    if (warp == kProducerWarp) {
      if (lane == 0) produce_rest(v1, sp1, &tm2, p.bw1, first1);
      __syncwarp();  // converge before the (cluster) barrier, which is .aligned
    } else {
      consume_tiles<NB, false>(v1, xv, sp1, p.bw1, zero16, warp, lane);
    }
    if (p.S > 1) cluster_sync(); else __syncthreads();
    float* h = p.h;
    const uint16_t* mid = p.mid;
    const int r = p.r;
    cluster_reduce<NB>(xv, sp1, p.S, crank,
                       [&](int bb, int64_t row, float val) {
                         h[static_cast<int64_t>(bb) * r + row] = __half2float(__ushort_as_half(mid[row])) * val;
                       },
                       kGemvThreads);
  }
  // ---- every CTA's h_scaled is in memory (and every peer is done with part)
  if (!grid_barrier(p.bar, gridDim.x)) {
    if (p.S > 1) cluster_sync();
    return;
  }
  // ---- phase 2: y = a (.) (U . h_scaled)
  {
    const float* h = p.h;
    const int r = p.r;
    quantise_input<NB>(xv, sp2,
                       [&](int bb, int k, float (&vv)[16]) {
                         const float4* hp = reinterpret_cast<const float4*>(h + static_cast<int64_t>(bb) * r + k);
#pragma unroll
                         for (int i = 0; i < 4; ++i) {
                           const float4 f = __ldcg(hp + i);
                           vv[4 * i] = f.x;
                           vv[4 * i + 1] = f.y;
                           vv[4 * i + 2] = f.z;
                           vv[4 * i + 3] = f.w;
                         }
                       },
                       kGemvThreads);
    __syncthreads();
    if (warp == kProducerWarp) {
      if (lane == 0) produce_rest(v2, sp2, &tm1, p.bw2, first2);
      __syncwarp();
    } else {
      consume_tiles<NB, false>(v2, xv, sp2, p.bw2, zero16, warp, lane);
    }
    if (p.S > 1) cluster_sync(); else __syncthreads();
    float* y = p.y;
    const uint16_t* a = p.a;
    const int m = p.m;
    cluster_reduce<NB>(xv, sp2, p.S, crank,
                       [&](int bb, int64_t row, float val) {
                         y[static_cast<int64_t>(bb) * m + row] = __half2float(__ushort_as_half(a[row])) * val;
                       },
                       kGemvThreads);
    if (p.S > 1) cluster_sync();
  }
}

// ------------------------------------------------------------------ host side

template <int NB>
static int dbf_max_clusters(int S, int smem_bytes) {
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
  int nclusters = 0;
  if (cudaFuncSetAttribute(dbf_small_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&nclusters, dbf_small_kernel<NB>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return nclusters;
}

static int dbf_bw(int NG, int S) { return (S == 1 || NG % (8 * S) == 0) ? 8 : 4; }

template <int NB>
static cudaError_t launch_dbf_small_nb(DbfParams p, const uint32_t* B1, const uint32_t* B2, cudaStream_t stream,
                                       int num_sms, int smem_cap) {
  using L = GemvLayout<NB>;
  // K split S (x digits within budget) and cluster count Q: all CTAs must be
  // co-resident (grid barrier), so Q never exceeds the occupancy limit
  const int T1 = (p.r + 15) / 16, T2 = (p.m + 15) / 16;
  const int NG1 = p.n / 128, NG2 = p.r / 128;
  for (int S = 1; S <= 8; S *= 2) {
    if (S > 1 && (S > NG1 || S > NG2)) break;
    DbfParams c = p;
    c.S = S;
    c.bw1 = dbf_bw(NG1, S);
    c.bw2 = dbf_bw(NG2, S);
    c.max_ng1 = ((NG1 + c.bw1 - 1) / c.bw1 + S - 1) / S * c.bw1;
    c.max_ng2 = ((NG2 + c.bw2 - 1) / c.bw2 + S - 1) / S * c.bw2;
    const int mng = c.max_ng1 > c.max_ng2 ? c.max_ng1 : c.max_ng2;
    if (mng * 4 * L::BLOCK > 72 * 1024 && S < 8) continue;
    int Q = num_sms / S;
    for (int iter = 0; iter < 3; ++iter) {
      c.max_tiles1 = (T1 + Q - 1) / Q;
      c.max_tiles2 = (T2 + Q - 1) / Q;
      c.ns1 = c.ns2 = 0;
      const int base = dbf_smem_layout<NB>(c).total;
      const int budget = smem_cap - base;
      const int per1 = ((c.max_ng1 + c.bw1 - 1) / c.bw1) * 256 * c.bw1 + 16;
      const int per2 = ((c.max_ng2 + c.bw2 - 1) / c.bw2) * 256 * c.bw2 + 16;
      c.ns1 = c.max_tiles1;
      c.ns2 = c.max_tiles2;
      if (c.ns1 * per1 + c.ns2 * per2 > budget) {
        c.ns1 = (budget / 2) / per1;
        c.ns2 = (budget / 2) / per2;
      }
      if (c.ns1 < 1 || c.ns2 < 1) break;
      const int smem = dbf_smem_layout<NB>(c).total;
      const int occ = dbf_max_clusters<NB>(S, smem);
      if (occ <= 0) break;
      if (occ < Q) {
        Q = occ;
        continue;
      }
      CUtensorMap tm2, tm1;
      if (!make_tmap_u32_rows(&tm2, B2, c.r, c.n / 32, 4 * c.bw1) ||
          !make_tmap_u32_rows(&tm1, B1, c.m, c.r / 32, 4 * c.bw2))
        return cudaErrorInvalidValue;
      cudaError_t err = cudaFuncSetAttribute(dbf_small_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (err != cudaSuccess) return err;
      if (getenv("W1_VERBOSE"))
        fprintf(stderr, "dbf plan: B=%d -> clusters=%d split=%d stages=%d/%d smem=%d\n", NB, Q, S, c.ns1, c.ns2, smem);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(Q * S));
      cfg.blockDim = dim3(kGemvThreads);
      cfg.dynamicSmemBytes = static_cast<size_t>(smem);
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
      return cudaLaunchKernelEx(&cfg, dbf_small_kernel<NB>, tm2, tm1, c);
    }
  }
  return cudaErrorInvalidConfiguration;
}

size_t dbf_tc_workspace_bytes(int64_t r, int64_t n, int64_t B);
cudaError_t launch_dbf_tc(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                          const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B, float* y,
                          void* workspace, cudaStream_t stream, int num_sms);

// Batches of at least this many rows run on the tensor-core path.
constexpr int64_t kDbfTensorMinBatch = 64;

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
  DbfParams p = {};
  p.a = a;
  p.mid = mid;
  p.b = b;
  p.bar = reinterpret_cast<unsigned int*>(workspace);
  p.h = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + 256);
  p.m = static_cast<int>(m);
  p.r = static_cast<int>(r);
  p.n = static_cast<int>(n);
  // batches of up to 8 rows through the fused small-batch kernel
  for (int64_t b0 = 0; b0 < B; b0 += 8) {
    const int nb = static_cast<int>((B - b0) < 8 ? (B - b0) : 8);
    p.x = x + b0 * n;
    p.y = y + b0 * m;
    cudaError_t err;
    switch (nb) {
      case 1: err = launch_dbf_small_nb<1>(p, B1, B2, stream, num_sms, smem_cap); break;
      case 2: err = launch_dbf_small_nb<2>(p, B1, B2, stream, num_sms, smem_cap); break;
      case 3: err = launch_dbf_small_nb<3>(p, B1, B2, stream, num_sms, smem_cap); break;
      case 4: err = launch_dbf_small_nb<4>(p, B1, B2, stream, num_sms, smem_cap); break;
      case 5: err = launch_dbf_small_nb<5>(p, B1, B2, stream, num_sms, smem_cap); break;
      case 6: err = launch_dbf_small_nb<6>(p, B1, B2, stream, num_sms, smem_cap); break;
      case 7: err = launch_dbf_small_nb<7>(p, B1, B2, stream, num_sms, smem_cap); break;
      default: err = launch_dbf_small_nb<8>(p, B1, B2, stream, num_sms, smem_cap); break;
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

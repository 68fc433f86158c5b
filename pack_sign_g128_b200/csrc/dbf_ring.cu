// DBF chain for groups of 5-8 batch rows: the joint V-D_mid-U kernel of
// dbf.cu built on the ring GEMV core (gemv_core.cuh: TMA-fed swizzled tiles,
// the sign bytes as the A operand of int8 mma.sync, 16 consumer warps), which
// measures faster than the direct core at these batch sizes.  Same phases as
// dbf_direct_kernel: both sign matrices' slices bulk-copied at kernel start,
// phase 1 on b (.) x with h_scaled = mid (.) h to the workspace (fp32), the
// bounded grid barrier, phase 2 on h_scaled with y = a (.) (...).
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cuda_fp16.h>

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

template <int NB>
__global__ void __launch_bounds__(kGemvThreads, 1)
    dbf_ring_kernel(const __grid_constant__ CUtensorMap tm2, const __grid_constant__ CUtensorMap tm1,
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
static int dbf_ring_max_clusters(int S, int smem_bytes) {
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
  if (ensure_dyn_smem(reinterpret_cast<const void*>(dbf_ring_kernel<NB>), smem_bytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&nclusters, dbf_ring_kernel<NB>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return nclusters;
}

static int dbf_bw(int NG, int S) { return (S == 1 || NG % (8 * S) == 0) ? 8 : 4; }

template <int NB>
static cudaError_t launch_dbf_ring_nb(DbfParams p, const uint32_t* B1, const uint32_t* B2, cudaStream_t stream,
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
      const int occ = dbf_ring_max_clusters<NB>(S, smem);
      if (occ <= 0) break;
      if (occ < Q) {
        Q = occ;
        continue;
      }
      CUtensorMap tm2, tm1;
      if (!make_tmap_u32_rows(&tm2, B2, c.r, c.n / 32, 4 * c.bw1) ||
          !make_tmap_u32_rows(&tm1, B1, c.m, c.r / 32, 4 * c.bw2))
        return cudaErrorInvalidValue;
      cudaError_t err = ensure_dyn_smem(reinterpret_cast<const void*>(dbf_ring_kernel<NB>), smem);
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
      return cudaLaunchKernelEx(&cfg, dbf_ring_kernel<NB>, tm2, tm1, c);
    }
  }
  return cudaErrorInvalidConfiguration;
}

}  // namespace w1

// Matrix-approximation measurement ("LLM binarization episode 01: DBF",
// section 8 "Current measurements": the relative Frobenius and spectral
// residuals of E = W - W_approx, each matrix normalised by its own norm,
// spectral norms by fixed-seed 32-iteration power iteration).
//
// residual_g128_kernel  E = W - w_hat for the group-128 sign code, with
//                       sum E^2 and sum W^2.  HBM-bound: reads W and the
//                       packed bytes once, writes E if asked.
// dbf_residual_kernel   the same for diag(a) U diag(mid) V diag(b): 128 x 128
//                       tiles of W_approx formed on CUDA cores (8 x 8 outputs
//                       per thread, +-1 times +-mid products summed over r in
//                       fp32), E and the sums in the epilogue; W_approx is
//                       never stored.  ALU-bound: 2 m n r flops.
// pi_* kernels          power iteration on A^T A in fp64 (A read as fp32):
//                       A v by a warp per row, A^T u by column partial sums
//                       over row chunks, the norm by one CTA.
//
// Every sum has a fixed order: a CTA reduces its threads through a fixed
// shuffle tree and then its warps in order; the last CTA to finish (a ticket
// counter) adds the per-CTA partials the same way, thread t taking partials
// t, t + 256, ... in order.  Results are bitwise
// reproducible for a given shape and device.
#include <algorithm>
#include <cstdint>

#include <cuda_fp16.h>

#include "w1_common.cuh"

namespace w1 {

namespace meas {
constexpr int kThreads = 256;
constexpr int kMaxResidualCtas = 8192;
constexpr int kPiChunks = 64;  // most row chunks of A^T u
}  // namespace meas

__device__ __forceinline__ float meas_half_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Fixed-order sum of one double per thread over a CTA of meas::kThreads; the
// result is valid in thread 0.
__device__ __forceinline__ double meas_block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < meas::kThreads / 32; ++w) s += red[w];
  return s;
}

// Per-CTA partial pair -> partials[cta] (cta = linear CTA index of ncta); the
// last CTA to finish adds all partials into out[0..1]: thread t takes
// partials t, t + kThreads, ... in order, then the fixed tree.
__device__ __forceinline__ void meas_finish_pair(double e2, double w2, double* partials, unsigned int* ticket,
                                                 double* out) {
  const unsigned int cta = blockIdx.y * gridDim.x + blockIdx.x;
  const unsigned int ncta = gridDim.x * gridDim.y;
  __shared__ double red[meas::kThreads / 32];
  __shared__ bool last;
  e2 = meas_block_sum(e2, red);
  w2 = meas_block_sum(w2, red);
  if (threadIdx.x == 0) {
    partials[2 * cta] = e2;
    partials[2 * cta + 1] = w2;
    __threadfence();
    last = atomicAdd(ticket, 1u) == ncta - 1;
  }
  __syncthreads();
  if (last) {  // uniform across the CTA
    __threadfence();
    double se = 0.0, sw = 0.0;
    for (unsigned int c = threadIdx.x; c < ncta; c += meas::kThreads) {
      se += __ldcg(partials + 2 * c);
      sw += __ldcg(partials + 2 * c + 1);
    }
    se = meas_block_sum(se, red);
    sw = meas_block_sum(sw, red);
    if (threadIdx.x == 0) {
      out[0] = se;
      out[1] = sw;
    }
  }
}

// ----------------------------------------------------------------- group-128 sign code

__global__ void __launch_bounds__(meas::kThreads) residual_g128_kernel(const float* __restrict__ W, int N, int K,
                                                                       const uint32_t* __restrict__ signs,
                                                                       const uint16_t* __restrict__ scales,
                                                                       float* __restrict__ E, double* partials,
                                                                       unsigned int* ticket, double* out) {
  pdl_wait();
  const int K4 = K >> 2, KW = K >> 5, NG = K >> 7;
  double e2 = 0.0, w2 = 0.0;
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    const float4* wr = reinterpret_cast<const float4*>(W + static_cast<size_t>(n) * K);
    const uint32_t* sr = signs + static_cast<size_t>(n) * KW;
    const uint16_t* cr = scales + static_cast<size_t>(n) * NG;
    float4* er = E ? reinterpret_cast<float4*>(E + static_cast<size_t>(n) * K) : nullptr;
#pragma unroll 4
    for (int k4 = threadIdx.x; k4 < K4; k4 += meas::kThreads) {
      const float4 w = __ldcs(wr + k4);
      const uint32_t bits = __ldg(sr + (k4 >> 3)) >> ((k4 & 7) * 4);
      const float s = meas_half_to_float(__ldg(cr + (k4 >> 5)));
      float4 e;
      e.x = w.x - ((bits & 1u) ? -s : s);
      e.y = w.y - ((bits & 2u) ? -s : s);
      e.z = w.z - ((bits & 4u) ? -s : s);
      e.w = w.w - ((bits & 8u) ? -s : s);
      e2 += static_cast<double>(e.x) * e.x + static_cast<double>(e.y) * e.y + static_cast<double>(e.z) * e.z +
            static_cast<double>(e.w) * e.w;
      w2 += static_cast<double>(w.x) * w.x + static_cast<double>(w.y) * w.y + static_cast<double>(w.z) * w.z +
            static_cast<double>(w.w) * w.w;
      if (er) __stcs(er + k4, e);
    }
  }
  meas_finish_pair(e2, w2, partials, ticket, out);
}

// ----------------------------------------------------------------- DBF chain

namespace dres {
constexpr int kTile = 128;  // rows and columns of W per CTA
constexpr int kMicro = 8;   // rows and columns per thread
constexpr int kChunk = 32;  // r per staging step (one U word per row)
}  // namespace dres

struct DbfResParams {
  const float* W;
  const uint16_t* a;
  const uint32_t* U;  // [m][r/32]
  const uint16_t* mid;
  const uint32_t* V;  // [r][n/32]
  const uint16_t* b;
  float* E;
  int m, r, n;
  double* partials;
  unsigned int* ticket;
  double* out;
};

__global__ void __launch_bounds__(meas::kThreads) dbf_residual_kernel(DbfResParams p) {
  using namespace dres;
  __shared__ uint32_t Vs[kChunk][kTile / 32];
  __shared__ float Ms[kChunk];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int i0 = blockIdx.y * kTile + ty * kMicro;  // this thread's first row
  const int j0 = blockIdx.x * kTile + tx * kMicro;  // and first column
  const int rw = p.r >> 5, nw = p.n >> 5;
  pdl_wait();
  float acc[kMicro][kMicro];
#pragma unroll
  for (int u = 0; u < kMicro; ++u)
#pragma unroll
    for (int v = 0; v < kMicro; ++v) acc[u][v] = 0.f;

  for (int kc = 0; kc < rw; ++kc) {
    __syncthreads();
    if (threadIdx.x < kChunk * (kTile / 32)) {
      const int kk = threadIdx.x >> 2, c = threadIdx.x & 3;
      Vs[kk][c] = __ldg(p.V + static_cast<size_t>(kc * kChunk + kk) * nw + (blockIdx.x * kTile >> 5) + c);
    } else if (threadIdx.x < kChunk * (kTile / 32) + kChunk) {
      const int kk = threadIdx.x - kChunk * (kTile / 32);
      Ms[kk] = meas_half_to_float(__ldg(p.mid + kc * kChunk + kk));
    }
    uint32_t uw[kMicro];
#pragma unroll
    for (int u = 0; u < kMicro; ++u) uw[u] = __ldg(p.U + static_cast<size_t>(i0 + u) * rw + kc);
    __syncthreads();
    const int vshift = (tx * kMicro) & 31, vword = (tx * kMicro) >> 5;
#pragma unroll 4
    for (int kk = 0; kk < kChunk; ++kk) {
      const float mk = Ms[kk];
      const uint32_t vb = Vs[kk][vword] >> vshift;
      float vm[kMicro], su[kMicro];
#pragma unroll
      for (int v = 0; v < kMicro; ++v) vm[v] = ((vb >> v) & 1u) ? -mk : mk;
#pragma unroll
      for (int u = 0; u < kMicro; ++u) su[u] = ((uw[u] >> kk) & 1u) ? -1.f : 1.f;
#pragma unroll
      for (int u = 0; u < kMicro; ++u)
#pragma unroll
        for (int v = 0; v < kMicro; ++v) acc[u][v] = fmaf(su[u], vm[v], acc[u][v]);
    }
  }

  // W_approx = (acc a_i) b_j in fp32; E = W - W_approx.
  double e2 = 0.0, w2 = 0.0;
  float bj[kMicro];
#pragma unroll
  for (int v = 0; v < kMicro; ++v) bj[v] = meas_half_to_float(__ldg(p.b + j0 + v));
#pragma unroll
  for (int u = 0; u < kMicro; ++u) {
    const float ai = meas_half_to_float(__ldg(p.a + i0 + u));
    const float4* wr = reinterpret_cast<const float4*>(p.W + static_cast<size_t>(i0 + u) * p.n + j0);
    const float4 w0 = __ldcs(wr), w1 = __ldcs(wr + 1);
    const float wv[kMicro] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float ev[kMicro];
#pragma unroll
    for (int v = 0; v < kMicro; ++v) {
      ev[v] = wv[v] - (acc[u][v] * ai) * bj[v];
      e2 += static_cast<double>(ev[v]) * ev[v];
      w2 += static_cast<double>(wv[v]) * wv[v];
    }
    if (p.E) {
      float4* er = reinterpret_cast<float4*>(p.E + static_cast<size_t>(i0 + u) * p.n + j0);
      __stcs(er, make_float4(ev[0], ev[1], ev[2], ev[3]));
      __stcs(er + 1, make_float4(ev[4], ev[5], ev[6], ev[7]));
    }
  }
  meas_finish_pair(e2, w2, p.partials, p.ticket, p.out);
}

// ----------------------------------------------------------------- power iteration

// w = v0 (as fp64) and ss = sum v0^2; one CTA.
__global__ void __launch_bounds__(meas::kThreads) pi_init_kernel(const float* v0, int n, double* w, double* ss) {
  __shared__ double red[meas::kThreads / 32];
  pdl_wait();
  double s = 0.0;
  for (int j = threadIdx.x; j < n; j += meas::kThreads) {
    const double v = v0[j];
    w[j] = v;
    s += v * v;
  }
  s = meas_block_sum(s, red);
  if (threadIdx.x == 0) *ss = s;
}

// u[i] = sum_j A[i][j] * w[j] / sqrt(ss), a warp per row (ss = 0 gives u = 0).
__global__ void __launch_bounds__(meas::kThreads) pi_av_kernel(const float* __restrict__ A, int m, int n,
                                                               const double* __restrict__ w, const double* ss,
                                                               double* __restrict__ u) {
  pdl_wait();
  const double s = *ss;
  const double inv = s > 0.0 ? 1.0 / sqrt(s) : 0.0;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (meas::kThreads / 32) + (threadIdx.x >> 5);
  if (row >= m) return;
  const float4* ar = reinterpret_cast<const float4*>(A + static_cast<size_t>(row) * n);
  double acc = 0.0;
  for (int j4 = lane; j4 < (n >> 2); j4 += 32) {
    const float4 a = __ldg(ar + j4);
    const double* wj = w + 4 * j4;
    acc += static_cast<double>(a.x) * wj[0] + static_cast<double>(a.y) * wj[1] + static_cast<double>(a.z) * wj[2] +
           static_cast<double>(a.w) * wj[3];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) u[row] = acc * inv;
}

// part[c][j] = sum over rows i of chunk c of A[i][j] * u[i], rows ascending.
__global__ void __launch_bounds__(meas::kThreads) pi_atu_kernel(const float* __restrict__ A, int m, int n,
                                                                const double* __restrict__ u, int rows_per_chunk,
                                                                double* __restrict__ part) {
  pdl_wait();
  const int j = blockIdx.x * meas::kThreads + threadIdx.x;
  const int c = blockIdx.y;
  if (j >= n) return;
  const int r0 = c * rows_per_chunk, r1 = min(m, r0 + rows_per_chunk);
  double acc = 0.0;
  for (int i = r0; i < r1; ++i) acc += static_cast<double>(__ldg(A + static_cast<size_t>(i) * n + j)) * u[i];
  part[static_cast<size_t>(c) * n + j] = acc;
}

// w[j] = sum_c part[c][j] (c ascending), ss = sum w^2; one CTA.
__global__ void __launch_bounds__(meas::kThreads) pi_reduce_kernel(const double* __restrict__ part, int chunks, int n,
                                                                   double* __restrict__ w, double* ss) {
  __shared__ double red[meas::kThreads / 32];
  pdl_wait();
  double s = 0.0;
  for (int j = threadIdx.x; j < n; j += meas::kThreads) {
    double v = 0.0;
    for (int c = 0; c < chunks; ++c) v += part[static_cast<size_t>(c) * n + j];
    w[j] = v;
    s += v * v;
  }
  s = meas_block_sum(s, red);
  if (threadIdx.x == 0) *ss = s;
}

// sigma = sqrt(sum u^2); one CTA.
__global__ void __launch_bounds__(meas::kThreads) pi_norm_kernel(const double* __restrict__ u, int m, double* sigma) {
  __shared__ double red[meas::kThreads / 32];
  pdl_wait();
  double s = 0.0;
  for (int i = threadIdx.x; i < m; i += meas::kThreads) s += u[i] * u[i];
  s = meas_block_sum(s, red);
  if (threadIdx.x == 0) *sigma = sqrt(s);
}

// ----------------------------------------------------------------- host side

// Workspace layout (bytes, 256-aligned pieces): ticket | partials [8192][2] |
// u [m] | w [n] | ss | part [kPiChunks][n].
static size_t meas_align(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

size_t measure_workspace_bytes(int64_t m, int64_t n) {
  if (m <= 0 || n <= 0) return 0;
  return meas_align(16) + meas_align(sizeof(double) * 2 * meas::kMaxResidualCtas) +
         meas_align(sizeof(double) * m) + meas_align(sizeof(double) * n) + meas_align(sizeof(double)) +
         meas_align(sizeof(double) * meas::kPiChunks * n);
}

struct MeasWs {
  unsigned int* ticket;
  double* partials;
  double* u;
  double* w;
  double* ss;
  double* part;
};

static MeasWs meas_ws(void* base, int64_t m, int64_t n) {
  char* p = static_cast<char*>(base);
  MeasWs ws;
  ws.ticket = reinterpret_cast<unsigned int*>(p);
  p += meas_align(16);
  ws.partials = reinterpret_cast<double*>(p);
  p += meas_align(sizeof(double) * 2 * meas::kMaxResidualCtas);
  ws.u = reinterpret_cast<double*>(p);
  p += meas_align(sizeof(double) * m);
  ws.w = reinterpret_cast<double*>(p);
  p += meas_align(sizeof(double) * n);
  ws.ss = reinterpret_cast<double*>(p);
  p += meas_align(sizeof(double));
  ws.part = reinterpret_cast<double*>(p);
  return ws;
}

template <typename Kern, typename... Args>
static cudaError_t meas_launch(Kern kernel, dim3 grid, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(meas::kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_residual_g128(const float* W, int64_t N, int64_t K, const uint32_t* signs, const uint16_t* scales,
                                 float* E, double* sums, void* workspace, cudaStream_t stream, int num_sms) {
  MeasWs ws = meas_ws(workspace, N, K);
  cudaError_t e = cudaMemsetAsync(ws.ticket, 0, sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(std::min<int64_t>(N, std::min(8 * num_sms, meas::kMaxResidualCtas)));
  return meas_launch(residual_g128_kernel, dim3(grid), stream, W, static_cast<int>(N), static_cast<int>(K), signs,
                     scales, E, ws.partials, ws.ticket, sums);
}

cudaError_t launch_dbf_residual(const float* W, const uint16_t* a, const uint32_t* B1, const uint16_t* mid,
                                const uint32_t* B2, const uint16_t* b, int64_t m, int64_t r, int64_t n, float* E,
                                double* sums, void* workspace, cudaStream_t stream) {
  MeasWs ws = meas_ws(workspace, m, n);
  const int64_t tiles = (m / dres::kTile) * (n / dres::kTile);
  if (tiles > meas::kMaxResidualCtas || n / dres::kTile > 65535 || m / dres::kTile > 65535)
    return cudaErrorNotSupported;
  cudaError_t e = cudaMemsetAsync(ws.ticket, 0, sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  DbfResParams p;
  p.W = W;
  p.a = a;
  p.U = B1;
  p.mid = mid;
  p.V = B2;
  p.b = b;
  p.E = E;
  p.m = static_cast<int>(m);
  p.r = static_cast<int>(r);
  p.n = static_cast<int>(n);
  p.partials = ws.partials;
  p.ticket = ws.ticket;
  p.out = sums;
  return meas_launch(dbf_residual_kernel, dim3(static_cast<unsigned>(n / dres::kTile),
                                               static_cast<unsigned>(m / dres::kTile)),
                     stream, p);
}

cudaError_t launch_power_iteration(const float* A, int64_t m, int64_t n, const float* v0, int64_t iters,
                                   double* sigma, void* workspace, cudaStream_t stream, int num_sms) {
  MeasWs ws = meas_ws(workspace, m, n);
  const int M = static_cast<int>(m), Nn = static_cast<int>(n);
  const int col_blocks = (Nn + meas::kThreads - 1) / meas::kThreads;
  int chunks = 1;
  while (chunks < meas::kPiChunks && col_blocks * chunks < 2 * num_sms && chunks * 2 <= M) chunks *= 2;
  const int rows_per_chunk = (M + chunks - 1) / chunks;
  const dim3 av_grid((M + meas::kThreads / 32 - 1) / (meas::kThreads / 32));
  cudaError_t e = meas_launch(pi_init_kernel, dim3(1), stream, v0, Nn, ws.w, ws.ss);
  for (int64_t it = 0; it < iters && e == cudaSuccess; ++it) {
    e = meas_launch(pi_av_kernel, av_grid, stream, A, M, Nn, static_cast<const double*>(ws.w),
                    static_cast<const double*>(ws.ss), ws.u);
    if (e == cudaSuccess)
      e = meas_launch(pi_atu_kernel, dim3(col_blocks, chunks), stream, A, M, Nn, static_cast<const double*>(ws.u),
                      rows_per_chunk, ws.part);
    if (e == cudaSuccess)
      e = meas_launch(pi_reduce_kernel, dim3(1), stream, static_cast<const double*>(ws.part), chunks, Nn, ws.w,
                      ws.ss);
  }
  if (e == cudaSuccess)
    e = meas_launch(pi_av_kernel, av_grid, stream, A, M, Nn, static_cast<const double*>(ws.w),
                    static_cast<const double*>(ws.ss), ws.u);
  if (e == cudaSuccess) e = meas_launch(pi_norm_kernel, dim3(1), stream, static_cast<const double*>(ws.u), M, sigma);
  return e;
}

// ---------------------------------------------------------------- launch floor
// Reads two byte ranges (a product's sign words and scales) with 16-byte
// loads, every load of a thread issued before any is used, and folds them
// into one word per CTA (so that the loads cannot be dropped).  It does the
// memory work of a decode product and nothing else: back-to-back launches of
// it give the per-launch floor a product kernel is measured against.
// early: the loads are issued before the grid dependency wait (as a product
// with W1_GEMV_STATIC_WEIGHTS does), else after it.
constexpr int kProbeThreads = 256;
constexpr int kProbeLoads = 8;  // 16-byte loads per thread and pass
__global__ void __launch_bounds__(kProbeThreads) stream_probe_kernel(const uint4* __restrict__ a, int64_t na,
                                                                     const uint4* __restrict__ b, int64_t nb,
                                                                     int early, uint32_t* __restrict__ out) {
  pdl_launch_dependents();
  if (!early) pdl_wait();
  const int64_t n = na + nb;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kProbeThreads;
  uint32_t acc = 0;
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * kProbeThreads + threadIdx.x; i0 < n;
       i0 += kProbeLoads * stride) {
    uint4 v[kProbeLoads];
#pragma unroll
    for (int j = 0; j < kProbeLoads; ++j) {
      const int64_t i = i0 + j * stride;
      v[j] = i < na ? __ldcs(a + i) : (i < n ? __ldcs(b + (i - na)) : make_uint4(0, 0, 0, 0));
    }
#pragma unroll
    for (int j = 0; j < kProbeLoads; ++j) acc += v[j].x ^ v[j].y ^ v[j].z ^ v[j].w;
  }
  if (early) pdl_wait();
  acc = __reduce_add_sync(0xFFFFFFFFu, acc);
  if ((threadIdx.x & 31) == 0) atomicAdd(out + blockIdx.x, acc);
}

cudaError_t launch_stream_probe(const void* a, int64_t abytes, const void* b, int64_t bbytes, int ctas, bool early,
                                uint32_t* out, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(kProbeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stream_probe_kernel, static_cast<const uint4*>(a), abytes / 16,
                            static_cast<const uint4*>(b), bbytes / 16, early ? 1 : 0, out);
}

}  // namespace w1

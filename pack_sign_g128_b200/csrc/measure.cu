// Matrix-approximation measurement ("LLM binarization episode 01: DBF",
// section 8 "Current measurements": the relative Frobenius and spectral
// residuals of E = W - W_approx, each matrix normalised by its own norm,
// spectral norms by fixed-seed 32-iteration power iteration).
//
// residual_g128_kernel  E = W - w_hat for the group-128 sign code, with
//                       sum E^2 and sum W^2.  HBM-bound: reads W and the
//                       packed bytes once, writes E if asked.
// dres_* + sign GEMM    the same for diag(a) U diag(mid) V diag(b): W_approx^T
//                       formed on the tensor cores by the sign GEMM
//                       (sign_gemm.cu: +-1 rows of U times H = mid (.) V^T in
//                       fp16, exact products, fp32 accumulation, row diagonal
//                       a, token scale b), then E and the sums through a
//                       transposing shared tile.  2 m n r flops on tcgen05.
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
// W_approx = diag(a) U diag(mid) V diag(b) on the tensor cores: with
// H[j][k] = mid_k V_kj (fp16, exact: a sign on an fp16 value), the sign GEMM
// (sign_gemm.cu, +-1 rows of U, fp32 accumulation over k in TMEM) forms
// W_approx^T[j][i] = (a_i sum_k U_ik H[j][k]) b_j with n as its token rows;
// then E = W - W_approx and the sums, through a transposing shared tile.

// H [n][r] (fp16 bits: mid_k with V's sign) and bs [n] = b as float.  One
// warp per 32 x 32 block of V: lane l holds row k = 32 kb + l's word.
__global__ void __launch_bounds__(meas::kThreads) dres_h_kernel(const uint32_t* __restrict__ V,
                                                                 const uint16_t* __restrict__ mid,
                                                                 const uint16_t* __restrict__ b, int r, int n,
                                                                 uint16_t* __restrict__ H, float* __restrict__ bs) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * (meas::kThreads / 32) + (threadIdx.x >> 5);
  const int nw = n >> 5, rw = r >> 5;
  if (blk < static_cast<int64_t>(nw) * rw) {  // warp-uniform
    const int kb = static_cast<int>(blk / nw), jb = static_cast<int>(blk - static_cast<int64_t>(kb) * nw);
    const int k = kb * 32 + lane;
    const uint32_t w = __ldg(V + static_cast<int64_t>(k) * nw + jb);
    const uint32_t mk = __ldg(mid + k);
#pragma unroll 4
    for (int jj = 0; jj < 32; ++jj)
      H[static_cast<int64_t>(jb * 32 + jj) * r + k] = static_cast<uint16_t>(mk ^ (((w >> jj) & 1u) << 15));
    if (kb == 0) bs[jb * 32 + lane] = meas_half_to_float(__ldg(b + jb * 32 + lane));
  }
  pdl_launch_dependents();
}

// E = W - W_approx (W_approx read transposed through a 64 x 64 shared tile),
// sum E^2 and sum W^2.  CTAs stride over the tiles.
namespace dres {
constexpr int kT = 64;
}
__global__ void __launch_bounds__(meas::kThreads) dres_e_kernel(const float* __restrict__ W,
                                                                 const float* __restrict__ WaT, int m, int n,
                                                                 float* __restrict__ E, double* partials,
                                                                 unsigned int* ticket, double* out) {
  using dres::kT;
  __shared__ float T[kT][kT + 1];
  pdl_wait();
  const int tn = n / kT, tiles = (m / kT) * tn;
  double e2 = 0.0, w2 = 0.0;
  for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
    const int i0 = (t / tn) * kT, j0 = (t % tn) * kT;
    __syncthreads();  // the previous tile's reads are done
    for (int e = threadIdx.x; e < kT * kT; e += meas::kThreads) {
      const int jj = e / kT, ii = e % kT;
      T[jj][ii] = __ldcs(WaT + static_cast<int64_t>(j0 + jj) * m + i0 + ii);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kT * kT; e += meas::kThreads) {
      const int ii = e / kT, jj = e % kT;
      const int64_t o = static_cast<int64_t>(i0 + ii) * n + j0 + jj;
      const float w = __ldcs(W + o);
      const float ev = w - T[jj][ii];
      e2 += static_cast<double>(ev) * ev;
      w2 += static_cast<double>(w) * w;
      if (E) __stcs(E + o, ev);
    }
  }
  meas_finish_pair(e2, w2, partials, ticket, out);
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

// The sign GEMM's parameter block and launcher (sign_gemm.cu, the same
// translation unit of libw1).
template <bool HALF_OUT>
cudaError_t launch_sg_gemm(const SgParams& p, const void* bmat, int64_t bcols, cudaStream_t stream, int num_sms);

// Workspace of dbf_residual: the measurement header, H [n][r] fp16,
// W_approx^T [n][m] fp32, b [n] fp32.
struct DresWs {
  size_t h, wat, bs, total;
};
static DresWs dres_ws(int64_t m, int64_t r, int64_t n) {
  DresWs d;
  d.h = meas_align(measure_workspace_bytes(m, n));
  d.wat = d.h + meas_align(static_cast<size_t>(2) * n * r);
  d.bs = d.wat + meas_align(static_cast<size_t>(4) * n * m);
  d.total = d.bs + meas_align(static_cast<size_t>(4) * n);
  return d;
}
size_t dbf_residual_workspace_bytes(int64_t m, int64_t r, int64_t n) {
  if (m <= 0 || r <= 0 || n <= 0) return 0;
  return dres_ws(m, r, n).total;
}

cudaError_t launch_dbf_residual(const float* W, const uint16_t* a, const uint32_t* B1, const uint16_t* mid,
                                const uint32_t* B2, const uint16_t* b, int64_t m, int64_t r, int64_t n, float* E,
                                double* sums, void* workspace, cudaStream_t stream, int num_sms) {
  MeasWs ws = meas_ws(workspace, m, n);
  const DresWs L = dres_ws(m, r, n);
  unsigned char* base = static_cast<unsigned char*>(workspace);
  uint16_t* H = reinterpret_cast<uint16_t*>(base + L.h);
  float* WaT = reinterpret_cast<float*>(base + L.wat);
  float* bs = reinterpret_cast<float*>(base + L.bs);
  cudaError_t e = cudaMemsetAsync(ws.ticket, 0, sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  const int64_t hwarps = (n / 32) * (r / 32);
  e = meas_launch(dres_h_kernel, dim3(static_cast<unsigned>((hwarps + 7) / 8)), stream, B2, mid, b,
                  static_cast<int>(r), static_cast<int>(n), H, bs);
  if (e != cudaSuccess) return e;
  SgParams p = {};
  p.signs = B1;
  p.gscales = nullptr;
  p.rdiag = a;
  p.s1 = bs;
  p.out_f = WaT;
  p.M = static_cast<int>(n);
  p.rows = static_cast<int>(m);
  p.K = static_cast<int>(r);
  e = launch_sg_gemm<false>(p, H, r, stream, num_sms);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (m / dres::kT) * (n / dres::kT);
  const int grid = static_cast<int>(std::min<int64_t>(tiles, std::min(8 * num_sms, meas::kMaxResidualCtas)));
  return meas_launch(dres_e_kernel, dim3(static_cast<unsigned>(grid)), stream, W, static_cast<const float*>(WaT),
                     static_cast<int>(m), static_cast<int>(n), E, ws.partials, ws.ticket, sums);
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

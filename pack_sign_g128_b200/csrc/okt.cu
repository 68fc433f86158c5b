// Online orthogonal-Kronecker rotation of the activations (zhichai.net post
// on BWLA, section 3 "OKT": one orthogonal rotation of the input space,
// factored as H kron R with n1 n2 = K; section 5: the weights are binarised
// in the rotated coordinates and the activations take the same rotation, so
// the product is unchanged).
//
// For y = W x with W [N][K], the packed weights hold W (H kron R), and the
// activations become x_rot = (H kron R)^T x.  With x[i n2 + j] read as
// X[i][j] (n1 x n2, row-major), that is x_rot = H^T X R.
//
// okt_rotate_kernel: one CTA per (batch row, slice of RS rows i of the
// output view).  It stages the row's x (bf16), all of R and its RS columns of
// H in shared memory, then computes Z = H[:, slice]^T X (RS x n2, a length-n1
// dot per element) and x_rot[slice, :] = Z R (a length-n2 dot per element),
// each dot in fp32 in a fixed order.  No CTA repeats another's arithmetic.
// Where a CTA has fewer outputs than threads, T threads split each dot into
// contiguous parts, so the dependent chain per thread is n1 / T (n2 / T)
// long; the staging loads and shared-memory issue, not the FMAs, set the
// time.
// The work is a few MFLOP per row and the bytes are a few tens of KB, so a
// launch costs about its latency; the kernel lets the next kernel (the
// product) launch at once, so that product can stage its weights meanwhile.
#include <cstdint>

#include "w1_common.cuh"

namespace w1 {

namespace okt {
constexpr int kThreads = 256;
constexpr int kMaxN2 = 128;
constexpr int kMaxN1 = 1024;
constexpr int kMaxK = 65536;
}  // namespace okt

struct OktParams {
  const float* H;     // [n1][n1]
  const float* R;     // [n2][n2]
  const uint16_t* x;  // [B][K] bf16
  float* out;         // [B][K] fp32
  int n1, n2, K, RS;
  int T;              // threads per output (a power of two, RS n2 T <= kThreads)
  int early;          // H and R may be read before the preceding kernel completes
};

__device__ __forceinline__ float bf16_to_f32(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

// Shared memory: Xs bf16 [K] | Rs fp32 [n2 n2] | Hs fp32 [n1][RS] | Zs fp32 [RS][n2]
// | Ps fp32 [kThreads] (partial sums).
static size_t okt_smem_bytes(int n1, int n2, int RS) {
  const size_t K = static_cast<size_t>(n1) * n2;
  return ((K * 2 + 15) / 16) * 16 + static_cast<size_t>(n2) * n2 * 4 + static_cast<size_t>(n1) * RS * 4 +
         static_cast<size_t>(RS) * n2 * 4 + okt::kThreads * 4;
}

// All of R, and columns i0 .. i0 + RS - 1 of H (zero past n1), into shared memory.
__device__ __forceinline__ void okt_load_factors(const OktParams& p, float* Rs, float* Hs, int i0, int tid) {
  const int n1 = p.n1, n2 = p.n2, RS = p.RS;
  const int rr = n2 * n2;
  const int r4 = rr >> 2;  // R is 16-byte aligned
  const float4* R4 = reinterpret_cast<const float4*>(p.R);
  for (int t = tid; t < r4; t += okt::kThreads) reinterpret_cast<float4*>(Rs)[t] = __ldg(R4 + t);
  for (int t = (r4 << 2) + tid; t < rr; t += okt::kThreads) Rs[t] = __ldg(p.R + t);
  for (int t = tid; t < n1 * RS; t += okt::kThreads) {
    const int pp = t / RS, r = t - pp * RS;
    const int i = i0 + r;
    Hs[t] = i < n1 ? __ldg(p.H + static_cast<size_t>(pp) * n1 + i) : 0.f;
  }
}

__global__ void __launch_bounds__(okt::kThreads) okt_rotate_kernel(OktParams p) {
  extern __shared__ __align__(16) unsigned char okt_smem[];
  const int n1 = p.n1, n2 = p.n2, K = p.K, RS = p.RS;
  const int b = blockIdx.y;
  const int i0 = blockIdx.x * RS;
  const int tid = threadIdx.x;
  uint16_t* Xs = reinterpret_cast<uint16_t*>(okt_smem);
  float* Rs = reinterpret_cast<float*>(okt_smem + ((static_cast<size_t>(K) * 2 + 15) / 16) * 16);
  float* Hs = Rs + n2 * n2;
  float* Zs = Hs + n1 * RS;

  if (p.early) okt_load_factors(p, Rs, Hs, i0, tid);
  // The product that follows may launch now; it reads x_rot only after this
  // grid has completed (its own dependent-launch wait).
  pdl_launch_dependents();
  pdl_wait();
  if (!p.early) okt_load_factors(p, Rs, Hs, i0, tid);
  {
    const uint4* x4 = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(b) * K);
    for (int t = tid; t < (K >> 3); t += okt::kThreads) reinterpret_cast<uint4*>(Xs)[t] = x4[t];
  }
  __syncthreads();

  // Z[r][q] = sum_p H[p][i0 + r] X[p][q] and then
  // x_rot[i0 + r][j] = sum_q Z[r][q] R[q][j].  With nout = RS n2 outputs per
  // phase and nout T <= kThreads, T threads share an output: thread (t, o)
  // sums the t-th contiguous part of the dot, ascending, and the T partials
  // are added in order of t.  With nout > kThreads (T = 1) a thread takes
  // outputs o, o + kThreads, ...  Every sum has a fixed order for a given
  // shape and batch size.
  const int nout = RS * n2;
  const int T = p.T;
  float* Ps = Zs + RS * n2;  // [T][nout] partial sums (T > 1)
  const int part = tid / nout, po = tid - part * nout;
  if (T > 1) {
    if (part < T) {
      const int r = po / n2, q = po - r * n2;
      const int p0 = (part * n1) / T, p1 = ((part + 1) * n1) / T;
      float z = 0.f;
#pragma unroll 4
      for (int pp = p0; pp < p1; ++pp) z = fmaf(Hs[pp * RS + r], bf16_to_f32(Xs[pp * n2 + q]), z);
      Ps[part * nout + po] = z;
    }
    __syncthreads();
    if (tid < nout) {
      float z = Ps[tid];
      for (int t = 1; t < T; ++t) z += Ps[t * nout + tid];
      Zs[tid] = z;
    }
  } else {
    for (int o = tid; o < nout; o += okt::kThreads) {
      const int r = o / n2, q = o - r * n2;
      float z = 0.f;
#pragma unroll 4
      for (int pp = 0; pp < n1; ++pp) z = fmaf(Hs[pp * RS + r], bf16_to_f32(Xs[pp * n2 + q]), z);
      Zs[o] = z;
    }
  }
  __syncthreads();

  float* out = p.out + static_cast<size_t>(b) * K;
  if (T > 1) {
    if (part < T) {
      const int r = po / n2, j = po - r * n2;
      const int q0 = (part * n2) / T, q1 = ((part + 1) * n2) / T;
      const float* z = Zs + r * n2;
      float v = 0.f;
#pragma unroll 4
      for (int q = q0; q < q1; ++q) v = fmaf(z[q], Rs[q * n2 + j], v);
      Ps[part * nout + po] = v;
    }
    __syncthreads();
    if (tid < nout) {
      const int r = tid / n2, j = tid - r * n2;
      float v = Ps[tid];
      for (int t = 1; t < T; ++t) v += Ps[t * nout + tid];
      if (i0 + r < n1) out[static_cast<size_t>(i0 + r) * n2 + j] = v;
    }
  } else {
    for (int o = tid; o < nout; o += okt::kThreads) {
      const int r = o / n2, j = o - r * n2;
      if (i0 + r >= n1) continue;
      const float* z = Zs + r * n2;
      float v = 0.f;
#pragma unroll 4
      for (int q = 0; q < n2; ++q) v = fmaf(z[q], Rs[q * n2 + j], v);
      out[static_cast<size_t>(i0 + r) * n2 + j] = v;
    }
  }
}

// Rows of the output view per CTA.  Start from the smallest power of two (at
// most 8) that keeps B ceil(n1 / RS) CTAs within one wave; fewer rows per CTA
// spread the staging loads over more SMs, more rows cut the repeated reads
// of R (every CTA stages all of it).  Then shrink RS to one output per
// thread (RS n2 <= kThreads) if the grid stays within two CTAs per SM;
// otherwise take the smallest RS that fits two per SM.
static int okt_rows_per_cta(int n1, int n2, int B, int num_sms) {
  auto ctas = [&](int rs) { return static_cast<int64_t>(B) * ((n1 + rs - 1) / rs); };
  int rs1 = 1;
  while (rs1 < 8 && ctas(rs1) > num_sms) rs1 *= 2;
  int rs2 = rs1;
  while (rs2 > 1 && rs2 * n2 > okt::kThreads) rs2 /= 2;
  if (ctas(rs2) <= 2 * static_cast<int64_t>(num_sms)) return rs2;
  int rs = rs2;
  while (rs < 8 && ctas(rs) > 2 * static_cast<int64_t>(num_sms)) rs *= 2;
  return rs;
}

// Threads per output: the largest power of two T <= 8 with RS n2 T <= kThreads.
static int okt_threads_per_output(int nout) {
  int t = 1;
  while (t < 8 && nout * (2 * t) <= okt::kThreads) t *= 2;
  return t;
}

bool okt_shape_ok(int64_t n1, int64_t n2, int64_t K) {
  return n1 >= 1 && n2 >= 1 && n1 <= okt::kMaxN1 && n2 <= okt::kMaxN2 && n1 * n2 == K && K <= okt::kMaxK;
}

cudaError_t launch_okt_rotate(const float* H, int n1, const float* R, int n2, const uint16_t* x, int B, float* out,
                              bool early, cudaStream_t stream, int num_sms, int smem_optin) {
  OktParams p;
  p.H = H;
  p.R = R;
  p.x = x;
  p.out = out;
  p.n1 = n1;
  p.n2 = n2;
  p.K = n1 * n2;
  p.RS = okt_rows_per_cta(n1, n2, B, num_sms);
  p.T = okt_threads_per_output(p.RS * n2);
  p.early = early ? 1 : 0;
  const size_t smem = okt_smem_bytes(n1, n2, p.RS);
  if (smem > static_cast<size_t>(smem_optin)) return cudaErrorNotSupported;
  const cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(okt_rotate_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((n1 + p.RS - 1) / p.RS), static_cast<unsigned>(B), 1);
  cfg.blockDim = dim3(okt::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, okt_rotate_kernel, p);
}

}  // namespace w1

// DBF chain for many batch rows (B > 8) on tcgen05 tensor cores.
//
//   y = a (.) ( U . ( mid (.) ( V . ( b (.) x ) ) ) )      ("LLM binarization
//   episode 01: DBF", section 4 -- the chain, evaluated in order)
//
// Both binary products are plain +-1 contractions (no group scales) and run
// on the shared sign GEMM (sign_gemm.cu), each 128 x 128 output tile
// accumulating all of K in one TMEM accumulator:
//  1. sg_prep_kernel: x_s[t] = fp16( b (.) x[t] * 2^c_t ) with a per-row
//     power of two putting max |b x| in [2^14, 2^15) (exact scaling; fp16
//     keeps 11 significant bits of b x, which bf16 would not), and the row's
//     L1 norm, from which a second power of two d_t bounds |mid (.) h| * 2^d_t
//     below 2^15 so the fp16 intermediate cannot overflow.
//  2. sg_gemm<fp16 out>: D = V . x_s^T; epilogue h_s[t][j] = fp16(mid_j D 2^(d_t - c_t)).
//  3. sg_gemm<fp32 out>: D = U . h_s^T; epilogue y[t][i] = a_i D 2^-d_t.
// Products of +-1 and fp16 are exact; accumulation is fp32.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "w1_common.cuh"

namespace w1 {

struct SgParams;

namespace dbftc {
// Workspace of the tensor path (after the 256-byte barrier header):
// per-row scales (float [B] 2^-c_t, float [B] 2^d_t), x_s fp16 [B][n],
// h_s fp16 [B][r].
struct Ws {
  size_t cscale, dscale, dinv, xs, hs, total;
};
__host__ __device__ inline Ws ws_layout(int64_t B, int64_t r, int64_t n) {
  Ws w;
  size_t off = 256;
  w.cscale = off;
  off += (4 * B + 255) / 256 * 256;
  w.dscale = off;
  off += (4 * B + 255) / 256 * 256;
  w.dinv = off;
  off += (4 * B + 255) / 256 * 256;
  w.xs = off;
  off += (2 * B * n + 1023) / 1024 * 1024;
  w.hs = off;
  off += (2 * B * r + 1023) / 1024 * 1024;
  w.total = off;
  return w;
}
}  // namespace dbftc

// ------------------------------------------------------------------ host side

size_t dbf_tc_workspace_bytes(int64_t r, int64_t n, int64_t B) { return dbftc::ws_layout(B, r, n).total; }

template <bool HALF_OUT>
cudaError_t launch_sg_gemm(const SgParams& p, const void* bmat, int64_t bcols, cudaStream_t stream, int num_sms);
cudaError_t launch_sg_prep(const uint16_t* x, const uint16_t* bdiag, const uint16_t* mid, int64_t n, int64_t r,
                          int64_t B, __half* xs, float* cscale, float* dscale, float* dinv, cudaStream_t stream);

cudaError_t launch_dbf_tc(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                          const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B, float* y,
                          void* workspace, cudaStream_t stream, int num_sms) {
  using namespace dbftc;
  const Ws L = ws_layout(B, r, n);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  float* cs = reinterpret_cast<float*>(ws + L.cscale);
  float* ds = reinterpret_cast<float*>(ws + L.dscale);
  float* di = reinterpret_cast<float*>(ws + L.dinv);
  __half* xs = reinterpret_cast<__half*>(ws + L.xs);
  __half* hs = reinterpret_cast<__half*>(ws + L.hs);
  cudaError_t err = launch_sg_prep(x, b, mid, n, r, B, xs, cs, ds, di, stream);
  if (err != cudaSuccess) return err;
  SgParams p1 = {};
  p1.signs = B2;
  p1.rdiag = mid;
  p1.s1 = cs;
  p1.s2 = ds;
  p1.out_h = hs;
  p1.M = static_cast<int>(B);
  p1.rows = static_cast<int>(r);
  p1.K = static_cast<int>(n);
  err = launch_sg_gemm<true>(p1, xs, n, stream, num_sms);
  if (err != cudaSuccess) return err;
  // phase 2 undoes the intermediate's scale: s1 = 2^-d
  SgParams p2 = {};
  p2.signs = B1;
  p2.rdiag = a;
  p2.s1 = di;
  p2.out_f = y;
  p2.M = static_cast<int>(B);
  p2.rows = static_cast<int>(m);
  p2.K = static_cast<int>(r);
  return launch_sg_gemm<false>(p2, hs, r, stream, num_sms);
}

}  // namespace w1

// w1_pack: fp32 weights -> sign words + fp16 group scales (mean |w|, exact RNE).
//
// Sign convention bit = IEEE sign bit (0 -> +1, 1 -> -1): "LLM binarization
// episode 01: DBF", section 1.  One fp16 scale per 128 weights: "Banyan ...",
// Abstract (1.125 bits per weight).
//
// One warp per group of 128 weights.  Lane l reads column 32*i + l for
// i = 0..3, so __ballot_sync of the sign bits yields the LSB-first words
// directly.  The group sum of |w| is formed in fp64; if an interval around it
// (a rigorous bound on the fp64 summation error) rounds to a single fp16
// value, that value is the exact answer.  Otherwise (a result within ~2^-45 of
// an fp16 rounding midpoint, or of the overflow threshold) one lane recomputes
// the sum exactly in 192-bit fixed point and rounds it to fp16 by hand.
#include <cstdint>

#include "w1_common.cuh"

namespace w1 {

__device__ __forceinline__ uint16_t f64_to_f16_rn(double v) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return h;
}

// Exact sum of |w| over the group, as a 192-bit integer in units of 2^-149,
// then RNE to fp16 of (sum / 128).  Only reached when every |w| < 2^23 (larger
// values make the result +inf without ambiguity).
__device__ uint16_t exact_scale_fp16(const float* __restrict__ wg) {
  uint64_t acc[3] = {0, 0, 0};
  for (int i = 0; i < 128; ++i) {
    uint32_t b = __float_as_uint(wg[i]) & 0x7FFFFFFFu;
    uint32_t ex = b >> 23;
    uint64_t man = b & 0x7FFFFFu;
    uint32_t sh = 0;
    if (ex != 0) {
      man |= 0x800000u;
      sh = ex - 1;  // value * 2^149 = man << (ex - 1)
    }
    // add man << sh into the 3-limb accumulator (sh <= 171 here)
    uint64_t part[3] = {0, 0, 0};
    uint32_t limb = sh >> 6, off = sh & 63;
    part[limb] = man << off;
    if (off != 0 && limb + 1 < 3) part[limb + 1] = man >> (64 - off);
    uint64_t c = 0;
    for (int j = 0; j < 3; ++j) {
      uint64_t s = acc[j] + part[j];
      uint64_t c1 = s < acc[j];
      uint64_t s2 = s + c;
      uint64_t c2 = s2 < s;
      acc[j] = s2;
      c = c1 | c2;
    }
  }
  // T = acc * 2^-156.  Position of the leading one.
  int p = -1;
  for (int j = 2; j >= 0; --j) {
    if (acc[j] != 0) {
      p = 64 * j + 63 - __clzll(static_cast<long long>(acc[j]));
      break;
    }
  }
  if (p < 0) return 0;
  int e = p - 156;           // floor(log2 T)
  if (e < -14) e = -14;      // subnormal range shares the quantum 2^-24
  int q = e - 10;            // quantum exponent
  int qb = q + 156;          // quantum bit position in acc (>= 132)
  // n = acc >> qb ; rem = acc & (2^qb - 1)
  uint64_t n = 0;
  {
    int limb = qb >> 6, off = qb & 63;
    n = acc[limb] >> off;
    if (off != 0 && limb + 1 < 3) n |= acc[limb + 1] << (64 - off);
  }
  // compare remainder with half = 2^(qb-1)
  int hb = qb - 1;
  int hl = hb >> 6, ho = hb & 63;
  bool half_bit = (acc[hl] >> ho) & 1ull;
  bool below_nonzero = false;
  {
    uint64_t mask = (ho == 0) ? 0ull : ((1ull << ho) - 1ull);
    if (acc[hl] & mask) below_nonzero = true;
    for (int j = 0; j < hl; ++j)
      if (acc[j]) below_nonzero = true;
  }
  if (half_bit && (below_nonzero || (n & 1ull))) n += 1;
  // bits = ((q + 24) << 10) + n covers subnormals, normals and the carry
  int64_t bits = (static_cast<int64_t>(q + 24) << 10) + static_cast<int64_t>(n);
  if (bits >= 0x7C00) return 0x7C00;
  return static_cast<uint16_t>(bits);
}

__global__ void __launch_bounds__(256) pack_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                                   uint32_t* __restrict__ signs,
                                                   uint16_t* __restrict__ scales) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t groups_per_row = K >> 7;
  const int64_t total = N * groups_per_row;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t gi = warp0; gi < total; gi += nwarps) {
    const int64_t n = gi / groups_per_row;
    const int64_t g = gi - n * groups_per_row;
    const float* wg = W + n * K + (g << 7);
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __ldcs(wg + 32 * i + lane);
    uint32_t words[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) words[i] = __ballot_sync(0xFFFFFFFFu, __float_as_uint(v[i]) >> 31);
    bool finite = true;
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      finite &= isfinite(v[i]);
      s += static_cast<double>(fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    finite = __all_sync(0xFFFFFFFFu, finite);
    if (lane == 0) {
      uint4 wv = make_uint4(words[0], words[1], words[2], words[3]);
      *reinterpret_cast<uint4*>(signs + n * (K >> 5) + (g << 2)) = wv;
    }
    uint16_t h;
    if (!finite) {
      h = f64_to_f16_rn(s * 0.0078125);
      if (lane == 0) set_status(W1_ERR_NONFINITE);
    } else {
      // s carries relative error < 8 * 2^-53 (nonnegative terms, depth-8 tree);
      // the interval [t(1-2^-44), t(1+2^-44)] contains the exact mean.
      const double t = s * 0.0078125;
      const uint16_t lo = f64_to_f16_rn(t * (1.0 - 0x1p-44));
      const uint16_t hi = f64_to_f16_rn(t * (1.0 + 0x1p-44));
      h = lo;
      if (lo != hi) {
        // rare: resolve exactly (values are < 2^23 here, else lo == hi == inf)
        if (lane == 0) h = exact_scale_fp16(wg);
        h = __shfl_sync(0xFFFFFFFFu, h, 0);
      }
      if (h == 0x7C00 && lane == 0) set_status(W1_ERR_RANGE);
    }
    if (lane == 0) scales[n * groups_per_row + g] = h;
  }
  pdl_launch_dependents();
}

cudaError_t launch_pack(const float* W, int64_t N, int64_t K, uint32_t* signs, uint16_t* scales,
                        cudaStream_t stream, int num_sms) {
  const int64_t groups = N * (K >> 7);
  const int threads = 256;
  int64_t blocks = (groups + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pack_kernel, W, N, K, signs, scales);
}

}  // namespace w1

// Host side of the libw1 C ABI: argument validation, device capability
// checks, the device status word and kernel launches.  See include/w1.h.
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "w1_common.cuh"

namespace w1 {



cudaError_t launch_pack(const float* W, int64_t N, int64_t K, uint32_t* signs, uint16_t* scales,
                        cudaStream_t stream, int num_sms);
cudaError_t launch_gemv(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                        const void* x, bool xf, int B, float* y, cudaStream_t stream, int num_sms,
                        int smem_cap, bool static_weights);
bool okt_shape_ok(int64_t n1, int64_t n2, int64_t K);
size_t measure_workspace_bytes(int64_t m, int64_t n);
cudaError_t launch_residual_g128(const float* W, int64_t N, int64_t K, const uint32_t* signs, const uint16_t* scales,
                                 float* E, double* sums, void* workspace, cudaStream_t stream, int num_sms);
cudaError_t launch_dbf_residual(const float* W, const uint16_t* a, const uint32_t* B1, const uint16_t* mid,
                                const uint32_t* B2, const uint16_t* b, int64_t m, int64_t r, int64_t n, float* E,
                                double* sums, void* workspace, cudaStream_t stream, int num_sms);
size_t dbf_residual_workspace_bytes(int64_t m, int64_t r, int64_t n);
cudaError_t launch_power_iteration(const float* A, int64_t m, int64_t n, const float* v0, int64_t iters,
                                   double* sigma, void* workspace, cudaStream_t stream, int num_sms);
cudaError_t launch_okt_rotate(const float* H, int n1, const float* R, int n2, const uint16_t* x, int B, float* out,
                              bool early, cudaStream_t stream, int num_sms, int smem_optin);
cudaError_t launch_gemm(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
                        const uint16_t* x, int64_t M, float* y, void* workspace, cudaStream_t stream,
                        int num_sms);
size_t gemm_workspace_bytes(int64_t M, int64_t K);

cudaError_t launch_dbf(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                       const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B,
                       float* y, void* workspace, cudaStream_t stream, int num_sms, int smem_cap,
                       bool allow_tensor_path);
size_t dbf_workspace_bytes(int64_t m, int64_t r, int64_t n, int64_t B);
cudaError_t launch_stream_probe(const void* a, int64_t abytes, const void* b, int64_t bbytes, int ctas, bool early,
                                uint32_t* out, cudaStream_t stream);
bool reproject_shape_ok(int64_t m, int64_t r, int64_t n);
size_t reproject_workspace_bytes(int64_t m, int64_t r, int64_t n);
cudaError_t launch_reproject_mid(const float* W, const uint16_t* a, const uint32_t* B1, const uint32_t* B2,
                                 const uint16_t* b, int64_t m, int64_t r, int64_t n, int max_iter, double tol,
                                 uint16_t* mid, double* mid64, int* info, void* workspace, cudaStream_t stream,
                                 int num_sms);

struct DeviceInfo {
  bool ok = false;
  bool valid = false;
  int sms = 0;
  int smem_optin = 0;
};

static constexpr int kMaxDevices = 64;
static DeviceInfo g_info[kMaxDevices];
static std::mutex g_info_mu;

// Current device's capabilities; W1_OK only on sm_100 class parts.
static int device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W1_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_info_mu);
  DeviceInfo& d = g_info[dev];
  if (!d.valid) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return W1_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    d.valid = true;
  }
  *out = d;
  return d.ok ? W1_OK : W1_ERR_UNSUPPORTED;
}

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static inline int launch_result(cudaError_t e) {
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    return W1_ERR_UNSUPPORTED;
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? W1_OK : W1_ERR_CUDA;
}

}  // namespace w1

using namespace w1;

extern "C" {

const char* w1_status_string(int status) {
  switch (status) {
    case W1_OK: return "W1_OK";
    case W1_ERR_NULL: return "W1_ERR_NULL: null pointer";
    case W1_ERR_SHAPE: return "W1_ERR_SHAPE: invalid dimension";
    case W1_ERR_ALIGN: return "W1_ERR_ALIGN: pointer not 16-byte aligned";
    case W1_ERR_NONFINITE: return "W1_ERR_NONFINITE: NaN/Inf in input";
    case W1_ERR_RANGE: return "W1_ERR_RANGE: scale overflowed fp16";
    case W1_ERR_CUDA: return "W1_ERR_CUDA: CUDA error";
    case W1_ERR_TIMEOUT: return "W1_ERR_TIMEOUT: bounded device wait gave up";
    case W1_ERR_WORKSPACE: return "W1_ERR_WORKSPACE: workspace missing or too small";
    case W1_ERR_UNSUPPORTED: return "W1_ERR_UNSUPPORTED: device is not sm_100, or no kernel plan fits these sizes";
    case W1_ERR_TOO_LARGE: return "W1_ERR_TOO_LARGE: sizes exceed the static scratch of dbf_apply_noalloc";
    case W1_ERR_NOT_CONVERGED: return "W1_ERR_NOT_CONVERGED: the iterative solve stopped at its iteration limit";
    default: return "unknown w1 status";
  }
}

int w1_sync_status(w1_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return W1_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return W1_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return W1_ERR_CUDA;
  return static_cast<int>(v);
}

int w1_set_knob(const char* name, const char* value) {
  if (!name) return W1_ERR_NULL;
  for (int i = 0; i < kKnobCount; ++i) {
    if (strcmp(name, knob_spec(i).name) != 0) continue;
    KnobTable& t = knob_table();
    int v = t.env[i];
    if (value && *value && !parse_knob(i, value, &v)) return W1_ERR_SHAPE;
    t.v[i].store(v, std::memory_order_relaxed);
    return W1_OK;
  }
  return W1_ERR_SHAPE;
}

int w1_pack(const float* W, int64_t N, int64_t K, uint32_t* signs, uint16_t* scales,
            w1_stream_t stream) {
  if (!W || !signs || !scales) return W1_ERR_NULL;
  if (N <= 0 || K <= 0 || (K % 128) != 0) return W1_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(signs) || !aligned16(scales)) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_pack(W, N, K, signs, scales, reinterpret_cast<cudaStream_t>(stream), d.sms));
}

int w1_gemv_ex(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
               const uint16_t* x, int64_t B, float* y, uint32_t flags, w1_stream_t stream) {
  if (!signs || !scales || !x || !y) return W1_ERR_NULL;
  if (N <= 0 || K <= 0 || (K % 128) != 0 || B < 1 || B > 8) return W1_ERR_SHAPE;
  if (K / 128 > (int64_t)1 << 20 || N > ((int64_t)1 << 40)) return W1_ERR_SHAPE;
  if ((flags & ~static_cast<uint32_t>(W1_GEMV_STATIC_WEIGHTS)) != 0) return W1_ERR_SHAPE;
  if (!aligned16(signs) || !aligned16(scales) || !aligned16(x) || !aligned16(y)) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  const int cap = d.smem_optin < 110 * 1024 ? d.smem_optin : 110 * 1024;
  return launch_result(launch_gemv(signs, scales, N, K, x, false, static_cast<int>(B), y,
                                   reinterpret_cast<cudaStream_t>(stream), d.sms, cap,
                                   (flags & W1_GEMV_STATIC_WEIGHTS) != 0));
}

int w1_gemv(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
            const uint16_t* x, int64_t B, float* y, w1_stream_t stream) {
  return w1_gemv_ex(signs, scales, N, K, x, B, y, 0u, stream);
}

size_t w1_measure_workspace_size(int64_t m, int64_t n) {
  if (m <= 0 || n <= 0 || m > ((int64_t)1 << 31) - 1 || n > ((int64_t)1 << 31) - 1) return 0;
  return measure_workspace_bytes(m, n);
}

static inline bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

int w1_residual(const float* W, int64_t N, int64_t K, const uint32_t* signs, const uint16_t* scales, float* E,
                double* sums, void* workspace, size_t ws_bytes, w1_stream_t stream) {
  if (!W || !signs || !scales || !sums) return W1_ERR_NULL;
  if (N <= 0 || K <= 0 || (K % 128) != 0 || N > ((int64_t)1 << 31) - 1 || K > ((int64_t)1 << 30))
    return W1_ERR_SHAPE;
  if (!workspace || ws_bytes < measure_workspace_bytes(N, K)) return W1_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(signs) || !aligned16(scales) || (E && !aligned16(E)) || !aligned16(workspace) ||
      !aligned8(sums))
    return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_residual_g128(W, N, K, signs, scales, E, sums, workspace,
                                            reinterpret_cast<cudaStream_t>(stream), d.sms));
}

int w1_stream_probe(const void* a, int64_t abytes, const void* b, int64_t bbytes, int64_t ctas, uint32_t flags,
                    uint32_t* out, w1_stream_t stream) {
  if (!a || !out || (bbytes > 0 && !b)) return W1_ERR_NULL;
  if (abytes <= 0 || bbytes < 0 || (abytes % 16) != 0 || (bbytes % 16) != 0 || ctas < 1 || ctas > 65535 ||
      (flags & ~1u) != 0)
    return W1_ERR_SHAPE;
  if (!aligned16(a) || (bbytes > 0 && !aligned16(b)) || !aligned16(out)) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_stream_probe(a, abytes, b, bbytes, static_cast<int>(ctas), (flags & 1u) != 0, out,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

size_t dbf_reproject_mid_workspace_size(int64_t m, int64_t r, int64_t n) { return reproject_workspace_bytes(m, r, n); }

int dbf_reproject_mid(const float* W, const uint16_t* a, const uint32_t* B1, const uint32_t* B2, const uint16_t* b,
                      int64_t m, int64_t r, int64_t n, int64_t max_iter, double tol, uint16_t* mid, double* mid64,
                      int* info, void* workspace, size_t ws_bytes, w1_stream_t stream) {
  if (!W || !a || !B1 || !B2 || !b || !mid) return W1_ERR_NULL;
  if (!reproject_shape_ok(m, r, n) || max_iter < 0 || max_iter > (int64_t(1) << 30) || !(tol >= 0.0)) return W1_ERR_SHAPE;
  if (!workspace || ws_bytes < reproject_workspace_bytes(m, r, n)) return W1_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(a) || !aligned16(B1) || !aligned16(B2) || !aligned16(b) || !aligned16(mid) ||
      (mid64 && !aligned16(mid64)) || (info && !aligned8(info)) || !aligned16(workspace))
    return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_reproject_mid(W, a, B1, B2, b, m, r, n, static_cast<int>(max_iter), tol, mid, mid64,
                                            info, workspace, reinterpret_cast<cudaStream_t>(stream), d.sms));
}

int dbf_residual(const float* W, const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                 const uint16_t* b, int64_t m, int64_t r, int64_t n, float* E, double* sums, void* workspace,
                 size_t ws_bytes, w1_stream_t stream) {
  if (!W || !a || !B1 || !mid || !B2 || !b || !sums) return W1_ERR_NULL;
  if (m <= 0 || r <= 0 || n <= 0 || (m % 128) != 0 || (r % 128) != 0 || (n % 128) != 0) return W1_ERR_SHAPE;
  if ((m / 128) * (n / 128) > 8192 || r > ((int64_t)1 << 24)) return W1_ERR_SHAPE;
  if (!workspace || ws_bytes < dbf_residual_workspace_bytes(m, r, n)) return W1_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(a) || !aligned16(B1) || !aligned16(mid) || !aligned16(B2) || !aligned16(b) ||
      (E && !aligned16(E)) || !aligned16(workspace) || !aligned8(sums))
    return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_dbf_residual(W, a, B1, mid, B2, b, m, r, n, E, sums, workspace,
                                           reinterpret_cast<cudaStream_t>(stream), d.sms));
}

size_t dbf_residual_workspace_size(int64_t m, int64_t r, int64_t n) {
  if (m <= 0 || r <= 0 || n <= 0 || (m % 128) != 0 || (r % 128) != 0 || (n % 128) != 0) return 0;
  return dbf_residual_workspace_bytes(m, r, n);
}

int w1_power_iteration(const float* A, int64_t m, int64_t n, const float* v0, int64_t iters, double* sigma,
                       void* workspace, size_t ws_bytes, w1_stream_t stream) {
  if (!A || !v0 || !sigma) return W1_ERR_NULL;
  if (m <= 0 || n <= 0 || (n % 4) != 0 || m > ((int64_t)1 << 31) - 1 || n > ((int64_t)1 << 28) || iters < 0 ||
      iters > 100000)
    return W1_ERR_SHAPE;
  if (!workspace || ws_bytes < measure_workspace_bytes(m, n)) return W1_ERR_WORKSPACE;
  if (!aligned16(A) || !aligned16(v0) || !aligned16(workspace) || !aligned8(sigma)) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_power_iteration(A, m, n, v0, iters, sigma, workspace,
                                              reinterpret_cast<cudaStream_t>(stream), d.sms));
}

int w1_okt_rotate(const float* H, int64_t n1, const float* R, int64_t n2, const uint16_t* x, int64_t B,
                  float* x_rot, w1_stream_t stream) {
  if (!H || !R || !x || !x_rot) return W1_ERR_NULL;
  if (B < 1 || B > 65535 || n1 < 1 || n2 < 1 || n1 > 1024 || n2 > 128) return W1_ERR_SHAPE;
  if (!okt_shape_ok(n1, n2, n1 * n2) || ((n1 * n2) % 128) != 0) return W1_ERR_SHAPE;
  if (!aligned16(H) || !aligned16(R) || !aligned16(x) || !aligned16(x_rot)) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_okt_rotate(H, static_cast<int>(n1), R, static_cast<int>(n2), x, static_cast<int>(B),
                                         x_rot, false, reinterpret_cast<cudaStream_t>(stream), d.sms,
                                         d.smem_optin));
}

int w1_okt_gemv(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K, const float* H, int64_t n1,
                const float* R, int64_t n2, const uint16_t* x, int64_t B, float* x_rot, float* y, uint32_t flags,
                w1_stream_t stream) {
  if (!signs || !scales || !H || !R || !x || !x_rot || !y) return W1_ERR_NULL;
  if (N <= 0 || K <= 0 || (K % 128) != 0 || B < 1 || B > 8) return W1_ERR_SHAPE;
  if (N > ((int64_t)1 << 30) || n1 < 1 || n2 < 1 || n1 > 1024 || n2 > 128 || !okt_shape_ok(n1, n2, K))
    return W1_ERR_SHAPE;
  if ((flags & ~static_cast<uint32_t>(W1_GEMV_STATIC_WEIGHTS)) != 0) return W1_ERR_SHAPE;
  if (!aligned16(signs) || !aligned16(scales) || !aligned16(H) || !aligned16(R) || !aligned16(x) ||
      !aligned16(x_rot) || !aligned16(y))
    return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  const bool static_weights = (flags & W1_GEMV_STATIC_WEIGHTS) != 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = launch_result(launch_okt_rotate(H, static_cast<int>(n1), R, static_cast<int>(n2), x, static_cast<int>(B),
                                       x_rot, static_weights, s, d.sms, d.smem_optin));
  if (st != W1_OK) return st;
  const int cap = d.smem_optin < 110 * 1024 ? d.smem_optin : 110 * 1024;
  return launch_result(launch_gemv(signs, scales, N, K, x_rot, true, static_cast<int>(B), y, s, d.sms, cap,
                                   static_weights));
}

int w1_gemm(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
            const uint16_t* x, int64_t M, float* y, void* workspace, size_t ws_bytes,
            w1_stream_t stream) {
  if (!signs || !scales || !x || !y) return W1_ERR_NULL;
  if (N <= 0 || K <= 0 || M <= 0 || (K % 128) != 0) return W1_ERR_SHAPE;
  if (M > (int64_t)1 << 31 || N > (int64_t)1 << 31) return W1_ERR_SHAPE;
  if (!aligned16(signs) || !aligned16(scales) || !aligned16(x) || !aligned16(y)) return W1_ERR_ALIGN;
  if (!workspace || ws_bytes < gemm_workspace_bytes(M, K)) return W1_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  return launch_result(launch_gemm(signs, scales, N, K, x, M, y, workspace,
                                   reinterpret_cast<cudaStream_t>(stream), d.sms));
}

size_t w1_gemm_workspace_size(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0 || (K % 128) != 0 || M > (int64_t)1 << 31) return 0;
  return gemm_workspace_bytes(M, K);
}

size_t dbf_workspace_size(int64_t m, int64_t r, int64_t n, int64_t B) {
  if (m <= 0 || r <= 0 || n <= 0 || B <= 0) return 0;
  return dbf_workspace_bytes(m, r, n, B);
}

int dbf_apply(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
              const uint16_t* b, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B, float* y,
              void* workspace, size_t ws_bytes, w1_stream_t stream) {
  if (!a || !B1 || !mid || !B2 || !b || !x || !y) return W1_ERR_NULL;
  if (m <= 0 || r <= 0 || n <= 0 || B <= 0 || (r % 128) != 0 || (n % 128) != 0) return W1_ERR_SHAPE;
  if (m > (int64_t)1 << 30 || r > (int64_t)1 << 30 || n > (int64_t)1 << 30) return W1_ERR_SHAPE;
  if (!aligned16(a) || !aligned16(B1) || !aligned16(mid) || !aligned16(B2) || !aligned16(b) || !aligned16(x) ||
      !aligned16(y))
    return W1_ERR_ALIGN;
  if (!workspace || ws_bytes < dbf_workspace_bytes(m, r, n, B)) return W1_ERR_WORKSPACE;
  if (!aligned16(workspace)) return W1_ERR_ALIGN;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != W1_OK) return st;
  const int cap = d.smem_optin < 200 * 1024 ? d.smem_optin : 200 * 1024;
  return launch_result(launch_dbf(a, B1, mid, B2, b, m, r, n, x, B, y, workspace,
                                  reinterpret_cast<cudaStream_t>(stream), d.sms, cap, true));
}

}  // extern "C"

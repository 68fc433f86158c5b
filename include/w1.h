/*
 * w1.h -- C ABI of libw1: matrix products against 1-bit weights on B200 (sm_100a).
 *
 * Storage format.  A weight matrix W (N rows = outputs, K columns = inputs)
 * is stored as one sign bit per weight plus one fp16 scale per group of 128
 * consecutive weights along K: 1 + 16/128 = 1.125 bits per weight
 * ("Banyan: Converting Pretrained Language Models to 1-Bit Weights ...",
 * Abstract; "Behaviour-Relearned Quantization", step 02 "Binarize experts").
 * Bit 0 means +1 and bit 1 means -1, the IEEE sign-bit convention ("LLM
 * binarization episode 01: DBF", section 1 "The representation").  The
 * dequantised weight is w_hat[n,k] = s[n, k/128] * (1 - 2*bit[n,k]).
 *
 * Layouts (canonical, row-major, no padding):
 *   signs   uint32 [N][K/32]   bit j of word t is column k = 32*t + j (LSB first);
 *                              little-endian bytes equal a uint64 LSB-first block
 *                              of 64 signs (the SIGN1 block, DBF post section 3).
 *   scales  fp16   [N][K/128]  passed as uint16_t bit patterns.
 *   x       bf16   [B][K]      activations, uint16_t bit patterns.
 *   y       fp32   [B][N]      y[b,n] = sum_k w_hat[n,k] * x[b,k].
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory, frees nothing and keeps no state except one
 *     status word per device.  Inputs and outputs must not alias.
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream) of the CURRENT device; the call returns without synchronising.
 *   - Argument errors are detected on the host and returned synchronously with
 *     nothing launched.  A failed launch returns W1_ERR_CUDA.  Conditions found
 *     on the device (non-finite or out-of-range data, a bounded wait that gave
 *     up) are recorded in the device status word; read them with
 *     w1_sync_status().
 *   - Pointers must be 16-byte aligned; K (and every contracted dimension) must
 *     be a positive multiple of 128.
 *   - Kernels use programmatic dependent launch: they may start while the
 *     previous kernel in the stream finishes, but touch no data before it has
 *     completed (only L2 prefetches of their own weight bytes are issued early).
 */
#ifndef W1_H_
#define W1_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* w1_stream_t;

typedef enum {
  W1_OK = 0,
  W1_ERR_NULL = 1,        /* a required pointer is NULL                         */
  W1_ERR_SHAPE = 2,       /* dimension <= 0, not a multiple of 128, batch range  */
  W1_ERR_ALIGN = 3,       /* pointer not 16-byte aligned                         */
  W1_ERR_NONFINITE = 4,   /* device: NaN/Inf in pack input                       */
  W1_ERR_RANGE = 5,       /* device: a group scale overflowed fp16 (stored +inf) */
  W1_ERR_CUDA = 6,        /* CUDA launch / runtime error                         */
  W1_ERR_TIMEOUT = 7,     /* device: a bounded wait gave up                      */
  W1_ERR_WORKSPACE = 8,   /* workspace missing or too small                      */
  W1_ERR_UNSUPPORTED = 9, /* device is not sm_100 (B200 class), or no kernel plan fits the sizes */
  W1_ERR_TOO_LARGE = 10,  /* sizes exceed dbf_apply_noalloc's static scratch     */
  W1_ERR_NOT_CONVERGED = 11 /* device: an iterative solve hit its iteration limit */
} w1_status;

/* Static, human-readable name of a status code. */
const char* w1_status_string(int status);

/* Synchronises `stream`, then returns and clears the current device's status
 * word (W1_OK if no kernel recorded an error).  Returns W1_ERR_CUDA if the
 * synchronisation itself failed. */
int w1_sync_status(w1_stream_t stream);

/* Process-wide testing and tuning knobs (no counterpart on the pages).  Each
 * starts from its W1_* environment variable, read once on first use; no call
 * reads the environment after that.  `value` NULL or "" restores the value
 * the environment gave.  Host-side only and not synchronised with calls in
 * flight on other host threads.
 *   "gemv_path"     "direct" | "direct16" | "tc" | "ring" | "flat" forces one GEMV kernel (W1_GEMV_PATH)
 *   "gemv_split"    1 | 2 | 4 | 8: forced K split of the split-capable GEMV kernels (W1_GEMV_SPLIT)
 *   "gemv_autotune" "0": the static kernel rule instead of first-call timing (W1_GEMV_AUTOTUNE)
 *   "moe_path"      "tiles" | "decode" | "grouped" forces a routed-MoE path (W1_MOE_PATH)
 *   "dbf_path"      "fused" | "twostep" forces a small-batch DBF chain form (W1_DBF_PATH)
 *   "dbf_warps"     8 | 16 warps per CTA of the small-batch DBF chain (W1_DBF_WARPS)
 *   "dbf_rank_split" 1..8 CTAs per cluster splitting r in the two-launch chain's U . h (W1_DBF_RANK_SPLIT)
 *   "dbf_core"      "flat" | "direct": the two-launch chain's GEMV core (W1_DBF_CORE)
 *   "sg_bm"         128 | 256 forces the sign GEMM's token tile (W1_SG_BM)
 *   "sg_exp"        4 | 8 forces the sign GEMM's expander warps per CTA (W1_SG_EXP)
 *   "sg_a"          "smem" | "tmem": where the sign GEMM's 128-token tiles keep the weight operand (W1_SG_A)
 *   "moe_tw"        2 | 4: 8-row n-tiles per warp in the decode MoE's per-route gate/up (W1_MOE_TW)
 *   "verbose"       nonzero prints plans and choices on stderr (W1_VERBOSE)
 * Returns W1_ERR_NULL for a NULL name, W1_ERR_SHAPE for an unknown name or
 * value. */
int w1_set_knob(const char* name, const char* value);

/*
 * w1_pack -- binarise W along K ("Behaviour-Relearned Quantization", step 02;
 * sign convention: DBF post, section 1).
 *   W       fp32 [N][K], device, read only.
 *   signs   uint32 [N][K/32] out: bit = IEEE sign bit of W (so -0.0 -> 1).
 *   scales  fp16 [N][K/128] out: RNE_fp16( sum_{k in group} |W| / 128 ), the sum
 *           taken exactly (the mean |w| is the least-squares scale for sign
 *           codes; the pages name "signs plus scales" without a formula).
 * Device-detected: NaN/Inf in W -> W1_ERR_NONFINITE (that group's scale is
 * NaN/Inf); a finite group whose scale rounds past fp16 -> W1_ERR_RANGE (+inf).
 */
int w1_pack(const float* W, int64_t N, int64_t K, uint32_t* signs, uint16_t* scales,
            w1_stream_t stream);

/*
 * w1_gemv -- decode-regime product, one vector per batch row ("LLM binarization
 * episode 01: DBF", section 4: generation applies each matrix to one vector at
 * a time; section 5: sign selection and addition).
 *   y[b][n] = sum_g s[n][g] * sum_{k in g} (1 - 2*bit[n][k]) * x[b][k],  1 <= B <= 8.
 *   signs [N][K/32], scales [N][K/128], x bf16 [B][K], y fp32 [B][N] (all device).
 * Accuracy: |y - y_exact| <= 1e-3 * sum_k |s x_k| per element (fp32
 * accumulation; the int8 kernels take x as 24-bit fixed point per 128-group,
 * the bf16 ones multiply x unchanged by +-1).
 * Kernel choice: the first call for a new (N, K, B) on a device, when `stream`
 * is not being captured, times the candidate kernels and K splits on `stream`
 * with the caller's buffers and keeps the fastest; that call blocks the host
 * until the timing finishes (about a millisecond).  Later calls, and calls
 * during stream capture, launch without synchronising.  Results of different
 * candidates differ only in fp32 summation order; a shape's choice is fixed
 * once made, so repeated calls are bitwise reproducible.
 */
int w1_gemv(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
            const uint16_t* x, int64_t B, float* y, w1_stream_t stream);

/* Flags for w1_gemv_ex. */
enum { W1_GEMV_STATIC_WEIGHTS = 1 };

/*
 * w1_gemv_ex -- w1_gemv with flags (0 gives w1_gemv exactly).  The pages have
 * no counterpart: this is a scheduling contract, not new arithmetic.
 * W1_GEMV_STATIC_WEIGHTS: the caller promises that `signs` and `scales` were
 * written before the kernel that precedes this call on `stream` began (weights
 * loaded once, used by many decode steps).  The kernel may then start reading
 * them while that kernel is still running (programmatic dependent launch),
 * which hides most of its load latency in a chain of back-to-back products.
 * Without the promise (or with weights written by the preceding kernel, e.g.
 * w1_pack immediately before) the flag can return stale weights: leave it 0.
 * x and y are always ordered after the preceding kernel.  Other flag bits:
 * W1_ERR_SHAPE.
 */
int w1_gemv_ex(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
               const uint16_t* x, int64_t B, float* y, uint32_t flags, w1_stream_t stream);

/*
 * w1_gemv_choice -- inspection: writes the kernel and K split that w1_gemv /
 * w1_gemv_ex has chosen for (N, K, B, flags) on the current device, as
 * "direct/<split>" (8 warps per CTA), "direct16/<split>" (16 warps),
 * "tc/<split>" or "ring/<split>" (split 0: the kernel's own planner), or ""
 * when no call has chosen yet.  Host only, no GPU work.
 */
int w1_gemv_choice(int64_t N, int64_t K, int64_t B, uint32_t flags, char* out, size_t out_len);

/*
 * w1_gemv_set_choice -- pins the kernel for (N, K, B, flags) on the current
 * device, in the same notation as w1_gemv_choice ("direct/1", "direct16/2",
 * "tc/0", "ring/0"; direct splits 1, 2, 4, 8), replacing any earlier choice:
 * later calls for that shape skip the first-call timing and use it.  For
 * persisting a tuning across processes, or for profiling runs whose timing
 * would choose differently.  A pinned kernel whose plan does not fit the
 * shape fails its calls with W1_ERR_UNSUPPORTED.  Unknown name or invalid
 * sizes: W1_ERR_SHAPE; null name: W1_ERR_NULL.  Host only, no GPU work.
 */
int w1_gemv_set_choice(int64_t N, int64_t K, int64_t B, uint32_t flags, const char* name);

/*
 * w1_okt_rotate -- rotated activations for weights binarised in rotated
 * coordinates (zhichai.net post on BWLA, section 3 "OKT": one orthogonal
 * rotation factored as a Kronecker product H kron R of two small orthogonal
 * matrices, n1 n2 = K; section 5: the activations take the same rotation, so
 * the product is unchanged).
 *   x_rot[b] = (H kron R)^T x[b].  With x[b][i*n2 + j] read as X[i][j]
 *   (n1 x n2, row-major), x_rot[b] viewed the same way is H^T X R.
 *   H fp32 [n1][n1], R fp32 [n2][n2] (row-major; orthogonality is the
 *   caller's, nothing checks it), x bf16 [B][K], x_rot fp32 [B][K] (device).
 * Limits: n1 * n2 = K, K a multiple of 128 and <= 65536, 1 <= n1 <= 1024,
 * 1 <= n2 <= 128, 1 <= B <= 65535; otherwise W1_ERR_SHAPE.  A shape whose
 * staging exceeds the device's shared memory returns W1_ERR_UNSUPPORTED.
 * Accuracy: each element is two fp32 dot products in a fixed order (over
 * n1, then n2), so |x_rot - exact| <= (n1 + n2 + 2) * 2^-24 *
 * (|H|^T |X| |R|)[i][j]; results are bitwise reproducible.
 */
int w1_okt_rotate(const float* H, int64_t n1, const float* R, int64_t n2, const uint16_t* x, int64_t B,
                  float* x_rot, w1_stream_t stream);

/*
 * w1_okt_gemv -- decode product against weights stored in rotated
 * coordinates: w1_okt_rotate, then the 1-bit product on the fp32 x_rot.
 *   y[b][n] = sum_g s[n][g] * sum_{k in g} (1 - 2*bit[n][k]) * x_rot[b][k],
 *   where signs/scales are w1_pack of W (H kron R), so y = W x up to the
 *   binarisation.  1 <= B <= 8; the limits of w1_okt_rotate apply, with K
 *   the weights' K.
 *   x_rot: caller-owned fp32 [B][K] scratch; it receives the rotated
 *   activations.  It must not alias x or y.
 * flags: W1_GEMV_STATIC_WEIGHTS as for w1_gemv_ex.  The promise then also
 * covers H and R, which the rotation may read before the preceding kernel
 * completes.  Two kernels: the product launches while the rotation runs and
 * stages its weights; it reads x_rot only after the rotation has finished.
 * The product picks its kernel (the direct kernel, whose fp32 activation
 * path this uses) by first-call timing, like w1_gemv.
 * Accuracy: |y - y_exact| <= 1e-3 * sum_k |s x_rot_k| per element, plus the
 * rotation's error carried through the product.
 */
int w1_okt_gemv(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K, const float* H, int64_t n1,
                const float* R, int64_t n2, const uint16_t* x, int64_t B, float* x_rot, float* y, uint32_t flags,
                w1_stream_t stream);

/*
 * Approximation residuals ("LLM binarization episode 01: DBF", section 8
 * "Current measurements": the relative Frobenius residual ||E||_F / ||W||_F
 * and the relative spectral residual ||E||_2 / ||W||_2 of E = W - W_approx,
 * each matrix normalised by its own norm, spectral norms by fixed-seed
 * 32-iteration power iteration).  Measurement calls, not part of a product.
 * Every sum below has a fixed order (a per-CTA tree, then the CTAs in index
 * order), so results are bitwise reproducible for a shape on a device.
 *
 * w1_measure_workspace_size -- bytes of device workspace that w1_residual
 * and w1_power_iteration need for an m x n matrix (0 for invalid sizes); one
 * workspace serves both, one call at a time per stream.  dbf_residual needs
 * dbf_residual_workspace_size (larger).
 */
size_t w1_measure_workspace_size(int64_t m, int64_t n);

/*
 * w1_residual -- E = W - w_hat for a matrix and its group-128 sign code
 * (w_hat as in w1_gemv), and sums[0] = sum E^2, sums[1] = sum W^2.
 *   W fp32 [N][K]; signs [N][K/32], scales [N][K/128] (device, read only).
 *   E fp32 [N][K] out (each element w - w_hat rounded once to fp32), or NULL.
 *   sums: device double[2] out; each square is taken of the fp32 values in
 *   fp64.
 *   workspace: device, >= w1_measure_workspace_size(N, K) bytes, else
 *   W1_ERR_WORKSPACE.
 */
int w1_residual(const float* W, int64_t N, int64_t K, const uint32_t* signs, const uint16_t* scales, float* E,
                double* sums, void* workspace, size_t ws_bytes, w1_stream_t stream);

/*
 * dbf_residual -- the same for a DBF matrix W_approx = diag(a) U diag(mid)
 * V diag(b) (dbf_apply's operands; m, r, n multiples of 128 and
 * (m/128)(n/128) <= 8192, else W1_ERR_SHAPE).
 *   W_approx[i][j] = (acc_ij * a_i) * b_j in fp32, where acc_ij is the sum
 *   over k of U_ik * (mid_k V_kj) with fp32 accumulation (tensor cores: the
 *   products are exact in fp16); so
 *   |W_approx - exact| <= (r + 2) * 2^-24 * |a_i| |b_j| sum_k |mid_k|.
 *   E fp32 [m][n] out (or NULL), sums as for w1_residual.
 *   workspace: device, >= dbf_residual_workspace_size(m, r, n) bytes (it
 *   holds mid (.) V^T in fp16 and W_approx^T in fp32: about 2 n r + 4 n m),
 *   else W1_ERR_WORKSPACE.
 */
size_t dbf_residual_workspace_size(int64_t m, int64_t r, int64_t n);
int dbf_residual(const float* W, const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                 const uint16_t* b, int64_t m, int64_t r, int64_t n, float* E, double* sums, void* workspace,
                 size_t ws_bytes, w1_stream_t stream);

/*
 * w1_stream_probe -- the per-launch floor of a decode product (a measurement
 * aid; the pages have no counterpart).  Reads the byte ranges [a, a + abytes)
 * and [b, b + bbytes) once with 16-byte loads spread over `ctas` CTAs, every
 * load of a thread issued before any is used, and adds one word per CTA into
 * out[cta] (so the loads cannot be dropped; the values mean nothing).  Timed
 * as back-to-back launches over a product's sign words and scales, it is the
 * memory work of that product and nothing else.
 *   flags: 1 = issue the loads before the programmatic-dependent-launch wait
 *   (the analogue of W1_GEMV_STATIC_WEIGHTS), 0 = after it.
 *   abytes > 0, bbytes >= 0, both multiples of 16; 1 <= ctas <= 65535; else
 *   W1_ERR_SHAPE.  a, b (if bbytes > 0) and out (uint32 [ctas]) 16-byte
 *   aligned, else W1_ERR_ALIGN.
 */
int w1_stream_probe(const void* a, int64_t abytes, const void* b, int64_t bbytes, int64_t ctas, uint32_t flags,
                    uint32_t* out, w1_stream_t stream);

/*
 * dbf_reproject_mid -- least-squares refit of the DBF middle diagonal ("LLM
 * binarization episode 01: DBF", section 1.2 "What we inherit from DBF": one
 * final linear least-squares reprojection of the middle diagonal, the signs
 * and the outer scalers held fixed).  With P_k = (a * U[:, k]) (V[k, :] * b)^T
 * (U, V the +-1 matrices of B1, B2; a, b as in dbf_apply), the minimiser of
 * ||W - sum_k mid_k P_k||_F solves G mid = c with
 *   G_kl = (U^T diag(a^2) U)_kl (V diag(b^2) V^T)_kl,  c_k = <W, P_k>.
 * G and c are formed in fp64 (G exactly while the partial sums of the a^2 and
 * b^2 terms span under 2^53: for fp16 diagonals in [0.01, 0.3] and m, n <=
 * 65536, always); the system is solved by conjugate gradients in fp64 from
 * mid = 0, which for a singular G converges to the minimum-norm solution
 * (what least squares gives).  Model-conversion work, not per-token work.
 *   W fp32 [m][n]; a fp16 [m]; B1 [m][r/32]; B2 [r][n/32]; b fp16 [n]
 *     (device, read only).  1 <= m <= 2^24; r, n multiples of 128;
 *     r <= 16384; n <= 2^24; else W1_ERR_SHAPE.
 *   max_iter: iteration limit (0 <= max_iter <= 2^30); tol: stop when
 *     ||c - G mid||_2 <= tol ||c||_2 (tol >= 0; 1e-13 is enough for fp16
 *     output).  Reaching max_iter first records W1_ERR_NOT_CONVERGED in the
 *     device status word and keeps the last iterate.
 *   mid: fp16 [r] out, the solution rounded once to nearest-even (an
 *     overflow to inf records W1_ERR_RANGE).  mid64: fp64 [r] out, or NULL.
 *   info: device int[2] out, or NULL: iterations taken, converged (1) or not.
 *   workspace: device, >= dbf_reproject_mid_workspace_size(m, r, n) bytes
 *     (8 r^2 for G plus O(m r / 16 + n r / 8)), 16-byte aligned.
 * Every sum has a fixed order: results are bitwise reproducible for a shape
 * on a device.  Uses a cooperative launch (one CTA per SM at most).
 */
size_t dbf_reproject_mid_workspace_size(int64_t m, int64_t r, int64_t n);
int dbf_reproject_mid(const float* W, const uint16_t* a, const uint32_t* B1, const uint32_t* B2, const uint16_t* b,
                      int64_t m, int64_t r, int64_t n, int64_t max_iter, double tol, uint16_t* mid, double* mid64,
                      int* info, void* workspace, size_t ws_bytes, w1_stream_t stream);

/*
 * w1_power_iteration -- spectral norm estimate of A (fp32 [m][n], n a
 * multiple of 4) by power iteration on A^T A from the start vector v0 (fp32
 * [n]; the fixed-seed draw is the caller's):
 *   v = v0 / ||v0||; `iters` times: u = A v, w = A^T u, v = w / ||w||;
 *   *sigma = ||A v|| (device double).  A zero vector along the way gives 0.
 * All vectors and sums are fp64; A is read as given.  The relative spectral
 * residual is this on E (from w1_residual / dbf_residual) divided by this
 * on W.
 */
int w1_power_iteration(const float* A, int64_t m, int64_t n, const float* v0, int64_t iters, double* sigma,
                       void* workspace, size_t ws_bytes, w1_stream_t stream);

/*
 * w1_gemm -- prefill-regime product for many token rows (DBF post, section 4:
 * prompt processing amortises weight loads across columns).
 *   y[m][n] = sum_g s[n][g] * sum_{k in g} (1 - 2*bit[n][k]) * x[m][k].
 *   signs [N][K/32], scales [N][K/128], x bf16 [M][K], y fp32 [M][N] (device).
 * tcgen05 tensor cores.  x is first rewritten to fp16 with an exact
 * power-of-two per token row (max |x| in [2^14, 2^15)); the weight operand is
 * the group scale with the weight's sign bit (+-s, exact in fp16), so the
 * blockwise scale is applied inside the MMA and all of K accumulates in one
 * fp32 TMEM tile.  Same accuracy bound as w1_gemv.
 * workspace: >= w1_gemm_workspace_size(M, K) bytes of device memory, 256-byte
 *   aligned (the fp16 copy of x and the token scales); contents on entry are
 *   ignored, nothing is carried between calls; calls sharing a workspace must
 *   not overlap.  Too small / null: W1_ERR_WORKSPACE; misaligned: W1_ERR_ALIGN.
 * Two kernels on `stream` (prep, GEMM).
 */
int w1_gemm(const uint32_t* signs, const uint16_t* scales, int64_t N, int64_t K,
            const uint16_t* x, int64_t M, float* y, void* workspace, size_t ws_bytes,
            w1_stream_t stream);

/* Bytes of workspace w1_gemm needs (0 for invalid sizes). */
size_t w1_gemm_workspace_size(int64_t M, int64_t K);

/*
 * w1_moe_grouped -- routed SwiGLU expert layer with 1-bit group-128 experts
 * ("LLM binarization episode 01: DBF", section 4: every (token, slot) route
 * carries an expert id and a route weight; gate/up consume the token's shared
 * hidden state, down consumes the route's own intermediate).
 *   p[t] = softmax(router_logits[t]) over the E experts (fp32); the top_k
 *   experts by probability (ties to the lower index) are the routes, each with
 *   weight p (no renormalisation).  For route (t, e):
 *     g = G_e x_t, u = U_e x_t, h = bf16( silu(g) * u ), out[t] += p * D_e h,
 *   the slot terms summed in slot order.  silu(z) = z / (1 + exp(-z)).
 *   x              bf16 [T][H]
 *   router_logits  fp32 [T][E]
 *   gate_*, up_*   experts stacked: signs uint32 [E][I][H/32], scales fp16 [E][I][H/128]
 *   down_*         signs uint32 [E][H][I/32], scales fp16 [E][H][I/128]
 *   out            fp32 [T][H]
 *   H, I multiples of 128; 1 <= top_k <= min(E, 32); E <= 256.
 * workspace: >= w1_moe_workspace_size(...) bytes, 1024-byte aligned; holds the
 *   routing (expert ids, weights, the expert-sorted route order), the tile
 *   lists, h (bf16, expert-sorted), the weighted route outputs, and the fp16
 *   copies of x rows and h rows in sorted route order with one power-of-two
 *   scale per route.  No state is carried between calls.  Calls sharing a
 *   workspace must not overlap.
 * T > 16: seven kernels on `stream`: router, counting sort, gather of x rows
 * into sorted order (fp16, exact per-token power of two), grouped gate/up GEMM
 * (tcgen05, +-s fp16 weight operand, fused SwiGLU), h to fp16 per route,
 * grouped down GEMM (route weight applied), slot-ordered combine.
 * T <= 16 (decode regime): per-route gate/up products with fused SwiGLU (up
 * to 4 tokens each CTA routes its token; above, a router kernel runs first),
 * then per-token down products over the token's slots with the slot-ordered
 * combine fused; the products are the batch-1 steps of w1_gemv.
 * Deterministic.  Accuracy per stage as w1_gemm: 1e-3 * sum|s x| for g, u and
 * D_e h.  The workspace must be 1024-byte aligned (W1_ERR_ALIGN otherwise).
 */
int w1_moe_grouped(const uint16_t* x, const float* router_logits, int64_t T, int64_t H, int64_t I, int64_t E,
                   int64_t top_k, const uint32_t* gate_signs, const uint16_t* gate_scales,
                   const uint32_t* up_signs, const uint16_t* up_scales, const uint32_t* down_signs,
                   const uint16_t* down_scales, float* out, void* workspace, size_t ws_bytes,
                   w1_stream_t stream);

/* Bytes of workspace w1_moe_grouped needs (0 for invalid sizes). */
size_t w1_moe_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int64_t top_k);

/*
 * dbf_apply -- Double Binary Factorization chain ("LLM binarization episode 01:
 * DBF", section 1 "The representation": W ~ D_out U D_mid V D_in; section 4:
 * evaluated as x_scaled = D_in x, h = V x_scaled, h_scaled = D_mid h,
 * y_core = U h_scaled, y = D_out y_core -- the chain, not a rebuilt dense W).
 *   y[b][i] = a[i] * sum_j U[i][j] * mid[j] * sum_k V[j][k] * bdiag[k] * x[b][k]
 *   a     fp16 [m]          D_out
 *   B1    uint32 [m][r/32]  U, sign bits (bit 0 -> +1, bit 1 -> -1), LSB first
 *   mid   fp16 [r]          D_mid
 *   B2    uint32 [r][n/32]  V
 *   bdiag fp16 [n]          D_in
 *   x     bf16 [B][n], y fp32 [B][m]; r and n multiples of 128.  No group scales.
 * workspace: device buffer of at least dbf_workspace_size(m, r, n, B) bytes,
 *   16-byte aligned.  Its first 4 bytes are the arrival count of a grid
 *   barrier: ZERO them before the first call; every call leaves the count at
 *   zero again (after a W1_ERR_TIMEOUT the caller must re-zero it).  After a call
 *   it holds h_scaled (fp32 [min(B,8)][r], byte offset 256) of the last group
 *   of up to 8 batch rows.  Calls sharing a workspace must not overlap.
 * Below 64 rows the batch runs in groups of up to 8 rows: a group of 1-4 rows
 * as two products (V then U, h_scaled through the workspace; U's K split
 * over r is the pages' "split rank", section 5 item 5), a group of 5-8 rows
 * as one kernel with a grid-wide barrier between the two products (section
 * 7; two products when that kernel has no co-resident plan).  From 64 rows on, two tensor-core sign GEMMs.  Accuracy:
 * |y - y_exact| <= 1e-3 * |a_i| * sum_j |mid_j h_j| per element.
 */
int dbf_apply(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
              const uint16_t* bdiag, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B,
              float* y, void* workspace, size_t ws_bytes, w1_stream_t stream);

/* Bytes of workspace dbf_apply needs for these sizes (0 for invalid sizes). */
size_t dbf_workspace_size(int64_t m, int64_t r, int64_t n, int64_t B);

/*
 * dbf_apply_noalloc -- dbf_apply for callers that cannot allocate device memory
 * (the pages have no counterpart: this is a deployment variant).  Some callers
 * cannot call cudaMalloc or take memory from an allocator: code embedded in a
 * host framework whose device memory is owned by that framework's pool, or a
 * latency-critical decode loop where an allocation would synchronise the
 * device or fail.  This entry point takes the same inputs and output as
 * dbf_apply but no workspace: its scratch is a fixed array inside the library
 * (256 bytes + 4*8*16384 bytes, held on every GPU that loads the library until
 * the process exits).  It allocates nothing and calls no allocating routine.
 *   Limit: r <= 16384, else W1_ERR_TOO_LARGE (other limits as dbf_apply).
 *   Every batch size runs the small-batch chain, in groups of up to 8 rows
 *   one after another: unlike dbf_apply it never takes the tensor-core path
 *   (that path needs a workspace that grows with B), so from B = 64 up it
 *   costs about ceil(B/8) times a group of 8 (64 launches at B = 512).
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.
 *   Every call shares the one array and clears its barrier count first; calls
 *   that overlap on the GPU (for instance on two streams) race on it.  After a
 *   call the array still holds that call's fp32 intermediate.
 */
int dbf_apply_noalloc(const uint16_t* a, const uint32_t* B1, const uint16_t* mid, const uint32_t* B2,
                      const uint16_t* bdiag, int64_t m, int64_t r, int64_t n, const uint16_t* x, int64_t B,
                      float* y, w1_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* W1_H_ */

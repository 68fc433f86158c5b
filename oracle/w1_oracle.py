"""Plain, slow CPU oracle for 1-bit group-128 matrix products.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  The library (``pack_sign_g128_b200``) never imports it, and this
module imports nothing from the library: the two share no code.  Inputs come
in as plain numpy arrays (bf16 / fp16 values as their uint16 bit patterns).

Everything is computed from the definitions, in float64 or in exact integer /
rational arithmetic:

* Storage format -- one sign bit per weight plus one 16-bit scale for each
  group of 128 consecutive weights, 1 + 16/128 = 1.125 bits per weight
  ("Behaviour-Relearned Quantization", step 02 "Binarize experts"; "Banyan:
  Converting Pretrained Language Models to 1-Bit Weights ...", Abstract).
* Sign convention -- bit 0 means +1 and bit 1 means -1, the IEEE sign-bit
  convention ("LLM binarization episode 01: DBF", section 1 "The
  representation").
* Scale -- mean |w| over the group, rounded once (round-to-nearest-even) to
  fp16.  The pages name "signs plus scales" but give no scale rule; mean |w|
  is the closed-form least-squares scale for sign codes (the plainest reading,
  pinned by brute force in the tests).
* Product -- multiplying by a binary weight selects x or -x (DBF post,
  section 1), so y[b, n] = sum_g s[n, g] * sum_{k in g} (1 - 2 bit[n, k]) x[b, k].
* DBF chain -- x_scaled = D_in x, h = V x_scaled, h_scaled = D_mid h,
  y_core = U h_scaled, y = D_out y_core, evaluated in that order (DBF post,
  section 4 "Teaching the model loader DBDBD").
* Bit budget -- bpe = [r(m+n) + 16(m+n+r)] / (mn) (DBF post, section 1.1).
* Routed MoE -- every (token, slot) route carries an expert id and a route
  weight; gate/up consume the token's shared hidden state, down consumes the
  route's own intermediate (DBF post, section 4, MoE input topologies).
* Approximation residuals -- E = W - W_approx; the relative Frobenius
  residual ||E||_F / ||W||_F and the relative spectral residual
  ||E||_2 / ||W||_2, spectral norms by power iteration (DBF post, section 8
  "Current measurements").
* Rotated activations -- one orthogonal rotation of the input space, factored
  as the Kronecker product of two small orthogonal matrices H and R; the
  weights are binarised in the rotated coordinates and the activations take
  the same rotation, so the product is unchanged (zhichai.net post on BWLA,
  section 3 "OKT" and section 5).

Readings where the pages are silent are listed in the repository's design
notes: scale rule mean|w|; fp16 scale; LSB-first bit order inside uint32
words (bit j of word t is k = 32 t + j); signbit semantics for +-0; softmax
over all experts, top-k by probability with ties to the lower index, no
renormalisation; SiLU(z) = z / (1 + exp(-z)).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

GROUP = 128

# ---------------------------------------------------------------------------
# Exact conversions of the 16-bit input formats (widening only, no rounding).
# ---------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def fp16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns (uint16) -> exact float64 values."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# Exact round-to-nearest-even of a non-negative rational to IEEE binary16.
# ---------------------------------------------------------------------------

_FP16_MAX = Fraction(65504)
_FP16_OVERFLOW = Fraction(65520)  # RNE threshold: 65504 + half of its 32 ulp


def _floor_log2(q: Fraction) -> int:
    """Largest e with 2**e <= q, for q > 0 (exact)."""
    e = q.numerator.bit_length() - q.denominator.bit_length()
    # bit lengths bound the ratio to within a factor of two; settle exactly
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    return e


def round_to_fp16_bits(q: Fraction) -> int:
    """IEEE binary16 bits of RNE(q) for a non-negative rational q.

    binary16: 11-bit significand, exponent range [-14, 15], subnormal quantum
    2**-24; values >= 65520 round to +inf.
    """
    if q < 0:
        raise ValueError("negative input")
    if q == 0:
        return 0
    if q >= _FP16_OVERFLOW:
        return 0x7C00
    e = max(_floor_log2(q), -14)
    quantum = Fraction(2) ** (e - 10)
    n = q / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    value = fl * quantum
    if value > _FP16_MAX:
        return 0x7C00
    # value is exactly representable in binary16 and in float64
    return int(np.array([float(value)], dtype=np.float64).astype(np.float16).view(np.uint16)[0])


# ---------------------------------------------------------------------------
# Pack (binarise): signs and group scales.
# ---------------------------------------------------------------------------


def _fp32_abs_scaled_ints(vals: np.ndarray) -> list[int]:
    """|v| * 2**149 as exact Python integers for float32 v (finite)."""
    bits = np.asarray(vals, dtype=np.float32).view(np.uint32) & np.uint32(0x7FFFFFFF)
    out = []
    for b in bits.tolist():
        ex = b >> 23
        man = b & 0x7FFFFF
        if ex == 0:          # subnormal: man * 2**-149
            out.append(man)
        else:                # normal: (man | 2**23) * 2**(ex - 150)
            out.append((man | 0x800000) << (ex - 1))
    return out


def group_scale_bits(vals: np.ndarray) -> int:
    """fp16 bits of RNE( sum|v| / len(v) ), the sum taken exactly."""
    vals = np.asarray(vals, dtype=np.float32)
    if not np.all(np.isfinite(vals)):
        raise ValueError("non-finite weight")
    total = sum(_fp32_abs_scaled_ints(vals))
    return round_to_fp16_bits(Fraction(total, (1 << 149) * len(vals)))


def sign_bits_ref(W: np.ndarray) -> np.ndarray:
    """bit = 1 exactly where the IEEE sign bit of the fp32 weight is set."""
    W = np.asarray(W, dtype=np.float32)
    return ((W.view(np.uint32) >> np.uint32(31)) & np.uint32(1)).astype(np.uint8)


def pack_bits_lsb_first(bits: np.ndarray) -> np.ndarray:
    """[N, K] 0/1 -> uint32 [N, K/32]; bit j of word t is column 32 t + j."""
    N, K = bits.shape
    assert K % 32 == 0
    b = bits.reshape(N, K // 32, 32).astype(np.uint64)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (b * weights).sum(axis=2).astype(np.uint32)


def unpack_bits_lsb_first(words: np.ndarray, K: int) -> np.ndarray:
    """uint32 [N, K/32] -> [N, K] 0/1 (inverse of pack_bits_lsb_first)."""
    w = np.asarray(words, dtype=np.uint32)
    N = w.shape[0]
    j = np.arange(32, dtype=np.uint32)
    bits = (w[:, :, None] >> j[None, None, :]) & np.uint32(1)
    return bits.reshape(N, K).astype(np.uint8)


def pack_ref(W: np.ndarray, group: int = GROUP):
    """Binarise fp32 W [N, K] (out x in) along K.

    Returns (signs uint32 [N, K/32], scales uint16 fp16-bits [N, K/group]).
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    if K % group or K % 32:
        raise ValueError("K must be a multiple of the group size and of 32")
    signs = pack_bits_lsb_first(sign_bits_ref(W))
    G = K // group
    scales = np.empty((N, G), dtype=np.uint16)
    for n in range(N):
        for g in range(G):
            scales[n, g] = group_scale_bits(W[n, g * group:(g + 1) * group])
    return signs, scales


def pack_scales_sampled(W: np.ndarray, rows, groups, group: int = GROUP) -> np.ndarray:
    """Scales for selected (row, group) pairs only (for full-size samples)."""
    W = np.asarray(W, dtype=np.float32)
    return np.array([group_scale_bits(W[n, g * group:(g + 1) * group])
                     for n, g in zip(rows, groups)], dtype=np.uint16)


# ---------------------------------------------------------------------------
# Dequantised products (GEMV / GEMM) and their tolerance scale.
# ---------------------------------------------------------------------------


def dequant_ref(signs: np.ndarray, scale_bits: np.ndarray, K: int, group: int = GROUP) -> np.ndarray:
    """w_hat[n, k] = s[n, g(k)] * (1 - 2 bit[n, k]) in float64."""
    bits = unpack_bits_lsb_first(signs, K).astype(np.float64)
    s = fp16_bits_to_f64(scale_bits)
    s_full = np.repeat(s, group, axis=1)
    return s_full * (1.0 - 2.0 * bits)


def matmul_ref(x: np.ndarray, signs: np.ndarray, scale_bits: np.ndarray, K: int, group: int = GROUP):
    """y = x @ w_hat^T in float64, plus the per-element scale sum_k |s x_k|.

    x: float64 [B, K].  Returns (y [B, N], bound [B, N]).
    """
    w_hat = dequant_ref(signs, scale_bits, K, group)
    x = np.asarray(x, dtype=np.float64)
    y = x @ w_hat.T
    bound = np.abs(x) @ np.abs(w_hat).T
    return y, bound


# ---------------------------------------------------------------------------
# Bit accounting.
# ---------------------------------------------------------------------------


def sign_group_bits(N: int, K: int, group: int = GROUP, scale_bits: int = 16) -> int:
    """Storage bits of an N x K matrix: one sign per weight + one scale per group."""
    assert K % group == 0
    return N * K + scale_bits * N * (K // group)


def dbf_bits(m: int, n: int, r: int, diag_bits: int = 16) -> tuple[int, int, int]:
    """(binary-factor bits, diagonal bits, total) of a DBF m x n matrix at width r."""
    binary = r * n + m * r
    diag = diag_bits * (n + r + m)
    return binary, diag, binary + diag


def dbf_bits_per_element(m: int, n: int, r: int, diag_bits: int = 16) -> Fraction:
    return Fraction(dbf_bits(m, n, r, diag_bits)[2], m * n)


# ---------------------------------------------------------------------------
# DBF chain y = D_out U D_mid V D_in x.
# ---------------------------------------------------------------------------


def dbf_ref(a_bits, B1_words, mid_bits, B2_words, b_bits, x, m: int, r: int, n: int):
    """Evaluate the D-B-D-B-D chain right to left in float64.

    a: fp16 bits [m] (D_out); B1: uint32 [m, r/32] (U); mid: fp16 bits [r]
    (D_mid); B2: uint32 [r, n/32] (V); b: fp16 bits [n] (D_in); x: float64
    [B, n].  Signs follow bit 0 -> +1, bit 1 -> -1.

    Returns a dict with y [B, m], the stage values and two tolerance scales:
    ``bound`` = sum_j |a_i U_ij mid_j h_j| (second product fed the exact h) and
    ``h_bound`` = sum_k |V_jk b_k x_k| (first product).
    """
    a = fp16_bits_to_f64(a_bits)
    mid = fp16_bits_to_f64(mid_bits)
    b = fp16_bits_to_f64(b_bits)
    U = 1.0 - 2.0 * unpack_bits_lsb_first(B1_words, r).astype(np.float64)   # [m, r]
    V = 1.0 - 2.0 * unpack_bits_lsb_first(B2_words, n).astype(np.float64)   # [r, n]
    x = np.asarray(x, dtype=np.float64)
    x_scaled = x * b[None, :]
    h = x_scaled @ V.T
    h_scaled = h * mid[None, :]
    y_core = h_scaled @ U.T
    y = y_core * a[None, :]
    bound = np.abs(a)[None, :] * (np.abs(h_scaled) @ np.abs(U).T)
    h_bound = np.abs(x_scaled) @ np.abs(V).T
    return {"y": y, "h": h, "h_scaled": h_scaled, "bound": bound, "h_bound": h_bound,
            "U": U, "V": V}


def dbf_dense_ref(a_bits, B1_words, mid_bits, B2_words, b_bits, m: int, r: int, n: int) -> np.ndarray:
    """The reconstructed dense matrix diag(a) U diag(mid) V diag(b) [m, n]."""
    a = fp16_bits_to_f64(a_bits)
    mid = fp16_bits_to_f64(mid_bits)
    b = fp16_bits_to_f64(b_bits)
    U = 1.0 - 2.0 * unpack_bits_lsb_first(B1_words, r).astype(np.float64)
    V = 1.0 - 2.0 * unpack_bits_lsb_first(B2_words, n).astype(np.float64)
    return (a[:, None] * U) @ (mid[:, None] * (V * b[None, :]))


# ---------------------------------------------------------------------------
# Matrix-approximation measurement (DBF post, section 8 "Current
# measurements": relative Frobenius and spectral residuals, each matrix
# normalised by its own norm, spectral norms by fixed-seed 32-iteration power
# iteration).
# ---------------------------------------------------------------------------


def residual_g128_ref(W, signs, scale_bits) -> np.ndarray:
    """E = W - w_hat in float64 for a matrix and its 1-bit group-128 packing."""
    W = np.asarray(W, dtype=np.float64)
    return W - dequant_ref(signs, scale_bits, W.shape[1])


def dbf_residual_ref(W, a_bits, B1_words, mid_bits, B2_words, b_bits, m: int, r: int, n: int) -> np.ndarray:
    """E = W - diag(a) U diag(mid) V diag(b) in float64."""
    return np.asarray(W, dtype=np.float64) - dbf_dense_ref(a_bits, B1_words, mid_bits, B2_words, b_bits, m, r, n)


def dbf_reproject_mid_ref(W, a_bits, B1_words, B2_words, b_bits, m: int, r: int, n: int):
    """Least-squares middle diagonal for fixed signs and outer scalers.

    DBF post, section 1.2: one final linear least-squares reprojection of the
    middle diagonal, with U, V, a and b held fixed.  W_approx(mid) =
    sum_k mid_k P_k with P_k = (a * U[:, k]) (V[k, :] * b)^T is linear in mid, so
    the minimiser of ||W - W_approx(mid)||_F solves the normal equations
    G mid = c with G_kl = <P_k, P_l> = (U^T diag(a^2) U)_kl (V diag(b^2) V^T)_kl
    and c_k = <W, P_k> = (a * U[:, k])^T W (V[k, :] * b).  A singular G (more
    middle entries than independent P_k) takes the minimum-norm solution.

    Returns (mid float64 [r], fp16 bits [r] of RNE(mid)): the storage keeps
    the diagonals in fp16, so the stored diagonal is the rounded solution.
    """
    W = np.asarray(W, dtype=np.float64)
    a = fp16_bits_to_f64(a_bits)
    b = fp16_bits_to_f64(b_bits)
    U = 1.0 - 2.0 * unpack_bits_lsb_first(B1_words, r).astype(np.float64)   # [m, r]
    V = 1.0 - 2.0 * unpack_bits_lsb_first(B2_words, n).astype(np.float64)   # [r, n]
    Pu = a[:, None] * U           # columns p_k
    Qv = V * b[None, :]           # rows q_k
    G = (Pu.T @ Pu) * (Qv @ Qv.T)
    c = np.einsum("ik,ij,kj->k", Pu, W, Qv)
    # least squares on the normal equations (SVD, numpy's default cutoff):
    # G^-1 c for a nonsingular G, the minimum-norm solution for a singular
    # one -- an LU solve would return an arbitrary split between dependent
    # P_k whenever rounding hides an exact singularity from the pivoting
    mid = np.linalg.lstsq(G, c, rcond=None)[0]
    bits = np.array([round_to_fp16_bits(Fraction(abs(v))) | (0x8000 if v < 0 else 0) for v in mid], dtype=np.uint16)
    return mid, bits


def sum_squares_ref(A) -> float:
    """sum of A^2, exactly rounded once (math.fsum over float64 squares; the
    squares of float32 values are exact in float64)."""
    A = np.asarray(A, dtype=np.float64).ravel()
    return math.fsum((A * A).tolist())


def power_iteration_ref(A, v0, iters: int) -> float:
    """Spectral norm estimate of A [m, n] by power iteration on A^T A.

    v = v0 / ||v0||; then `iters` times: u = A v, w = A^T u, v = w / ||w||;
    the estimate is ||A v||.  If some w is zero (A v = 0), the estimate is 0.
    The section names the method, the iteration count and a fixed seed; the
    start vector is the caller's (drawn from the fixed seed), and this update
    order is the plainest reading.
    """
    A = np.asarray(A, dtype=np.float64)
    v = np.asarray(v0, dtype=np.float64).copy()
    nv = np.linalg.norm(v)
    if nv == 0.0:
        return 0.0
    v /= nv
    for _ in range(iters):
        w = A.T @ (A @ v)
        nw = np.linalg.norm(w)
        if nw == 0.0:
            return 0.0
        v = w / nw
    return float(np.linalg.norm(A @ v))


# ---------------------------------------------------------------------------
# Orthogonal-Kronecker rotation of the activations (zhichai.net post on BWLA,
# sections 3 and 5).
# ---------------------------------------------------------------------------


def okt_rotate_ref(H, R, x) -> np.ndarray:
    """Rotated activations x_rot = (H kron R)^T x for every batch row, float64.

    H: [n1, n1], R: [n2, n2] (any float dtype, taken exactly), x: [B, K] with
    K = n1 n2.  The post writes the rotation as H kron R with n1 n2 = K
    (section 3) and applies its transpose to the activations (section 5).  For
    y = W x with W [N, K] (outputs x inputs), the weights are stored as
    W (H kron R), and W (H kron R) (H kron R)^T x = W x.  Read x[b, i n2 + j]
    as X[i, j] (n1 x n2, row-major).  Then (A kron B) x is A X B^T, so
    (H kron R)^T x is H^T X R.
    """
    H = np.asarray(H, dtype=np.float64)
    R = np.asarray(R, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    n1, n2 = H.shape[0], R.shape[0]
    Bn, K = x.shape
    assert H.shape == (n1, n1) and R.shape == (n2, n2) and n1 * n2 == K
    out = np.empty((Bn, K), dtype=np.float64)
    for b in range(Bn):
        X = x[b].reshape(n1, n2)
        out[b] = (H.T @ X @ R).reshape(K)
    return out


def okt_gemv_ref(signs, scale_bits, H, R, x, K: int):
    """y = w_hat (H kron R)^T x: the packed weights (stored in the rotated
    coordinates) applied to the rotated activations, in float64.

    Returns (y [B, N], bound [B, N], x_rot [B, K]); bound is
    sum_k |s x_rot_k|, the scale of the product's error tolerance.
    """
    x_rot = okt_rotate_ref(H, R, x)
    y, bound = matmul_ref(x_rot, signs, scale_bits, K)
    return y, bound, x_rot


# ---------------------------------------------------------------------------
# Routed MoE FFN layer.
# ---------------------------------------------------------------------------


def softmax_ref(logits: np.ndarray) -> np.ndarray:
    """Row softmax in float64 (max-subtracted)."""
    z = np.asarray(logits, dtype=np.float64)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def topk_ref(p: np.ndarray, k: int):
    """Per row, the k largest entries; equal values go to the lower index.

    Returns (ids [T, k] int64 in descending-probability order, vals [T, k]).
    """
    T, E = p.shape
    ids = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-p[t, e], e))
        ids[t] = order[:k]
    vals = np.take_along_axis(p, ids, axis=1)
    return ids, vals


def silu_ref(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def moe_route_ref(logits: np.ndarray, top_k: int, renorm: bool = False):
    """Router: softmax over all experts, top-k, route weight = probability."""
    p = softmax_ref(logits)
    ids, w = topk_ref(p, top_k)
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return ids, w


def moe_ref(x, logits, gate, up, down, H: int, I: int, E: int, top_k: int,
            h_override=None, renorm: bool = False):
    """Routed SwiGLU expert layer in float64.

    x: float64 [T, H]; logits: float32/64 [T, E];
    gate, up: (signs [E, I, H/32], scales [E, I, H/128]);
    down: (signs [E, H, I/32], scales [E, H, I/128]).
    For every route (t, slot) with expert e = ids[t, slot] and weight p:
    g = G_e x_t, u = U_e x_t, h = silu(g) * u, out_t += p * D_e h, the slot
    terms added in slot order.  ``h_override`` [T, top_k, I] replaces h for
    the down stage (a stagewise check fed the device's own intermediate).

    Returns a dict with out [T, H], ids, w, g, u, h and tolerance scales.
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    ids, w = moe_route_ref(logits, top_k, renorm)
    g = np.zeros((T, top_k, I))
    u = np.zeros((T, top_k, I))
    g_bound = np.zeros((T, top_k, I))
    u_bound = np.zeros((T, top_k, I))
    for e in range(E):
        sel = np.argwhere(ids == e)
        if sel.size == 0:
            continue
        xs = x[sel[:, 0]]
        yg, bg = matmul_ref(xs, gate[0][e], gate[1][e], H)
        yu, bu = matmul_ref(xs, up[0][e], up[1][e], H)
        g[sel[:, 0], sel[:, 1]] = yg
        u[sel[:, 0], sel[:, 1]] = yu
        g_bound[sel[:, 0], sel[:, 1]] = bg
        u_bound[sel[:, 0], sel[:, 1]] = bu
    h = silu_ref(g) * u
    h_in = h if h_override is None else np.asarray(h_override, dtype=np.float64)
    d = np.zeros((T, top_k, H))
    d_bound = np.zeros((T, top_k, H))
    for e in range(E):
        sel = np.argwhere(ids == e)
        if sel.size == 0:
            continue
        yd, bd = matmul_ref(h_in[sel[:, 0], sel[:, 1]], down[0][e], down[1][e], I)
        d[sel[:, 0], sel[:, 1]] = yd
        d_bound[sel[:, 0], sel[:, 1]] = bd
    out = np.zeros((T, H))
    out_bound = np.zeros((T, H))
    for slot in range(top_k):
        out = out + w[:, slot:slot + 1] * d[:, slot]
        out_bound = out_bound + w[:, slot:slot + 1] * d_bound[:, slot]
    return {"out": out, "ids": ids, "w": w, "g": g, "u": u, "h": h,
            "g_bound": g_bound, "u_bound": u_bound, "d": d, "out_bound": out_bound}


def fsum_rows(a: np.ndarray) -> np.ndarray:
    """Correctly rounded row sums (used by tests for tight closed forms)."""
    return np.array([math.fsum(r) for r in np.asarray(a, dtype=np.float64)])


# ---------------------------------------------------------------------------
# Vectorised exact pack (same definition, for full-size test inputs).
# Pinned against pack_ref / group_scale_bits in the test suite.
# ---------------------------------------------------------------------------


def _bit_length_minus_one(S: np.ndarray) -> np.ndarray:
    """floor(log2 S) for positive int64 entries (0 where S == 0)."""
    L = np.zeros(S.shape, dtype=np.int64)
    s = S.copy()
    for k in (32, 16, 8, 4, 2, 1):
        m = (s >> k) > 0
        L += np.where(m, k, 0)
        s = np.where(m, s >> k, s)
    return L


def _round_scaled_int_to_fp16_bits(S: np.ndarray, p: np.ndarray) -> np.ndarray:
    """fp16 bits of RNE(S * 2**p) for int64 S >= 0 (exact integer rounding)."""
    S = S.astype(np.int64)
    p = p.astype(np.int64)
    L = _bit_length_minus_one(S)
    e = np.maximum(L + p, -14)          # exponent of the result's binade
    q = e - 10                          # quantum exponent
    qb = q - p                          # quantum position in units of S
    n = np.zeros_like(S)
    pos = qb > 0
    qbc = np.clip(qb, 1, 62)
    shifted = S >> qbc
    rem = S & ((np.int64(1) << qbc) - 1)
    half = np.int64(1) << (qbc - 1)
    up = (rem > half) | ((rem == half) & ((shifted & 1) == 1))
    big = qb >= 63                       # everything below half a quantum
    n = np.where(pos, np.where(big, 0, shifted + up.astype(np.int64)), S << np.clip(-qb, 0, 62))
    bits = ((q + 24) << 10) + n
    bits = np.where(bits >= 0x7C00, 0x7C00, bits)
    bits = np.where(S == 0, 0, bits)
    return bits.astype(np.uint16)


def pack_ref_fast(W: np.ndarray, group: int = GROUP):
    """Same result as pack_ref, computed with exact int64 sums per group.

    Each |w| = man * 2**(ex - 150) is aligned to 2**(ex_max - 31 - 150) of its
    group; a group holding a nonzero value below that alignment falls back to
    group_scale_bits (exact Python integers).  Rows are processed in blocks.
    """
    W = np.asarray(W, dtype=np.float32)
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    N, K = W.shape
    G = K // group
    signs = pack_bits_lsb_first(sign_bits_ref(W))
    scales = np.empty((N, G), dtype=np.uint16)
    lg = int(np.log2(group))
    for r0 in range(0, N, 256):
        Wb = W[r0:r0 + 256]
        nb = Wb.shape[0]
        b = (Wb.view(np.uint32) & np.uint32(0x7FFFFFFF)).reshape(nb, G, group)
        ex = (b >> np.uint32(23)).astype(np.int64)
        man = (b & np.uint32(0x7FFFFF)).astype(np.int64)
        man |= np.where(ex > 0, 0x800000, 0)
        np.maximum(ex, 1, out=ex)
        base = ex.max(axis=2, keepdims=True) - 31
        sh = ex - base
        ok = ((sh >= 0) | (man == 0)).all(axis=2)
        np.clip(sh, 0, 31, out=sh)
        S = np.left_shift(man, sh).sum(axis=2)
        sc = _round_scaled_int_to_fp16_bits(S, base[..., 0] - 150 - lg)
        for n, g in zip(*np.nonzero(~ok)):
            sc[n, g] = group_scale_bits(Wb[n, g * group:(g + 1) * group])
        scales[r0:r0 + nb] = sc
    return signs, scales

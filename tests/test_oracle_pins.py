"""Pins for the CPU oracle: what the pages and the mathematics fix.

None of these retypes an oracle formula.  Each checks the oracle against an
independent fact: a value the pages print, a closed form, a brute-force search,
a library routine for a special case, or an element-by-element loop.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special

from oracle import w1_oracle as O
from pack_sign_g128_b200 import synth


# ---------------------------------------------------------------- fp16 rounding

def _f16bits(v: float) -> int:
    return int(np.array([v], dtype=np.float64).astype(np.float16).view(np.uint16)[0])


def test_fp16_rounding_matches_library_conversion_off_midpoints():
    g = np.random.default_rng(11)
    vals = np.concatenate([
        np.abs(g.standard_normal(2000)) * 10.0 ** g.integers(-9, 5, 2000),
        np.abs(g.standard_normal(200)) * 1e-7,          # fp16 subnormal range
        [65503.9, 65519.0, 6.1035e-05, 5.96e-08, 1.0, 0.5],
    ])
    for v in vals:
        assert O.round_to_fp16_bits(Fraction(float(v))) == _f16bits(float(v)), v


def test_fp16_ties_go_to_even_and_overflow():
    one = Fraction(1)
    u = Fraction(1, 2 ** 10)                 # ulp of binary16 at 1.0
    assert O.round_to_fp16_bits(one + u / 2) == 0x3C00          # tie -> even (1.0)
    assert O.round_to_fp16_bits(one + 3 * u / 2) == 0x3C02      # tie -> even (1+2u)
    assert O.round_to_fp16_bits(one + u / 2 + Fraction(1, 2 ** 60)) == 0x3C01
    sub = Fraction(1, 2 ** 24)               # subnormal quantum
    assert O.round_to_fp16_bits(sub / 2) == 0x0000
    assert O.round_to_fp16_bits(3 * sub / 2) == 0x0002
    assert O.round_to_fp16_bits(Fraction(65519)) == 0x7BFF       # 65504
    assert O.round_to_fp16_bits(Fraction(65520)) == 0x7C00       # inf
    assert O.round_to_fp16_bits(Fraction(0)) == 0


# ---------------------------------------------------------------- scale rule

def _sq_err(w, alpha):
    w = np.asarray(w, dtype=np.float64)
    sgn = np.where(np.signbit(w), -1.0, 1.0)
    return float(np.sum((w - alpha * sgn) ** 2))


def test_scale_matches_brute_force_search_on_tiny_groups():
    """mean|w| is the least-squares scale for sign codes (brute-force search)."""
    g = np.random.default_rng(5)
    for group in (4, 8):
        for _ in range(20):
            w = (g.standard_normal(group) * 0.02).astype(np.float32)
            grid = np.linspace(0.0, float(np.max(np.abs(w))) * 1.5, 300001)
            sgn = np.where(np.signbit(w.astype(np.float64)), -1.0, 1.0)
            errs = ((w.astype(np.float64)[None, :] - grid[:, None] * sgn[None, :]) ** 2).sum(1)
            best = grid[int(np.argmin(errs))]
            s = float(np.array([O.group_scale_bits(w)], np.uint16).view(np.float16)[0])
            step = grid[1] - grid[0]
            half_ulp = 2.0 ** (math.floor(math.log2(best)) - 11)
            assert abs(s - best) <= step + half_ulp, (group, s, best)


def test_scale_is_the_best_fp16_value_for_each_group():
    g = synth.rng(7)
    W = synth.weights(g, 8, 512)
    _, scales = O.pack_ref(W)
    for n in range(8):
        for gi in range(4):
            w = W[n, gi * 128:(gi + 1) * 128]
            sb = int(scales[n, gi])
            s = float(np.array([sb], np.uint16).view(np.float16)[0])
            lo = float(np.array([sb - 1], np.uint16).view(np.float16)[0])
            hi = float(np.array([sb + 1], np.uint16).view(np.float16)[0])
            e = _sq_err(w, s)
            assert e <= _sq_err(w, lo) and e <= _sq_err(w, hi)


def test_flipping_any_sign_increases_error():
    g = synth.rng(8)
    W = synth.weights(g, 2, 128)
    signs, scales = O.pack_ref(W)
    w_hat = O.dequant_ref(signs, scales, 128)
    base = np.sum((W.astype(np.float64) - w_hat) ** 2, axis=1)
    for n in range(2):
        for k in range(128):
            alt = w_hat[n].copy()
            alt[k] = -alt[k]
            assert np.sum((W[n].astype(np.float64) - alt) ** 2) > base[n]


def test_scale_sum_is_exact_tiny_value_breaks_a_tie():
    """A sum that float64 would round onto an fp16 midpoint must still round
    from the exact value: 126*M + 2M + 2**-100 with M = 1 + 2**-11."""
    M = np.float32(1.0 + 2.0 ** -11)
    vals = np.array([M] * 126 + [np.float32(2.0) * M, np.float32(2.0 ** -100)], dtype=np.float32)
    assert math.fsum(np.abs(vals.astype(np.float64))) / 128 == float(M)   # fp64 lands on the tie
    assert O.group_scale_bits(vals) == 0x3C01                               # exact: just above it
    exact_tie = np.array([M] * 128, dtype=np.float32)
    assert O.group_scale_bits(exact_tie) == 0x3C00                          # true tie -> even


def test_scale_special_groups():
    assert O.group_scale_bits(np.zeros(128, np.float32)) == 0
    assert O.group_scale_bits(np.full(128, -0.0, np.float32)) == 0
    # all |w| = 2**-30: mean 2**-30 is below the fp16 subnormal quantum/2 -> 0
    assert O.group_scale_bits(np.full(128, 2.0 ** -30, np.float32)) == 0
    # mean |w| = 3 * 2**-25: subnormal tie between 2**-24 and 2**-23 -> even (2**-23)
    assert O.group_scale_bits(np.full(128, 3 * 2.0 ** -25, np.float32)) == 0x0002
    # overflow of the fp16 range
    assert O.group_scale_bits(np.full(128, 70000.0, np.float32)) == 0x7C00
    with pytest.raises(ValueError):
        O.group_scale_bits(np.array([np.nan] + [1.0] * 127, np.float32))


# ---------------------------------------------------------------- sign bits

def test_sign_convention_zero_is_plus_one():
    W = np.zeros((1, 128), np.float32)
    W[0, 1] = -0.0
    W[0, 2] = -1.5
    W[0, 3] = 2.0
    bits = O.sign_bits_ref(W)[0]
    assert bits[0] == 0 and bits[1] == 1 and bits[2] == 1 and bits[3] == 0
    signs, scales = O.pack_ref(W)
    w_hat = O.dequant_ref(signs, scales, 128)
    s = float(np.array([scales[0, 0]], np.uint16).view(np.float16)[0])
    assert w_hat[0, 0] == s and w_hat[0, 2] == -s and w_hat[0, 3] == s


def test_bit_order_lsb_first():
    bits = np.zeros((1, 64), np.uint8)
    bits[0, 0] = 1
    bits[0, 33] = 1
    bits[0, 63] = 1
    words = O.pack_bits_lsb_first(bits)
    assert words.tolist() == [[1, (1 << 1) | (1 << 31)]]
    # little-endian bytes of two LSB-first uint32 words == one LSB-first uint64 block
    u64 = int.from_bytes(words.astype('<u4').tobytes(), 'little')
    assert u64 == (1 << 0) | (1 << 33) | (1 << 63)


def test_pack_roundtrip():
    g = synth.rng(9)
    W = synth.weights(g, 16, 256)
    signs, _ = O.pack_ref(W)
    bits = O.unpack_bits_lsb_first(signs, 256)
    assert np.array_equal(bits.astype(bool), np.signbit(W))
    assert O.pack_bits_lsb_first(bits).tobytes() == signs.tobytes()


# ---------------------------------------------------------------- accounting

def test_bits_per_weight_is_1_125(golden_dir):
    with open(os.path.join(golden_dir, "format_accounting.json")) as f:
        gold = json.load(f)
    for N, K in [(512, 1024), (4096, 4096), (11008, 4096), (14336, 14336)]:
        assert Fraction(O.sign_group_bits(N, K), N * K) == Fraction(gold["bits_per_weight"])
    ratio = gold["parent_bits"] / gold["bits_per_weight"]
    assert round(ratio) == 14


def test_dbf_bit_budget_matches_page(golden_dir):
    with open(os.path.join(golden_dir, "dbf_bit_budget.json")) as f:
        gold = json.load(f)
    m, n, r = gold["m"], gold["n"], gold["r"]
    binary, diag, total = O.dbf_bits(m, n, r)
    assert binary == gold["binary_factor_bits"]
    assert diag == gold["fp16_diagonal_bits"]
    assert total == gold["total_bits"]
    assert O.dbf_bits_per_element(m, n, r) == Fraction(gold["bits_per_element"])
    q2k = int(Fraction(gold["q2k_bits_per_element"]) * m * n)
    assert q2k == gold["q2k_total_bits"]
    assert (q2k - total) // 8 == gold["dbf_smaller_by_bytes"]
    cnt = gold["routed_matrices"]
    bd = gold["routed_matrices_breakdown"]
    assert bd["layers"] * bd["experts"] * bd["projections"] == cnt
    gib = 8 * 2 ** 30
    assert round(total * cnt / gib, 4) == gold["dbf_total_gib"]
    assert round(q2k * cnt / gib, 4) == gold["q2k_total_gib"]
    assert round((q2k - total) * cnt / (8 * 2 ** 20)) == gold["margin_mib"]


# ---------------------------------------------------------------- products

def _scale_vals(scales):
    return scales.view(np.float16).astype(np.float64)


def test_product_all_positive_signs_is_group_sums():
    g = synth.rng(10)
    W = np.abs(synth.weights(g, 4, 384))
    x = synth.activations_bf16(g, 2, 384)
    signs, scales = O.pack_ref(W)
    assert not signs.any()
    xf = O.bf16_bits_to_f64(x)
    y, _ = O.matmul_ref(xf, signs, scales, 384)
    s = _scale_vals(scales)
    for b in range(2):
        for n in range(4):
            exp = sum(s[n, gi] * math.fsum(xf[b, gi * 128:(gi + 1) * 128]) for gi in range(3))
            assert y[b, n] == pytest.approx(exp, rel=1e-13, abs=1e-15)


def test_product_one_hot_reads_back_signed_scale():
    g = synth.rng(12)
    W = synth.weights(g, 6, 256)
    signs, scales = O.pack_ref(W)
    s = _scale_vals(scales)
    for k in (0, 1, 31, 32, 127, 128, 255):
        x = np.zeros((1, 256))
        x[0, k] = 1.0
        y, _ = O.matmul_ref(x, signs, scales, 256)
        for n in range(6):
            sgn = -1.0 if np.signbit(W[n, k]) else 1.0
            assert y[0, n] == sgn * s[n, k // 128]


def test_product_equals_dense_when_weights_are_already_binary():
    """W = +-c per group with fp16-exact c: the dequantised matrix is W itself."""
    g = np.random.default_rng(13)
    N, K = 5, 256
    c = np.array([0.015625, 0.0234375, 3.0, 0.5, 1.25, 0.0078125, 2.0, 0.375, 0.75, 1.5],
                 dtype=np.float32)[:N * 2].reshape(N, 2)
    sg = np.where(g.random((N, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    W = sg * np.repeat(c, 128, axis=1)
    signs, scales = O.pack_ref(W)
    x = O.bf16_bits_to_f64(synth.activations_bf16(synth.rng(1), 3, K))
    y, _ = O.matmul_ref(x, signs, scales, K)
    dense = x @ W.astype(np.float64).T
    assert np.allclose(y, dense, rtol=1e-14, atol=1e-14)


def test_product_integer_inputs_are_exact():
    g = np.random.default_rng(14)
    N, K = 7, 384
    c = (2.0 ** g.integers(-3, 3, size=(N, 3))).astype(np.float32)
    sg = np.where(g.random((N, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    W = sg * np.repeat(c, 128, axis=1)
    signs, scales = O.pack_ref(W)
    x = g.integers(-2, 3, size=(2, K)).astype(np.float64)
    y, _ = O.matmul_ref(x, signs, scales, K)
    for b in range(2):
        for n in range(N):
            exact = sum(Fraction(float(W[n, k])) * int(x[b, k]) for k in range(K))
            assert Fraction(y[b, n]) == exact


def test_tolerance_scale_is_abs_product_sum():
    g = synth.rng(15)
    W = synth.weights(g, 3, 256)
    x = O.bf16_bits_to_f64(synth.activations_bf16(g, 2, 256))
    signs, scales = O.pack_ref(W)
    _, bound = O.matmul_ref(x, signs, scales, 256)
    s = _scale_vals(scales)
    for b in range(2):
        for n in range(3):
            exp = math.fsum(abs(s[n, k // 128] * x[b, k]) for k in range(256))
            assert bound[b, n] == pytest.approx(exp, rel=1e-13)


# ---------------------------------------------------------------- DBF chain

def _sylvester(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def test_dbf_hadamard_closed_form():
    n = 256
    H = _sylvester(n)
    assert np.array_equal(H @ H, n * np.eye(n))
    words = O.pack_bits_lsb_first((H < 0).astype(np.uint8))
    ones = np.full(n, 0x3C00, np.uint16)
    x = O.bf16_bits_to_f64(synth.activations_bf16(synth.rng(3), 4, n))
    out = O.dbf_ref(ones, words, ones, words, ones, x, n, n, n)
    assert np.array_equal(out["y"], n * x)


def test_dbf_chain_matches_dense_reconstruction():
    a, B1, mid, B2, b, x = synth.dbf_case(m=96, r=160, n=128, B=3, seed=21)
    xf = O.bf16_bits_to_f64(x)
    out = O.dbf_ref(a, B1, mid, B2, b, xf, 96, 160, 128)
    dense = O.dbf_dense_ref(a, B1, mid, B2, b, 96, 160, 128)
    y2 = xf @ dense.T
    assert np.max(np.abs(out["y"] - y2)) <= 1e-12 * np.max(np.abs(y2))


def test_dbf_chain_elementwise_loop():
    """Explicit triple loop over the chain on a small case (independent of matmul)."""
    m, r, n = 32, 64, 32
    a, B1, mid, B2, b, x = synth.dbf_case(m=m, r=r, n=n, B=1, seed=22)
    xf = O.bf16_bits_to_f64(x)[0]
    out = O.dbf_ref(a, B1, mid, B2, b, xf[None, :], m, r, n)
    av, mv, bv = (np.array(v, np.uint16).view(np.float16).astype(float).tolist() for v in (a, mid, b))

    def bit(words, row, col):
        return (int(words[row, col // 32]) >> (col % 32)) & 1

    for i in range(m):
        acc = []
        for j in range(r):
            hj = math.fsum((1 - 2 * bit(B2, j, k)) * bv[k] * xf[k] for k in range(n))
            acc.append((1 - 2 * bit(B1, i, j)) * mv[j] * hj)
        yi = av[i] * math.fsum(acc)
        assert out["y"][0, i] == pytest.approx(yi, rel=1e-12, abs=1e-14)


# ---------------------------------------------------------------- MoE

def test_softmax_matches_library():
    g = np.random.default_rng(30)
    logits = g.standard_normal((20, 64)).astype(np.float32)
    assert np.allclose(O.softmax_ref(logits), scipy.special.softmax(logits.astype(np.float64), axis=1),
                       rtol=1e-14, atol=1e-16)


def test_topk_order_and_ties():
    p = np.array([[0.1, 0.3, 0.3, 0.05, 0.25]])
    ids, vals = O.topk_ref(p, 3)
    assert ids.tolist() == [[1, 2, 4]]
    assert vals.tolist() == [[0.3, 0.3, 0.25]]
    ids, w = O.moe_route_ref(np.zeros((2, 8), np.float32), 8)
    assert ids.tolist() == [list(range(8))] * 2
    assert np.allclose(w, 1.0 / 8)


def _tiny_moe(T=3, H=128, I=128, E=4, seed=31):
    x, logits, gate, up, down = synth.moe_case(T=T, H=H, I=I, E=E, seed=seed)
    pk = lambda A: tuple(np.stack(v) for v in zip(*[O.pack_ref(A[e]) for e in range(E)]))
    return O.bf16_bits_to_f64(x), logits, pk(gate), pk(up), pk(down)


def test_moe_elementwise_loop():
    T, H, I, E, K = 3, 128, 128, 4, 2
    x, logits, G, U, D = _tiny_moe(T, H, I, E)
    res = O.moe_ref(x, logits, G, U, D, H, I, E, K)
    Gd = [O.dequant_ref(G[0][e], G[1][e], H) for e in range(E)]
    Ud = [O.dequant_ref(U[0][e], U[1][e], H) for e in range(E)]
    Dd = [O.dequant_ref(D[0][e], D[1][e], I) for e in range(E)]
    for t in range(T):
        z = [float(v) for v in logits[t]]
        mx = max(z)
        ez = [math.exp(v - mx) for v in z]
        p = [v / math.fsum(ez) for v in ez]
        order = sorted(range(E), key=lambda e: (-p[e], e))[:K]
        for hcol in range(0, H, 37):
            total = 0.0
            for e in order:
                hvec = []
                for i in range(I):
                    gv = math.fsum(Gd[e][i, k] * x[t, k] for k in range(H))
                    uv = math.fsum(Ud[e][i, k] * x[t, k] for k in range(H))
                    hvec.append(gv / (1 + math.exp(-gv)) * uv)
                total += p[e] * math.fsum(Dd[e][hcol, i] * hvec[i] for i in range(I))
            assert res["out"][t, hcol] == pytest.approx(total, rel=1e-10, abs=1e-12)


def test_moe_single_expert_reduces_to_swiglu_ffn():
    T, H, I, E = 4, 256, 128, 1
    x, logits, G, U, D = _tiny_moe(T, H, I, E, seed=32)
    res = O.moe_ref(x, logits, G, U, D, H, I, E, 1)
    assert np.all(res["w"] == 1.0)
    g = x @ O.dequant_ref(G[0][0], G[1][0], H).T
    u = x @ O.dequant_ref(U[0][0], U[1][0], H).T
    h = g * scipy.special.expit(g) * u
    out = h @ O.dequant_ref(D[0][0], D[1][0], I).T
    assert np.allclose(res["out"], out, rtol=1e-12, atol=1e-14)


def test_moe_token_permutation_invariance():
    T, H, I, E, K = 6, 128, 128, 8, 3
    x, logits, G, U, D = _tiny_moe(T, H, I, E, seed=33)
    res = O.moe_ref(x, logits, G, U, D, H, I, E, K)
    perm = np.array([3, 0, 5, 1, 4, 2])
    res_p = O.moe_ref(x[perm], logits[perm], G, U, D, H, I, E, K)
    assert np.allclose(res_p["out"], res["out"][perm], rtol=1e-13, atol=1e-15)
    p = scipy.special.softmax(logits.astype(np.float64), axis=1)
    assert np.allclose(np.take_along_axis(p, res["ids"], 1), res["w"])
    assert np.all(res["w"].sum(1) <= 1.0 + 1e-12)


# ---------------------------------------------------------------- fast pack

def test_fast_pack_equals_plain_pack():
    g = synth.rng(40)
    W = synth.weights(g, 24, 512)
    # edge groups: ties, tie broken by a tiny value, subnormal means, zeros,
    # overflow, a huge exponent spread (forces the exact-integer fallback)
    M = np.float32(1.0 + 2.0 ** -11)
    W[0, :128] = M
    W[1, :128] = np.array([M] * 126 + [np.float32(2.0) * M, np.float32(2.0 ** -100)], np.float32)
    W[2, :128] = np.float32(3 * 2.0 ** -25)
    W[3, :128] = 0.0
    W[4, :128] = -0.0
    W[5, :128] = np.float32(70000.0)
    W[6, 5] = np.float32(2.0 ** -140)
    W[7, :128] = np.float32(2.0 ** -149)
    W[8, 128:256] = np.float32(65504.0)
    s1, c1 = O.pack_ref(W)
    s2, c2 = O.pack_ref_fast(W)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1, c2)


# ---------------------------------------------------------------- rotated activations

def _fwht(v):
    """Unnormalised fast Walsh-Hadamard transform along axis 0 (butterflies)."""
    v = np.array(v, dtype=np.float64)
    h = 1
    while h < v.shape[0]:
        for i in range(0, v.shape[0], 2 * h):
            a = v[i:i + h].copy()
            b = v[i + h:i + 2 * h].copy()
            v[i:i + h] = a + b
            v[i + h:i + 2 * h] = a - b
        h *= 2
    return v


@pytest.mark.parametrize("n1,n2", [(8, 16), (16, 16), (32, 4)])
def test_okt_rotate_equals_explicit_kronecker_matrix(n1, n2):
    """Brute force: build the K x K matrix (H kron R) and apply its transpose."""
    g = synth.rng(50 + n1)
    H = synth.orthogonal_f32(g, n1)
    R = synth.orthogonal_f32(g, n2)
    x = O.bf16_bits_to_f64(synth.activations_bf16(g, 3, n1 * n2))
    M = np.kron(H.astype(np.float64), R.astype(np.float64))
    ref = x @ M  # row b of this is (M^T x_b)^T
    out = O.okt_rotate_ref(H, R, x)
    assert np.max(np.abs(out - ref)) <= 1e-13 * np.max(np.abs(ref))


def test_okt_rotate_hadamard_factor_is_a_walsh_hadamard_transform():
    """H = Sylvester Hadamard / sqrt(n1), R = identity: each column j of the
    n1 x n2 view is Walsh-Hadamard transformed (H is symmetric)."""
    n1, n2 = 64, 8
    H = _sylvester(n1) / 8.0
    x = O.bf16_bits_to_f64(synth.activations_bf16(synth.rng(52), 2, n1 * n2))
    out = O.okt_rotate_ref(H, np.eye(n2), x)
    for b in range(2):
        ref = _fwht(x[b].reshape(n1, n2)) / 8.0
        assert np.max(np.abs(out[b].reshape(n1, n2) - ref)) <= 1e-14 * np.max(np.abs(ref))


def test_okt_rotate_permutation_factor_permutes_columns():
    """H = I, R a permutation matrix with R[pi(j), j] = 1: X R moves column
    pi(j) of the n1 x n2 view to column j, exactly."""
    n1, n2 = 4, 32
    pi = synth.rng(53).permutation(n2)
    R = np.zeros((n2, n2))
    R[pi, np.arange(n2)] = 1.0
    x = O.bf16_bits_to_f64(synth.activations_bf16(synth.rng(54), 2, n1 * n2))
    out = O.okt_rotate_ref(np.eye(n1), R, x)
    ref = x.reshape(2, n1, n2)[:, :, pi].reshape(2, n1 * n2)
    assert np.array_equal(out, ref)


def test_okt_rotate_preserves_norm_and_inverts():
    """Orthogonal factors: ||x_rot|| = ||x||, and rotating by (H^T, R^T)
    returns x (the rotation's inverse is its transpose)."""
    n1, n2 = 64, 64
    g = synth.rng(55)
    H = np.linalg.qr(g.standard_normal((n1, n1)))[0]
    R = np.linalg.qr(g.standard_normal((n2, n2)))[0]
    x = O.bf16_bits_to_f64(synth.activations_bf16(g, 4, n1 * n2))
    xr = O.okt_rotate_ref(H, R, x)
    assert np.allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12, atol=0)
    back = O.okt_rotate_ref(H.T, R.T, xr)
    assert np.max(np.abs(back - x)) <= 1e-12 * np.max(np.abs(x))


def test_okt_forward_equivalence():
    """W x = (W (H kron R)) ((H kron R)^T x) for dense W, and the packed product
    of the rotated weights is the dequantised rotated weights times x_rot."""
    n1, n2, N = 16, 16, 40
    K = n1 * n2
    g = synth.rng(56)
    H = np.linalg.qr(g.standard_normal((n1, n1)))[0]
    R = np.linalg.qr(g.standard_normal((n2, n2)))[0]
    W = g.standard_normal((N, K)) * 0.02
    x = O.bf16_bits_to_f64(synth.activations_bf16(g, 2, K))
    W_rot = W @ np.kron(H, R)
    xr = O.okt_rotate_ref(H, R, x)
    assert np.max(np.abs(xr @ W_rot.T - x @ W.T)) <= 1e-12 * np.max(np.abs(x @ W.T))
    signs, scales = O.pack_ref(W_rot.astype(np.float32))
    y, bound, x_rot = O.okt_gemv_ref(signs, scales, H, R, x, K)
    w_hat = O.dequant_ref(signs, scales, K)
    assert np.array_equal(x_rot, xr)
    assert np.max(np.abs(y - xr @ w_hat.T)) <= 1e-13 * np.max(bound)


# ---------------------------------------------------------------- approximation residuals

def test_g128_residual_energy_closed_form():
    """Per group, with w_hat = s sign(w): sum (w - w_hat)^2 = sum w^2 - 2 s sum|w| + 128 s^2
    (sign(w) w = |w| under the signbit convention)."""
    W = synth.weights(synth.rng(61), 24, 512)
    W[0, :128] = 0.0
    W[1, 5] = -0.0
    s, c = O.pack_ref(W)
    E = O.residual_g128_ref(W, s, c)
    sc = O.fp16_bits_to_f64(c)
    Wd = W.astype(np.float64)
    expect = 0.0
    for n in range(W.shape[0]):
        for g in range(W.shape[1] // 128):
            grp = Wd[n, 128 * g:128 * (g + 1)]
            expect += np.sum(grp * grp) - 2.0 * sc[n, g] * np.sum(np.abs(grp)) + 128.0 * sc[n, g] ** 2
    assert O.sum_squares_ref(E) == pytest.approx(expect, rel=1e-12)


def test_g128_relative_frobenius_of_gaussian_weights():
    """Gaussian weights: the mean-|w| sign code keeps 2/pi of the energy, so the
    relative Frobenius residual is close to sqrt(1 - 2/pi) = 0.6028 (slightly
    below it: each group fits its own scale)."""
    W = synth.weights(synth.rng(62), 256, 2048)
    s, c = O.pack_ref_fast(W)
    rel = math.sqrt(O.sum_squares_ref(O.residual_g128_ref(W, s, c)) / O.sum_squares_ref(W))
    assert 0.59 < rel < math.sqrt(1.0 - 2.0 / math.pi) + 1e-3


def test_dbf_residual_of_its_own_reconstruction_is_zero():
    """W built element by element as sum_k a_i U_ik mid_k V_kj b_j (no matmul):
    the residual against the chain's dense form is zero up to rounding."""
    m, r, n = 16, 32, 64
    a, B1, mid, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=63)
    av, mv, bv = (np.array(v, np.uint16).view(np.float16).astype(float) for v in (a, mid, b))

    def sgn(words, row, col):
        return 1 - 2 * ((int(words[row, col // 32]) >> (col % 32)) & 1)

    W = np.array([[av[i] * bv[j] * math.fsum(sgn(B1, i, k) * mv[k] * sgn(B2, k, j) for k in range(r))
                   for j in range(n)] for i in range(m)])
    E = O.dbf_residual_ref(W, a, B1, mid, B2, b, m, r, n)
    assert np.max(np.abs(E)) <= 1e-14 * np.max(np.abs(W))


def test_sum_squares_is_exact_on_integers():
    A = np.arange(-300, 301, dtype=np.float32).reshape(1, -1)
    assert O.sum_squares_ref(A) == 2 * sum(k * k for k in range(1, 301))


def test_power_iteration_diagonal_and_rank_one():
    d = np.array([0.5, -7.0, 3.0, 1.0])
    assert O.power_iteration_ref(np.diag(d), np.ones(4), 32) == pytest.approx(7.0, rel=1e-12)
    g = synth.rng(64)
    x, y = g.standard_normal(30), g.standard_normal(20)
    sigma = np.linalg.norm(x) * np.linalg.norm(y)
    assert O.power_iteration_ref(np.outer(x, y), g.standard_normal(20), 1) == pytest.approx(sigma, rel=1e-12)
    assert O.power_iteration_ref(np.zeros((5, 3)), np.ones(3), 32) == 0.0


def test_power_iteration_against_svd():
    """A planted gap (10 vs 5) converges to the largest singular value from the
    library SVD within rounding; without a gap the estimate never exceeds it."""
    g = synth.rng(65)
    Q1 = np.linalg.qr(g.standard_normal((60, 60)))[0]
    Q2 = np.linalg.qr(g.standard_normal((40, 40)))[0]
    sv = np.concatenate([[10.0, 5.0], g.uniform(0.0, 4.0, 38)])
    A = Q1[:, :40] @ np.diag(sv) @ Q2.T
    assert O.power_iteration_ref(A, g.standard_normal(40), 32) == pytest.approx(np.linalg.norm(A, 2), rel=1e-12)
    B = g.standard_normal((50, 70))
    est = O.power_iteration_ref(B, g.standard_normal(70), 32)
    assert est <= np.linalg.norm(B, 2) * (1 + 1e-12)
    assert est >= 0.9 * np.linalg.norm(B, 2)


# ---------------------------------------------------------------- D_mid reprojection

def _dbf_factors(m, r, n, seed):
    a, B1, mid, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=seed)
    return a, B1, mid, B2, b


def test_reproject_recovers_the_middle_diagonal_of_an_exact_dbf():
    m, r, n = 64, 32, 96
    a, B1, mid, B2, b = _dbf_factors(m, r, n, 80)
    W = O.dbf_dense_ref(a, B1, mid, B2, b, m, r, n)
    got, bits = O.dbf_reproject_mid_ref(W, a, B1, B2, b, m, r, n)
    assert np.max(np.abs(got - O.fp16_bits_to_f64(mid))) <= 1e-10 * np.max(np.abs(got))
    assert np.array_equal(bits, mid)  # the exact fp16 values come back


def test_reproject_matches_lstsq_on_the_explicit_design_matrix():
    """Independent formulation: least squares over the m n x r matrix whose
    columns are vec((a * U[:, k]) (V[k, :] * b)^T)."""
    m, r, n = 32, 32, 64
    a, B1, _, B2, b = _dbf_factors(m, r, n, 81)
    W = synth.weights(synth.rng(82), m, n, std=0.05).astype(np.float64)
    av, bv = O.fp16_bits_to_f64(a), O.fp16_bits_to_f64(b)

    def sgn(words, row, col):
        return 1 - 2 * ((int(words[row, col // 32]) >> (col % 32)) & 1)

    X = np.empty((m * n, r))
    for k in range(r):
        p = np.array([av[i] * sgn(B1, i, k) for i in range(m)])
        q = np.array([sgn(B2, k, j) * bv[j] for j in range(n)])
        X[:, k] = np.outer(p, q).ravel()
    ref = np.linalg.lstsq(X, W.ravel(), rcond=None)[0]
    got, _ = O.dbf_reproject_mid_ref(W, a, B1, B2, b, m, r, n)
    assert np.max(np.abs(got - ref)) <= 1e-9 * np.max(np.abs(ref))
    # the residual is orthogonal to every column (the normal equations)
    res = W.ravel() - X @ got
    assert np.max(np.abs(X.T @ res)) <= 1e-9 * np.max(np.abs(X.T @ W.ravel()))


def test_reproject_singular_design_takes_the_minimum_norm_solution():
    """Two equal columns of U and the matching two equal rows of V make
    P_k1 = P_k2: the least-squares minimiser is not unique, and the one of
    minimum norm (what lstsq on the explicit m n x r design matrix returns)
    splits the weight evenly between k1 and k2."""
    m, r, n = 32, 32, 64
    a, B1, _, B2, b = _dbf_factors(m, r, n, 86)
    k1, k2 = 3, 20
    U = O.unpack_bits_lsb_first(B1, r).astype(np.uint8)
    U[:, k2] = U[:, k1]
    B1 = np.packbits(U, axis=1, bitorder="little").view(np.uint32).reshape(m, r // 32)
    B2 = B2.copy()
    B2[k2] = B2[k1]
    W = synth.weights(synth.rng(87), m, n, std=0.05).astype(np.float64)
    av, bv = O.fp16_bits_to_f64(a), O.fp16_bits_to_f64(b)
    Us = 1.0 - 2.0 * U
    Vs = 1.0 - 2.0 * O.unpack_bits_lsb_first(B2, n)
    X = np.stack([np.outer(av * Us[:, k], Vs[k] * bv).ravel() for k in range(r)], axis=1)
    ref = np.linalg.lstsq(X, W.ravel(), rcond=None)[0]
    got, _ = O.dbf_reproject_mid_ref(W, a, B1, B2, b, m, r, n)
    assert abs(ref[k1] - ref[k2]) <= 1e-12 * np.max(np.abs(ref))
    assert np.max(np.abs(got - ref)) <= 1e-9 * np.max(np.abs(ref))


def test_reproject_is_optimal_and_bits_round_to_nearest():
    """Random perturbations of the solution raise the error; the stored bits
    are numpy's round-to-nearest fp16 of the solution."""
    m, r, n = 48, 32, 64
    a, B1, _, B2, b = _dbf_factors(m, r, n, 83)
    W = synth.weights(synth.rng(84), m, n, std=0.05).astype(np.float64)
    got, bits = O.dbf_reproject_mid_ref(W, a, B1, B2, b, m, r, n)
    av, bv = O.fp16_bits_to_f64(a), O.fp16_bits_to_f64(b)
    U = 1.0 - 2.0 * O.unpack_bits_lsb_first(B1, r)
    V = 1.0 - 2.0 * O.unpack_bits_lsb_first(B2, n)

    def err(mid):
        return float(np.sum((W - (av[:, None] * U) @ (mid[:, None] * V * bv[None, :])) ** 2))

    e0 = err(got)
    g = synth.rng(85)
    for _ in range(8):
        assert err(got + 1e-3 * g.standard_normal(r)) > e0
    assert np.array_equal(bits, got.astype(np.float16).view(np.uint16))


# ---------------------------------------------------------------- 16-bit input formats

def _ieee_decode(bits: int, ebits: int, mbits: int) -> float:
    """Value of a binary floating-point pattern from the IEEE 754 field layout
    (sign, biased exponent, fraction; exponent 0 = subnormal), exact in
    Python rationals; inf for an all-ones exponent with a zero fraction."""
    sign = -1 if (bits >> (ebits + mbits)) & 1 else 1
    e = (bits >> mbits) & ((1 << ebits) - 1)
    f = bits & ((1 << mbits) - 1)
    bias = (1 << (ebits - 1)) - 1
    if e == (1 << ebits) - 1:
        assert f == 0
        return sign * math.inf
    if e == 0:
        v = Fraction(f, 1 << mbits) * Fraction(2) ** (1 - bias)
    else:
        v = (1 + Fraction(f, 1 << mbits)) * Fraction(2) ** (e - bias)
    return math.copysign(float(v), sign)


def test_bf16_widening_hand_written_patterns():
    pats = {0x3F80: 1.0, 0xC000: -2.0, 0x3FC0: 1.5, 0x0080: 2.0 ** -126, 0x0001: 2.0 ** -133,
            0x007F: 127 * 2.0 ** -133, 0x7F7F: (2.0 - 2.0 ** -7) * 2.0 ** 127, 0x7F80: math.inf,
            0xFF80: -math.inf, 0x4049: 3.140625, 0x0000: 0.0}
    got = O.bf16_bits_to_f64(np.array(list(pats), dtype=np.uint16))
    assert got.tolist() == list(pats.values())
    neg0 = O.bf16_bits_to_f64(np.array([0x8000], dtype=np.uint16))[0]
    assert neg0 == 0.0 and math.copysign(1.0, neg0) == -1.0


def test_bf16_and_fp16_widening_match_the_field_layout_for_every_pattern():
    # brute force over all 65536 patterns except NaNs (all-ones exponent with a
    # nonzero fraction): bf16 = 1/8/7 with bias 127, binary16 = 1/5/10 with bias 15
    allp = np.arange(1 << 16, dtype=np.uint32)
    for fn, eb, mb in ((O.bf16_bits_to_f64, 8, 7), (O.fp16_bits_to_f64, 5, 10)):
        emask = ((1 << eb) - 1) << mb
        keep = ~(((allp & emask) == emask) & ((allp & ((1 << mb) - 1)) != 0))
        pats = allp[keep]
        got = fn(pats.astype(np.uint16))
        want = np.array([_ieee_decode(int(p), eb, mb) for p in pats], dtype=np.float64)
        assert np.array_equal(got, want)
        assert np.array_equal(np.signbit(got), (pats >> 15).astype(bool))


def test_bf16_widening_inverts_the_library_rounding_of_bf16_exact_values():
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(17)
    # values with at most 8 significant bits over the whole exponent range
    # (normal and subnormal), so the library's float32 -> bf16 conversion is exact
    man = g.integers(128, 256, 5000).astype(np.float64)
    ex = g.integers(-133, 120, 5000)
    sub = g.integers(1, 128, 500).astype(np.float64) * 2.0 ** -133   # bf16 subnormals
    v = np.concatenate([man * np.exp2(ex.astype(np.float64)), sub])
    v *= np.where(g.random(v.size) < 0.5, -1.0, 1.0)
    bits = torch.tensor(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_bits_to_f64(bits), v.astype(np.float32).astype(np.float64))


def test_fast_pack_equals_plain_pack_on_wide_exponent_spreads():
    # a few thousand groups whose magnitudes span up to 31 binades (the int64
    # alignment window) and beyond (the exact fallback), with random signs,
    # subnormals and zeros mixed in
    g = np.random.default_rng(41)
    rows, K = 96, 4096
    W = np.empty((rows, K), dtype=np.float32)
    for n in range(rows):
        for c in range(K // 128):
            spread = int(g.integers(0, 40))
            top = int(g.integers(-126, 100))
            ex = top - g.integers(0, spread + 1, 128)
            man = g.random(128) + 1.0
            v = np.ldexp(man, ex).astype(np.float32)
            if g.random() < 0.2:
                v[g.integers(0, 128, 8)] = np.float32(2.0 ** -149) * g.integers(1, 1 << 20, 8)
            if g.random() < 0.1:
                v[g.integers(0, 128, 16)] = 0.0
            if c % 4 == 0:
                # mean exactly on an fp16 rounding midpoint (fp16 value + half
                # an ulp), with or without a tie-breaker far below the
                # alignment window of the largest value
                h = np.float16(np.exp2(g.uniform(-13, 15)) * (1 + g.random()))
                if not np.isfinite(h) or h == 0 or h >= np.float16(65504):
                    h = np.float16(1.5)
                M = np.float32((float(h) + float(np.nextafter(h, np.float16(np.inf)))) / 2)
                v = np.full(128, M, dtype=np.float32)
                v[126] = np.float32(2.0) * M
                v[127] = np.float32(2.0) ** int(g.integers(-149, -60)) if g.random() < 0.5 else 0.0
                v = v[g.permutation(128)]
            v *= np.where(g.random(128) < 0.5, -1.0, 1.0).astype(np.float32)
            W[n, c * 128:(c + 1) * 128] = v
    s1, c1 = O.pack_ref(W)
    s2, c2 = O.pack_ref_fast(W)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1, c2)

"""w1_residual / dbf_residual / w1_power_iteration on the GPU vs the fp64 oracle.

E of the sign code is one fp32 rounding of w - w_hat: compared bit for bit.
E of a DBF chain carries the fp32 sum over r: |W_approx - exact| <=
(r + 2) 2^-24 |a_i| |b_j| sum_k |mid_k|, plus one rounding of E.  The sums of
squares follow from the elementwise bounds.  Power iteration is fp64 on both
sides and differs only in summation order.
"""
import functools

import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import dev, f32_dev, fp16_dev, words_dev

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


@functools.lru_cache(maxsize=None)
def g128_case(N, K, seed):
    W, _ = synth.gemv_case(N, K, 1, seed=seed)
    s, c = O.pack_ref_fast(W)
    return W, s, c


@pytest.mark.parametrize("N,K", [(512, 1024), (4096, 4096), (300, 1152), (1, 128), (11008, 4096)])
def test_residual_g128_parity(N, K):
    W, s, c = g128_case(N, K, 70)
    Wd = f32_dev(W)
    E, sums = ops.w1_residual(Wd, words_dev(s), fp16_dev(c))
    assert ops.sync_status() == _lib.W1_OK
    E_ref = O.residual_g128_ref(W, s, c)
    assert np.array_equal(E.cpu().numpy(), E_ref.astype(np.float32)), "E is not w - w_hat rounded once"
    se, sw = sums.cpu().numpy()
    assert se == pytest.approx(O.sum_squares_ref(E_ref), rel=4 * U)
    assert sw == pytest.approx(O.sum_squares_ref(W), rel=1e-12)
    _, sums2 = ops.w1_residual(Wd, words_dev(s), fp16_dev(c), want_E=False)
    _, sums3 = ops.w1_residual(Wd, words_dev(s), fp16_dev(c))
    assert torch.equal(sums, sums2) and torch.equal(sums, sums3), "sums depend on E or on the run"


def test_residual_g128_gaussian_relative_frobenius():
    W, s, c = g128_case(4096, 4096, 70)
    _, sums = ops.w1_residual(f32_dev(W), words_dev(s), fp16_dev(c), want_E=False)
    se, sw = sums.cpu().numpy()
    assert 0.59 < np.sqrt(se / sw) < np.sqrt(1 - 2 / np.pi) + 1e-3


@pytest.mark.parametrize("m,r,n", [(256, 128, 384), (512, 512, 512), (1024, 256, 640), (4096, 4096, 4096)])
def test_dbf_residual_parity(m, r, n):
    a, B1, mid, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=71)
    W = synth.weights(synth.rng(72), m, n)
    args = (fp16_dev(a), words_dev(B1), fp16_dev(mid), words_dev(B2), fp16_dev(b))
    E, sums = ops.dbf_residual(f32_dev(W), *args)
    assert ops.sync_status() == _lib.W1_OK
    E_ref = O.dbf_residual_ref(W, a, B1, mid, B2, b, m, r, n)
    av, mv, bv = (np.abs(O.fp16_bits_to_f64(v)) for v in (a, mid, b))
    delta = U * ((r + 3) * np.outer(av, bv) * mv.sum() + np.abs(E_ref))
    got = E.cpu().numpy().astype(np.float64)
    err = np.abs(got - E_ref)
    assert np.all(err <= delta), f"max err / bound {float((err / delta).max()):.3g}"
    se, sw = sums.cpu().numpy()
    se_ref = O.sum_squares_ref(E_ref)
    assert abs(se - se_ref) <= float(np.sum(2 * np.abs(E_ref) * delta + delta * delta)) + 1e-12 * se_ref
    assert sw == pytest.approx(O.sum_squares_ref(W), rel=1e-12)
    _, sums2 = ops.dbf_residual(f32_dev(W), *args, want_E=False)
    assert torch.equal(sums, sums2)


def test_dbf_residual_of_a_dbf_matrix_is_small():
    """W equal to the chain's own dense form (rounded to fp32): E is only rounding."""
    m = r = n = 256
    a, B1, mid, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=73)
    W = O.dbf_dense_ref(a, B1, mid, B2, b, m, r, n).astype(np.float32)
    E, sums = ops.dbf_residual(f32_dev(W), fp16_dev(a), words_dev(B1), fp16_dev(mid), words_dev(B2), fp16_dev(b))
    assert ops.sync_status() == _lib.W1_OK
    assert float(sums[0]) <= 1e-10 * float(sums[1])


@pytest.mark.parametrize("m,n,iters", [(512, 1024, 32), (4096, 4096, 32), (300, 1160, 32), (1, 128, 32),
                                       (64, 4, 32), (1000, 2048, 0), (777, 512, 5), (200, 8192, 7),
                                       (96, 8320, 4)])
def test_power_iteration_parity(m, n, iters):
    A = synth.weights(synth.rng(74), m, n, std=1.0)
    v0 = synth.start_vector(n)
    sig = ops.w1_power_iteration(f32_dev(A), f32_dev(v0), iters)
    assert ops.sync_status() == _lib.W1_OK
    ref = O.power_iteration_ref(A, v0, iters)
    assert float(sig) == pytest.approx(ref, rel=1e-9)
    sig2 = ops.w1_power_iteration(f32_dev(A), f32_dev(v0), iters)
    assert torch.equal(sig, sig2)


def test_power_iteration_special_cases():
    n = 256
    d = np.zeros((n, n), np.float32)
    d[np.arange(n), np.arange(n)] = np.linspace(0.1, 3.0, n, dtype=np.float32)
    d[7, 7] = -9.0
    sig = ops.w1_power_iteration(f32_dev(d), f32_dev(synth.start_vector(n)), 32)
    assert float(sig) == pytest.approx(9.0, rel=1e-12)
    zero = ops.w1_power_iteration(f32_dev(np.zeros((32, 64), np.float32)), f32_dev(synth.start_vector(64)), 32)
    assert float(zero) == 0.0
    z0 = ops.w1_power_iteration(f32_dev(d), f32_dev(np.zeros(n, np.float32)), 32)
    assert float(z0) == 0.0
    assert ops.sync_status() == _lib.W1_OK


def test_relative_spectral_residual_g128():
    """The section's spectral metric end to end on a 1024 x 1024 Gaussian matrix:
    ||E||_2 / ||W||_2 from the device equals the oracle's."""
    W, s, c = g128_case(1024, 1024, 75)
    Wd = f32_dev(W)
    E, _ = ops.w1_residual(Wd, words_dev(s), fp16_dev(c))
    v0 = f32_dev(synth.start_vector(1024))
    rel = float(ops.w1_power_iteration(E, v0, 32)) / float(ops.w1_power_iteration(Wd, v0, 32))
    E_ref = O.residual_g128_ref(W, s, c).astype(np.float32)
    v = synth.start_vector(1024)
    rel_ref = O.power_iteration_ref(E_ref, v, 32) / O.power_iteration_ref(W, v, 32)
    assert rel == pytest.approx(rel_ref, rel=1e-9)
    assert 0.3 < rel < 1.0


@pytest.mark.parametrize("abytes,bbytes,ctas,early", [(2359296, 0, 296, False), (4096 * 1024 // 8, 4096 * 8 * 2, 148, True),
                                                      (16, 48, 3, True), (6340608, 16, 1000, False)])
def test_stream_probe_reads_every_byte_once(abytes, bbytes, ctas, early):
    """w1_stream_probe folds each 16-byte chunk of both ranges into its CTA's
    word; the words' sum is the sum over all chunks of x ^ y ^ z ^ w (mod 2^32)
    whatever the CTA count -- so every chunk was read exactly once."""
    g = np.random.default_rng(abytes + bbytes + ctas)
    a = g.integers(0, 2 ** 32, size=abytes // 4, dtype=np.uint32)
    b = g.integers(0, 2 ** 32, size=max(bbytes // 4, 4), dtype=np.uint32)[: bbytes // 4]
    out = torch.zeros(ctas, dtype=torch.int32, device=dev())
    bd = words_dev(b) if bbytes else None
    ops.w1_stream_probe(words_dev(a), bd, out, ctas, early)
    assert ops.sync_status() == _lib.W1_OK

    def fold(v):
        q = v.reshape(-1, 4)
        return int(np.sum((q[:, 0] ^ q[:, 1] ^ q[:, 2] ^ q[:, 3]).astype(np.uint64)) % (1 << 32))

    want = (fold(a) + (fold(b) if bbytes else 0)) % (1 << 32)
    got = int(np.sum(out.cpu().numpy().view(np.uint32).astype(np.uint64)) % (1 << 32))
    assert got == want

"""dbf_reproject_mid on the GPU vs the fp64 oracle (dbf_reproject_mid_ref).

Both sides solve the same normal equations in fp64 (the oracle by LU /
least squares, the GPU by conjugate gradients), so the fp64 solutions agree
to a small multiple of the solve's stopping tolerance; the fp16 bits are one
round-to-nearest-even of the solution and must match wherever the oracle's
value is not within that tolerance of an fp16 rounding midpoint.  At full
size (4096^3) the oracle's triple contraction is out of reach, so the check
there is the closed form: W built from an exact DBF returns its own middle
diagonal bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import f32_dev, fp16_dev, words_dev, bits16_host

pytestmark = pytest.mark.gpu


def _args(a, B1, B2, b):
    return fp16_dev(a), words_dev(B1), words_dev(B2), fp16_dev(b)


def _fp16_near_midpoint(v: np.ndarray, rel: float) -> np.ndarray:
    """True where v lies within rel * |v| of a point halfway between two fp16 values."""
    h = v.astype(np.float16)
    lo = np.nextafter(h, np.float16(-np.inf)).astype(np.float64)
    hi = np.nextafter(h, np.float16(np.inf)).astype(np.float64)
    hv = h.astype(np.float64)
    d = np.minimum(np.abs(v - (hv + lo) / 2), np.abs(v - (hv + hi) / 2))
    return d <= rel * np.abs(v) + 1e-300


def _check_against_oracle(W, a, B1, B2, b, m, r, n, rel=1e-9):
    mid, mid64, info = ops.dbf_reproject_mid(f32_dev(W), *_args(a, B1, B2, b))
    assert ops.sync_status() == _lib.W1_OK
    it, conv = info.cpu().tolist()
    assert conv == 1 and 0 < it <= 200
    ref, ref_bits = O.dbf_reproject_mid_ref(W.astype(np.float64), a, B1, B2, b, m, r, n)
    got = mid64.cpu().numpy()
    assert np.max(np.abs(got - ref)) <= rel * np.max(np.abs(ref))
    bits = bits16_host(mid)
    ok = (bits == ref_bits) | _fp16_near_midpoint(ref, 10 * rel)
    assert np.all(ok), f"{np.count_nonzero(~ok)} fp16 roundings differ"
    assert np.array_equal(bits, got.astype(np.float16).view(np.uint16)), "bits are not the rounded fp64 result"
    return mid, mid64


@pytest.mark.parametrize("m,r,n", [(256, 128, 256), (200, 256, 384), (1000, 640, 1152), (77, 128, 128)])
def test_reproject_random_w_matches_oracle(m, r, n):
    a, B1, _, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=90)
    W = synth.weights(synth.rng(91), m, n, std=0.05)
    _check_against_oracle(W, a, B1, B2, b, m, r, n)


@pytest.mark.parametrize("m,r,n", [(256, 256, 256), (300, 128, 640)])
def test_reproject_recovers_exact_dbf(m, r, n):
    a, B1, mid0, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=92)
    W = O.dbf_dense_ref(a, B1, mid0, B2, b, m, r, n).astype(np.float32)
    mid, _ = _check_against_oracle(W, a, B1, B2, b, m, r, n)
    assert np.array_equal(bits16_host(mid), mid0)


def test_reproject_full_size_recovers_exact_dbf():
    m = r = n = 4096
    a, B1, mid0, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=93)
    W = O.dbf_dense_ref(a, B1, mid0, B2, b, m, r, n).astype(np.float32)
    mid, mid64, info = ops.dbf_reproject_mid(f32_dev(W), *_args(a, B1, B2, b))
    assert ops.sync_status() == _lib.W1_OK
    assert info.cpu().tolist()[1] == 1
    assert np.array_equal(bits16_host(mid), mid0)
    rel = np.abs(mid64.cpu().numpy() / O.fp16_bits_to_f64(mid0) - 1.0)
    assert np.max(rel) < 1e-6  # fp32 storage of W moves the optimum by ~2^-24


def test_reproject_singular_gram_takes_minimum_norm_solution():
    """Column k2 of U equal to column k1 and row k2 of V equal to row k1:
    P_k1 = P_k2, G is singular, and least squares splits the weight evenly."""
    m, r, n = 128, 128, 256
    a, B1, _, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=94)
    U = O.unpack_bits_lsb_first(B1, r)
    k1, k2 = 5, 70
    U[:, k2] = U[:, k1]
    B1 = np.packbits(U.astype(np.uint8), axis=1, bitorder="little").view(np.uint32).reshape(m, r // 32)
    B2 = B2.copy()
    B2[k2] = B2[k1]
    W = synth.weights(synth.rng(95), m, n, std=0.05)
    _, mid64 = _check_against_oracle(W, a, B1, B2, b, m, r, n, rel=1e-8)
    got = mid64.cpu().numpy()
    assert got[k1] == pytest.approx(got[k2], rel=1e-9)


def test_reproject_iteration_limit_and_reproducibility():
    m, r, n = 256, 256, 256
    a, B1, _, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1, seed=96)
    W = f32_dev(synth.weights(synth.rng(97), m, n, std=0.05))
    args = _args(a, B1, B2, b)
    mid, mid64, info = ops.dbf_reproject_mid(W, *args, max_iter=1, tol=0.0)
    assert ops.sync_status() == _lib.W1_ERR_NOT_CONVERGED
    assert info.cpu().tolist() == [1, 0]
    mid0, mid64_0, info0 = ops.dbf_reproject_mid(W, *args, max_iter=0)
    assert ops.sync_status() == _lib.W1_ERR_NOT_CONVERGED
    assert info0.cpu().tolist() == [0, 0] and torch.count_nonzero(mid64_0).item() == 0
    m1, d1, _ = ops.dbf_reproject_mid(W, *args)
    m2, d2, _ = ops.dbf_reproject_mid(W, *args)
    assert ops.sync_status() == _lib.W1_OK
    assert torch.equal(m1, m2) and torch.equal(d1, d2), "results depend on the run"

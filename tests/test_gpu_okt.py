"""w1_okt_rotate / w1_okt_gemv on the GPU vs the fp64 oracle, element by element.

Rotation bound: each element is two fp32 dot products (length n1, then n2),
so |x_rot - exact| <= (n1 + n2 + 2) 2^-24 (|H|^T |X| |R|)[i, j].
Product bound: the GEMV's 1e-3 * sum_k |s x_rot_k|, plus that rotation error
carried through the weights, sum_k |s_k| * rotation bound_k.
"""
import functools

import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import TOL, assert_within, bf16_dev, f32_dev, fp16_dev, words_dev

pytestmark = pytest.mark.gpu


def rot_bound(H, R, x):
    """(|H|^T |X| |R|) per row, with the fp32 two-dot error factor applied."""
    n1, n2 = H.shape[0], R.shape[0]
    absx = np.abs(O.bf16_bits_to_f64(x))
    Ha, Ra = np.abs(H.astype(np.float64)), np.abs(R.astype(np.float64))
    out = np.stack([(Ha.T @ absx[b].reshape(n1, n2) @ Ra).reshape(-1) for b in range(x.shape[0])])
    return (n1 + n2 + 2) * 2.0 ** -24 * out


def run_rotate(H, R, x):
    xr = ops.w1_okt_rotate(f32_dev(H), f32_dev(R), bf16_dev(x))
    assert ops.sync_status() == _lib.W1_OK
    return xr


@pytest.mark.parametrize("n1,n2,B", [(32, 32, 1), (64, 64, 1), (64, 64, 8), (86, 128, 3), (112, 128, 2),
                                     (1, 128, 1), (128, 1, 2), (8, 16, 5), (32, 32, 200),
                                     (512, 128, 1), (1024, 64, 2)])
def test_okt_rotate_parity(n1, n2, B):
    K = n1 * n2
    H, R, _, x = synth.okt_case(1, K, n1, n2, B, seed=60 + n1 + n2)
    xr = run_rotate(H, R, x)
    ref = O.okt_rotate_ref(H, R, O.bf16_bits_to_f64(x))
    got = xr.cpu().numpy().astype(np.float64)
    lim = rot_bound(H, R, x)
    bad = np.abs(got - ref) > lim
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} elements outside the fp32 dot bound"
    xr2 = run_rotate(H, R, x)
    assert torch.equal(xr, xr2), "rotation is not bitwise reproducible"


def test_okt_rotate_exact_special_factors():
    """Identity H and a permutation R move bf16 values exactly (one nonzero
    term per dot), so the device result equals the oracle bit for bit."""
    n1, n2 = 64, 64
    pi = synth.rng(70).permutation(n2)
    R = np.zeros((n2, n2), np.float32)
    R[pi, np.arange(n2)] = 1.0
    H = np.eye(n1, dtype=np.float32)
    x = synth.activations_bf16(synth.rng(71), 4, n1 * n2)
    got = run_rotate(H, R, x).cpu().numpy().astype(np.float64)
    assert np.array_equal(got, O.okt_rotate_ref(H, R, O.bf16_bits_to_f64(x)))


@functools.lru_cache(maxsize=None)
def okt_packed(N, K, n1, n2):
    H, R, W_rot, _ = synth.okt_case(N, K, n1, n2, 1)
    s, c = O.pack_ref_fast(W_rot)
    return H, R, s, c


@pytest.mark.parametrize("static_weights", [False, True])
@pytest.mark.parametrize("N,K,n1,n2,B", [(512, 1024, 32, 32, 1), (4096, 4096, 64, 64, 1), (4096, 4096, 64, 64, 4),
                                         (4096, 4096, 64, 64, 8), (11008, 4096, 64, 64, 8),
                                         (4096, 11008, 86, 128, 4), (300, 1152, 9, 128, 3),
                                         (17, 128, 1, 128, 2), (1000, 2048, 128, 16, 7)])
def test_okt_gemv_parity(N, K, n1, n2, B, static_weights):
    H, R, s, c = okt_packed(N, K, n1, n2)
    x = synth.activations_bf16(synth.rng(80 + B), B, K)
    xr = torch.empty((B, K), dtype=torch.float32, device="cuda")
    y = ops.w1_okt_gemv(words_dev(s), fp16_dev(c), f32_dev(H), f32_dev(R), bf16_dev(x), x_rot=xr,
                        static_weights=static_weights)
    assert ops.sync_status() == _lib.W1_OK
    y_ref, bound, x_rot_ref = O.okt_gemv_ref(s, c, H, R, O.bf16_bits_to_f64(x), K)
    rb = rot_bound(H, R, x)
    carried = rb @ np.abs(O.dequant_ref(s, c, K)).T
    got = y.cpu().numpy().astype(np.float64)
    err = np.abs(got - y_ref)
    lim = TOL * bound + carried
    bad = err > lim
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs outside the bound; max ratio " \
                          f"{float((err / np.maximum(lim, 1e-300)).max()):.3g}"
    # x_rot is the rotation's output, and the product is reproducible
    assert torch.equal(xr, run_rotate(H, R, x))
    y2 = ops.w1_okt_gemv(words_dev(s), fp16_dev(c), f32_dev(H), f32_dev(R), bf16_dev(x), x_rot=xr,
                         static_weights=static_weights)
    assert torch.equal(y, y2)


def test_okt_gemv_matches_plain_gemv_on_identity_rotation():
    """H = I, R = I: x_rot is x widened to fp32 exactly, so the product equals
    w1_gemv's on the same x up to fp32 summation order (both within the bound)."""
    N, K = 1024, 4096
    W, x = synth.gemv_case(N, K, 2, seed=90)
    s, c = O.pack_ref_fast(W)
    I64 = np.eye(64, dtype=np.float32)
    y_rot = ops.w1_okt_gemv(words_dev(s), fp16_dev(c), f32_dev(I64), f32_dev(I64), bf16_dev(x))
    y_plain = ops.w1_gemv(words_dev(s), fp16_dev(c), bf16_dev(x))
    assert ops.sync_status() == _lib.W1_OK
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s, c, K)
    assert_within(y_rot.cpu().numpy(), y_ref, bound, what="identity rotation")
    assert_within(y_plain.cpu().numpy(), y_ref, bound, what="plain")

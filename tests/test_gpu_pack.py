"""w1_pack on the GPU vs the oracle: bit-exact signs and scales."""
import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import f32_dev, words_host, bits16_host

pytestmark = pytest.mark.gpu


def _pack(W):
    signs, scales = ops.w1_pack(f32_dev(W))
    st = ops.sync_status()
    return words_host(signs), bits16_host(scales), st


def test_pack_tiny_config_bit_exact():
    W, _ = synth.tiny_case()
    s_ref, c_ref = O.pack_ref(W)
    s, c, st = _pack(W)
    assert st == _lib.W1_OK
    assert np.array_equal(s, s_ref)
    assert np.array_equal(c, c_ref)


def test_pack_edge_groups_bit_exact():
    g = synth.rng(50)
    W = synth.weights(g, 16, 512)
    M = np.float32(1.0 + 2.0 ** -11)
    W[0, :128] = M                                                    # exact tie -> even
    W[1, :128] = np.array([M] * 126 + [np.float32(2.0) * M, np.float32(2.0 ** -100)], np.float32)
    W[2, :128] = np.float32(3 * 2.0 ** -25)                           # subnormal tie
    W[3, :128] = 0.0
    W[4, :128] = -0.0
    W[5, 128:256] = np.float32(65519.0)                              # just below overflow
    W[6, 5] = np.float32(2.0 ** -140)
    W[7, :128] = np.float32(2.0 ** -149)
    W[8, :128] = np.float32(1.0 + 2.0 ** -11 + 2.0 ** -23)           # just above a tie
    W[9, 0:128:2] *= -1.0
    s_ref, c_ref = O.pack_ref(W)
    s, c, st = _pack(W)
    assert st == _lib.W1_OK
    assert np.array_equal(s, s_ref)
    assert np.array_equal(c, c_ref)


def test_pack_overflow_sets_range_status():
    W = synth.weights(synth.rng(51), 2, 256)
    W[1, 128:] = np.float32(70000.0)
    s_ref, c_ref = O.pack_ref(W)
    s, c, st = _pack(W)
    assert st == _lib.W1_ERR_RANGE
    assert c[1, 1] == 0x7C00 and np.array_equal(c, c_ref) and np.array_equal(s, s_ref)


def test_pack_nonfinite_sets_status():
    W = synth.weights(synth.rng(52), 2, 256)
    W[0, 3] = np.nan
    s, c, st = _pack(W)
    assert st == _lib.W1_ERR_NONFINITE
    Wc = W.copy()
    Wc[0, :128] = 1.0
    _, c_ref = O.pack_ref(Wc)
    assert np.array_equal(c[1], c_ref[1]) and np.array_equal(c[0, 1:], c_ref[0, 1:])


@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 14336)])
def test_pack_full_size_sampled_rows(N, K):
    W, _ = synth.gemm_case(1, N, K)
    s, c, st = _pack(W)
    assert st == _lib.W1_OK
    assert np.array_equal(s, O.pack_bits_lsb_first(O.sign_bits_ref(W)))
    rows = np.sort(np.random.default_rng(0).choice(N, 384, replace=False))
    _, c_ref = O.pack_ref_fast(W[rows])
    assert np.array_equal(c[rows], c_ref)

"""w1_gemm (tcgen05) on the GPU vs the fp64 oracle."""
import functools

import numpy as np
import pytest

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import assert_within, bf16_dev, fp16_dev, words_dev

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def packed(N, K, seed):
    W, _ = synth.gemm_case(1, N, K, seed=seed)
    return O.pack_ref_fast(W)


def run_gemm(signs, scales, x_bits):
    y = ops.w1_gemm(words_dev(signs), fp16_dev(scales), bf16_dev(x_bits))
    assert ops.sync_status() == _lib.W1_OK
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (256, 256, 512), (200, 300, 384), (1, 130, 256),
                                   (777, 1000, 1152), (129, 4097, 256)])
def test_gemm_small_and_ragged(M, N, K):
    s, c = packed(N, K, M + N + K)
    x = synth.activations_bf16(synth.rng(M), M, K)
    y = run_gemm(s, c, x)
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s, c, K)
    assert_within(y, y_ref, bound, what=f"{M}x{N}x{K}")


@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_gemm_config_shapes_full(N, K):
    M = 2048
    s, c = packed(N, K, synth.SEEDS["gemm"])
    x = synth.activations_bf16(synth.rng(synth.SEEDS["gemm"] + 100), M, K)
    y = run_gemm(s, c, x)
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s, c, K)
    assert_within(y, y_ref, bound, what=f"2048x{N}x{K}")


def test_gemm_config_14336_square_sampled_rows():
    M, N, K = 2048, 14336, 14336
    s, c = packed(N, K, synth.SEEDS["gemm"])
    x = synth.activations_bf16(synth.rng(synth.SEEDS["gemm"] + 100), M, K)
    y = run_gemm(s, c, x)
    rows = np.sort(np.random.default_rng(1).choice(N, 256, replace=False))
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s[rows], c[rows], K)
    assert_within(y[:, rows], y_ref, bound, what="2048x14336x14336 sampled")


def test_gemm_integer_inputs_bit_exact():
    g = np.random.default_rng(70)
    M, N, K = 256, 384, 1024
    c = (2.0 ** g.integers(-3, 3, size=(N, K // 128))).astype(np.float32)
    W = np.where(g.random((N, K)) < 0.5, -1.0, 1.0).astype(np.float32) * np.repeat(c, 128, axis=1)
    s, sc = O.pack_ref_fast(W)
    xi = g.integers(-2, 3, size=(M, K)).astype(np.float32)
    y = run_gemm(s, sc, synth.f32_to_bf16_bits(xi))
    y_ref, _ = O.matmul_ref(xi.astype(np.float64), s, sc, K)
    assert np.array_equal(y, y_ref)


@pytest.mark.parametrize("bm,exp,a", [(128, 4, "smem"), (128, 8, "smem"), (128, 4, "tmem"), (128, 8, "tmem"),
                                      (256, 4, "smem"), (256, 8, "smem")])
def test_gemm_every_kernel_form(knob, bm, exp, a):
    """Each token tile x expander count x weight-operand place on a ragged case
    with several tiles per CTA (persistent loop, both accumulators, stage ring
    wrapping across tiles): within the bound, and bit for bit equal to the
    shared-memory, 4-expander form of the same tile (same MMAs, same order)."""
    M, N, K = 1100, 2200, 1152
    s, c = packed(N, K, 91)
    x = synth.activations_bf16(synth.rng(92), M, K)
    knob("sg_bm", bm)
    knob("sg_exp", exp)
    knob("sg_a", a)
    y = run_gemm(s, c, x)
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s, c, K)
    assert_within(y, y_ref, bound, what=f"bm={bm} exp={exp} a={a}")
    knob("sg_exp", 4)
    knob("sg_a", "smem")
    assert np.array_equal(y, run_gemm(s, c, x))

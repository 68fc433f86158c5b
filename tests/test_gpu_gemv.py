"""w1_gemv on the GPU vs the fp64 oracle (element-wise, 1e-3 * sum|s x| bound).

Every test runs on each kernel, forced with the gemv_path knob: the
register-fed kernel with 8 and with 16 warps per CTA (flat / flat16: int8
activation digits up to 2 rows, bf16 activations above), the int8 direct
kernel with 8 and 16 warps (direct / direct16), the tcgen05 kernel (tc) and
the mma.sync ring kernel (ring, the fallback for other shapes)."""
import functools

import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import assert_within, bf16_dev, fp16_dev, words_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["flat", "flat16", "direct", "direct16", "tc", "ring"])
def gemv_path(request, knob):
    knob("gemv_path", request.param)
    return request.param


@functools.lru_cache(maxsize=None)
def packed_case(N, K, seed):
    W, _ = synth.gemv_case(N, K, 1, seed=seed)
    return O.pack_ref_fast(W)


def run_gemv(signs, scales, x_bits):
    y = ops.w1_gemv(words_dev(signs), fp16_dev(scales), bf16_dev(x_bits))
    assert ops.sync_status() == _lib.W1_OK
    return y.cpu().numpy().astype(np.float64)


def check(signs, scales, x_bits, K, what):
    y = run_gemv(signs, scales, x_bits)
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x_bits), signs, scales, K)
    return assert_within(y, y_ref, bound, what=what)


def test_gemv_tiny_config():
    W, x = synth.tiny_case()
    s, c = O.pack_ref(W)
    check(s, c, x, 1024, "tiny 512x1024 B=1")


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("B", [1, 4, 8])
def test_gemv_config_shapes(N, K, B):
    s, c = packed_case(N, K, synth.SEEDS["gemv"])
    x = synth.activations_bf16(synth.rng(100 + B), B, K)
    check(s, c, x, K, f"{N}x{K} B={B}")


@pytest.mark.parametrize("N,K,B", [(1, 128, 1), (15, 256, 2), (17, 384, 3), (1000, 1152, 5),
                                   (33, 128, 6), (257, 640, 7), (4097, 2176, 8), (100, 11008, 1)])
def test_gemv_ragged_and_small(N, K, B):
    W, x = synth.gemv_case(N, K, B, seed=N + K + B)
    s, c = O.pack_ref_fast(W)
    check(s, c, x, K, f"{N}x{K} B={B}")


def test_gemv_integer_inputs_bit_exact():
    g = np.random.default_rng(60)
    N, K, B = 300, 1024, 8
    c = (2.0 ** g.integers(-3, 3, size=(N, K // 128))).astype(np.float32)
    W = np.where(g.random((N, K)) < 0.5, -1.0, 1.0).astype(np.float32) * np.repeat(c, 128, axis=1)
    s, sc = O.pack_ref_fast(W)
    xi = g.integers(-2, 3, size=(B, K)).astype(np.float32)
    x = synth.f32_to_bf16_bits(xi)
    y = run_gemv(s, sc, x)
    y_ref, _ = O.matmul_ref(xi.astype(np.float64), s, sc, K)
    assert np.array_equal(y, y_ref)


def test_gemv_one_hot_reads_scales():
    N, K = 64, 512
    s, c = packed_case(N, K, 61)
    for k in (0, 1, 31, 32, 130, 511):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y = run_gemv(s, c, synth.f32_to_bf16_bits(x))
        y_ref, _ = O.matmul_ref(x.astype(np.float64), s, c, K)
        assert np.array_equal(y, y_ref), k


def test_gemv_extreme_activation_ranges():
    """Groups of x spanning huge / tiny magnitudes and one-large-many-tiny groups."""
    N, K, B = 256, 1024, 4
    s, c = packed_case(N, K, 62)
    g = synth.rng(63)
    x = synth.normal_f32(g, (B, K))
    x[0, :128] *= 1e30
    x[1, 128:256] *= 1e-30
    x[2, 256:384] = 1e-6 * x[2, 256:384]
    x[2, 300] = 50.0                      # one large value, the rest tiny
    x[3, :] = 0.0
    check(s, c, synth.f32_to_bf16_bits(x), K, "extreme x")


def test_gemv_is_deterministic():
    s, c = packed_case(4096, 4096, synth.SEEDS["gemv"])
    x = synth.activations_bf16(synth.rng(64), 8, 4096)
    a = run_gemv(s, c, x)
    b = run_gemv(s, c, x)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("split", ["1", "2", "4", "8"])
@pytest.mark.parametrize("N,K,B", [(4096, 4096, 1), (1000, 1152, 5), (4097, 2176, 8), (300, 1024, 2),
                                   (4096, 11008, 8)])
def test_gemv_direct_every_split(N, K, B, split, gemv_path, knob):
    """The cluster K split (1..8 CTAs) of the fp8 and direct kernels on the
    same inputs.  4096 x 11008 at B = 8 needs the direct kernel's reduction
    buffer over the activation scratch at 16 warps and small splits."""
    if not (gemv_path.startswith("direct") or gemv_path.startswith("flat")):
        pytest.skip("split sweep is for the split-capable kernels")
    knob("gemv_split", split)
    W, x = synth.gemv_case(N, K, B, seed=N + B)
    s, c = O.pack_ref_fast(W)
    try:
        check(s, c, x, K, f"{N}x{K} B={B} split={split}")
    except _lib.W1Error as e:
        if e.status != _lib.W1_ERR_UNSUPPORTED:
            raise
        pytest.skip(f"split {split} does not fit {N}x{K}")


def test_gemv_static_weights_flag_same_result(gemv_path):
    """W1_GEMV_STATIC_WEIGHTS changes only when the weights are read: the
    weights here were written long before, so results are identical."""
    s, c = packed_case(4096, 4096, synth.SEEDS["gemv"])
    x = bf16_dev(synth.activations_bf16(synth.rng(65), 4, 4096))
    sd, cd = words_dev(s), fp16_dev(c)
    torch.cuda.synchronize()
    a = ops.w1_gemv(sd, cd, x)
    b = ops.w1_gemv(sd, cd, x, static_weights=True)
    assert ops.sync_status() == _lib.W1_OK
    assert torch.equal(a, b)

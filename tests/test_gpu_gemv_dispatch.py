"""w1_gemv through the default dispatch (kernel and K split chosen by timing
on the first call of a shape) vs the fp64 oracle."""
import numpy as np
import pytest

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import assert_within, bf16_dev, fp16_dev, words_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def default_dispatch(knob):
    knob("gemv_path", "0")
    knob("gemv_split", "0")
    knob("gemv_autotune", "1")


@pytest.mark.parametrize("N,K,B", [(4096, 4096, 1), (4096, 4096, 4), (4096, 4096, 8), (1000, 1152, 3),
                                   (4097, 2176, 8), (100, 11008, 2)])
def test_tuned_dispatch_parity_and_reproducibility(N, K, B):
    W, x = synth.gemv_case(N, K, B, seed=7 * N + K + B)
    s, c = O.pack_ref_fast(W)
    sd, cd, xd = words_dev(s), fp16_dev(c), bf16_dev(x)
    first = ops.w1_gemv(sd, cd, xd)          # times the candidates, then launches the winner
    second = ops.w1_gemv(sd, cd, xd)         # cached choice
    third = ops.w1_gemv(sd, cd, xd, static_weights=True)
    assert ops.sync_status() == _lib.W1_OK
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s, c, K)
    for y in (first, second, third):
        assert_within(y.cpu().numpy().astype(np.float64), y_ref, bound, what=f"tuned {N}x{K} B={B}")
    assert np.array_equal(first.cpu().numpy(), second.cpu().numpy())


def test_autotune_off_uses_the_rule(knob):
    knob("gemv_autotune", "0")
    N, K, B = 300, 1024, 5
    W, x = synth.gemv_case(N, K, B, seed=11)
    s, c = O.pack_ref_fast(W)
    y = ops.w1_gemv(words_dev(s), fp16_dev(c), bf16_dev(x))
    assert ops.sync_status() == _lib.W1_OK
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s, c, K)
    assert_within(y.cpu().numpy().astype(np.float64), y_ref, bound, what="rule dispatch")


@pytest.mark.parametrize("name", ["direct/1", "direct/2", "direct16/1", "direct16/4", "tc/0", "ring/0"])
def test_pinned_choice_is_used_and_reported(name):
    """w1_gemv_set_choice replaces the timed choice: later calls report and run it."""
    N, K, B = 2056, 2048, 4
    W, x = synth.gemv_case(N, K, B, seed=19)
    s, c = O.pack_ref_fast(W)
    sd, cd, xd = words_dev(s), fp16_dev(c), bf16_dev(x)
    ops.gemv_set_choice(N, K, B, name)
    y = ops.w1_gemv(sd, cd, xd)
    assert ops.sync_status() == _lib.W1_OK
    assert ops.gemv_choice(N, K, B) == name
    y_ref, bound = O.matmul_ref(O.bf16_bits_to_f64(x), s, c, K)
    assert_within(y.cpu().numpy().astype(np.float64), y_ref, bound, what=f"pinned {name}")
    assert ops.gemv_choice(N, K, B, static_weights=True) in ("", name)  # the flag keys its own entry

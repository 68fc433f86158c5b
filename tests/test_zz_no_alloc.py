"""dbf_apply_noalloc: the DBF chain for callers that cannot allocate device memory.

Such callers (code inside a framework that owns all device memory, or a
decode loop that must not synchronise on an allocation) get an entry point
whose scratch is a fixed array inside the library.  This test calls it
through the C ABI twice in a row and checks each result against the regular
dbf_apply (which takes a caller-allocated workspace), within the same
1e-3 * |a_i| sum_j |mid_j h_j| bound the other DBF tests use.  It lives in a
file of its own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import _lib, ops, synth
from gpu_helpers import assert_within, bf16_dev, fp16_dev, words_dev

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    lib = _lib.load()
    # B = 20: three groups of up to 8 rows through the one static array in
    # sequence (the barrier count and the intermediate are reused)
    for seed, (m, r, n, B) in [(0, (4096, 4096, 4096, 8)), (1, (1000, 640, 1152, 5)), (2, (1000, 640, 1152, 20))]:
        case = synth.dbf_case(m=m, r=r, n=n, B=B, seed=40 + seed)
        a, B1, mid, B2, b, x = case
        dv = [fp16_dev(a), words_dev(B1), fp16_dev(mid), words_dev(B2), fp16_dev(b), bf16_dev(x)]
        ref = O.dbf_ref(a, B1, mid, B2, b, O.bf16_bits_to_f64(x), m, r, n)
        y_ws = ops.dbf_apply(*dv)
        assert ops.sync_status() == _lib.W1_OK
        expected = y_ws.cpu().numpy().astype(np.float64)
        for call in range(2):
            y = torch.full((B, m), float("nan"), dtype=torch.float32, device="cuda")
            st = lib.dbf_apply_noalloc(*[t.data_ptr() for t in dv[:5]], m, r, n, dv[5].data_ptr(), B,
                                       y.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert st == _lib.W1_OK
            assert ops.sync_status() == _lib.W1_OK
            got = y.cpu().numpy().astype(np.float64)
            assert_within(got, expected, ref["bound"], what=f"noalloc call {call} vs dbf_apply")
            assert_within(got, ref["y"], ref["bound"], what=f"noalloc call {call} vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = _lib.load()
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    st = lib.dbf_apply_noalloc(p, p, p, p, p, 128, 16384 + 128, 128, p, 1, p, None)
    assert st == _lib.W1_ERR_TOO_LARGE

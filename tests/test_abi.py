"""The C-ABI library builds, loads and exports every symbol include/w1.h declares.

Host-side argument checks are exercised without a GPU (no compute call is made:
every call here is rejected before any CUDA work).
"""
import ctypes
import os
import re

import pytest

from pack_sign_g128_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "w1.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:w1|dbf)_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declares_the_calls():
    fns = declared_functions()
    for name in ("w1_pack", "w1_gemv", "w1_gemm", "w1_status_string", "w1_sync_status"):
        assert name in fns


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings(lib):
    for code, name in _lib.W1_STATUS.items():
        assert lib.w1_status_string(code).decode().startswith(name)


def test_knobs_accept_their_words_and_reject_the_rest(lib):
    ok = [("gemv_path", "direct"), ("gemv_path", "direct16"), ("gemv_path", "tc"), ("gemv_path", "ring"),
          ("gemv_path", "flat"), ("gemv_split", "4"), ("gemv_autotune", "0"), ("moe_path", "tiles"),
          ("moe_path", "decode"), ("moe_path", "grouped"), ("dbf_path", "fused"), ("dbf_path", "twostep"), ("dbf_warps", "16"),
          ("dbf_rank_split", "4"), ("sg_bm", "256"), ("dbf_core", "direct"), ("sg_exp", "8"), ("sg_a", "tmem"),
          ("sg_a", "smem"), ("moe_tw", "4"),
          ("verbose", "1")]
    try:
        for name, value in ok:
            assert lib.w1_set_knob(name.encode(), value.encode()) == _lib.W1_OK, (name, value)
        assert lib.w1_set_knob(b"gemv_path", b"fast") == _lib.W1_ERR_SHAPE
        assert lib.w1_set_knob(b"gemv_split", b"-1") == _lib.W1_ERR_SHAPE
        assert lib.w1_set_knob(b"no_such_knob", b"1") == _lib.W1_ERR_SHAPE
        assert lib.w1_set_knob(None, b"1") == _lib.W1_ERR_NULL
    finally:
        for name in {n for n, _ in ok}:
            assert lib.w1_set_knob(name.encode(), None) == _lib.W1_OK


def test_host_side_argument_errors(lib):
    good = ctypes.c_void_p(1 << 20)     # never dereferenced: calls fail validation first
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lib.w1_pack(None, 4, 128, good, good, None) == _lib.W1_ERR_NULL
    assert lib.w1_pack(good, 4, 100, good, good, None) == _lib.W1_ERR_SHAPE
    assert lib.w1_pack(good, 0, 128, good, good, None) == _lib.W1_ERR_SHAPE
    assert lib.w1_pack(odd, 4, 128, good, good, None) == _lib.W1_ERR_ALIGN
    assert lib.w1_gemv(good, good, 16, 128, good, 9, good, None) == _lib.W1_ERR_SHAPE
    assert lib.w1_gemv(good, good, 16, 128, good, 0, good, None) == _lib.W1_ERR_SHAPE
    assert lib.w1_gemv(good, None, 16, 128, good, 1, good, None) == _lib.W1_ERR_NULL
    assert lib.w1_gemv(good, good, 16, 130, good, 1, good, None) == _lib.W1_ERR_SHAPE
    assert lib.w1_gemv(good, good, 16, 128, odd, 1, good, None) == _lib.W1_ERR_ALIGN
    buf = ctypes.create_string_buffer(32)
    assert lib.w1_gemv_choice(16, 128, 1, 0, None, 32) == _lib.W1_ERR_NULL
    assert lib.w1_gemv_choice(16, 100, 1, 0, buf, 32) == _lib.W1_ERR_SHAPE
    assert lib.w1_gemv_choice(16, 128, 9, 0, buf, 32) == _lib.W1_ERR_SHAPE
    assert lib.w1_gemv_set_choice(16, 128, 1, 0, None) == _lib.W1_ERR_NULL
    for bad in (b"direct", b"direct/3", b"direct/0", b"direct32/1", b"tc/x", b"gemv/1", b"direct/1 ", b""):
        assert lib.w1_gemv_set_choice(16, 128, 1, 0, bad) == _lib.W1_ERR_SHAPE, bad
    assert lib.w1_gemv_set_choice(16, 100, 1, 0, b"direct/1") == _lib.W1_ERR_SHAPE
    assert lib.w1_gemv_set_choice(16, 128, 9, 0, b"direct/1") == _lib.W1_ERR_SHAPE
    assert lib.w1_gemv_set_choice(16, 128, 1, 2, b"direct/1") == _lib.W1_ERR_SHAPE
    assert lib.w1_gemm(good, good, 16, 128, good, 0, good, good, 1 << 30, None) == _lib.W1_ERR_SHAPE
    assert lib.w1_gemm(good, good, 16, 128, good, 4, None, good, 1 << 30, None) == _lib.W1_ERR_NULL
    need = lib.w1_gemm_workspace_size(4, 128)
    assert need >= 4 * 128 * 2 + 4
    assert lib.w1_gemm(good, good, 16, 128, good, 4, good, good, need - 1, None) == _lib.W1_ERR_WORKSPACE
    assert lib.w1_gemm(good, good, 16, 128, good, 4, good, None, need, None) == _lib.W1_ERR_WORKSPACE
    assert lib.w1_gemm(good, good, 16, 128, good, 4, good, odd, need, None) == _lib.W1_ERR_ALIGN
    assert lib.w1_gemm_workspace_size(4, 100) == 0


def test_dbf_host_side_argument_errors(lib):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    args = [good] * 5
    assert lib.dbf_apply(None, *args[1:], 64, 128, 128, good, 1, good, good, 1 << 20, None) == _lib.W1_ERR_NULL
    assert lib.dbf_apply(*args, 64, 100, 128, good, 1, good, good, 1 << 20, None) == _lib.W1_ERR_SHAPE
    assert lib.dbf_apply(*args, 64, 128, 128, good, 0, good, good, 1 << 20, None) == _lib.W1_ERR_SHAPE
    assert lib.dbf_apply(*args, 64, 128, 128, good, 1, good, None, 1 << 20, None) == _lib.W1_ERR_WORKSPACE
    assert lib.dbf_apply(*args, 64, 128, 128, good, 1, good, good, 16, None) == _lib.W1_ERR_WORKSPACE
    assert lib.dbf_apply(*args, 64, 128, 128, odd, 1, good, good, 1 << 20, None) == _lib.W1_ERR_ALIGN
    assert lib.dbf_workspace_size(64, 128, 128, 1) >= 256 + 4 * 128
    assert lib.dbf_workspace_size(0, 128, 128, 1) == 0


def test_moe_host_side_argument_errors(lib):
    good = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 30)
    base = [good, good, 16, 256, 128, 8, 2] + [good] * 7
    n = lib.w1_moe_workspace_size(16, 256, 128, 8, 2)
    assert n > 0
    assert lib.w1_moe_workspace_size(16, 256, 128, 8, 9) == 0          # top_k > E
    assert lib.w1_moe_workspace_size(16, 256, 128, 300, 2) == 0        # E > 256
    assert lib.w1_moe_grouped(*base, ws, n - 1, None) == _lib.W1_ERR_WORKSPACE
    bad = list(base)
    bad[3] = 200                                                       # H not a multiple of 128
    assert lib.w1_moe_grouped(*bad, ws, n, None) == _lib.W1_ERR_SHAPE
    bad = list(base)
    bad[0] = None
    assert lib.w1_moe_grouped(*bad, ws, n, None) == _lib.W1_ERR_NULL
    assert lib.w1_moe_grouped(*base, ctypes.c_void_p((1 << 30) + 256), n, None) == _lib.W1_ERR_ALIGN


def test_okt_host_side_argument_errors(lib):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    rot = lib.w1_okt_rotate
    assert rot(None, 64, good, 64, good, 1, good, None) == _lib.W1_ERR_NULL
    assert rot(good, 64, good, 64, good, 1, None, None) == _lib.W1_ERR_NULL
    assert rot(good, 64, good, 32, good, 1, good, None) != _lib.W1_ERR_NULL   # n1 n2 = 2048: a valid K
    assert rot(good, 3, good, 10, good, 1, good, None) == _lib.W1_ERR_SHAPE    # K = 30, not a multiple of 128
    assert rot(good, 16, good, 256, good, 1, good, None) == _lib.W1_ERR_SHAPE  # n2 > 128
    assert rot(good, 2048, good, 1, good, 1, good, None) == _lib.W1_ERR_SHAPE  # n1 > 1024
    assert rot(good, 1024, good, 128, good, 1, good, None) == _lib.W1_ERR_SHAPE  # K > 65536
    assert rot(good, 0, good, 128, good, 1, good, None) == _lib.W1_ERR_SHAPE
    assert rot(good, 64, good, 64, good, 0, good, None) == _lib.W1_ERR_SHAPE
    assert rot(good, 64, good, 64, good, 65536, good, None) == _lib.W1_ERR_SHAPE
    assert rot(odd, 64, good, 64, good, 1, good, None) == _lib.W1_ERR_ALIGN
    assert rot(good, 64, good, 64, good, 1, odd, None) == _lib.W1_ERR_ALIGN
    g = lib.w1_okt_gemv
    assert g(good, good, 16, 4096, good, 64, good, 64, good, 1, None, good, 0, None) == _lib.W1_ERR_NULL
    assert g(good, good, 16, 4096, good, 64, good, 32, good, 1, good, good, 0, None) == _lib.W1_ERR_SHAPE  # 64*32 != K
    assert g(good, good, 16, 4096, good, 64, good, 64, good, 9, good, good, 0, None) == _lib.W1_ERR_SHAPE  # B > 8
    assert g(good, good, 16, 4096, good, 64, good, 64, good, 1, good, good, 2, None) == _lib.W1_ERR_SHAPE  # flag
    assert g(good, good, 0, 4096, good, 64, good, 64, good, 1, good, good, 0, None) == _lib.W1_ERR_SHAPE
    assert g(good, good, 16, 4096, good, 64, good, 64, good, 1, good, odd, 0, None) == _lib.W1_ERR_ALIGN


def test_measure_host_side_argument_errors(lib):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    ws = lib.w1_measure_workspace_size(256, 512)
    assert ws > 0 and lib.w1_measure_workspace_size(0, 512) == 0
    assert lib.w1_measure_workspace_size(4096, 4096) >= 8 * (4096 + 65 * 4096)
    res = lib.w1_residual
    assert res(None, 256, 512, good, good, None, good, good, ws, None) == _lib.W1_ERR_NULL
    assert res(good, 256, 500, good, good, None, good, good, ws, None) == _lib.W1_ERR_SHAPE
    assert res(good, 0, 512, good, good, None, good, good, ws, None) == _lib.W1_ERR_SHAPE
    assert res(good, 256, 512, good, good, None, good, None, ws, None) == _lib.W1_ERR_WORKSPACE
    assert res(good, 256, 512, good, good, None, good, good, ws - 1, None) == _lib.W1_ERR_WORKSPACE
    assert res(good, 256, 512, good, good, odd, good, good, ws, None) == _lib.W1_ERR_ALIGN
    d = lib.dbf_residual
    wsd = lib.dbf_residual_workspace_size(256, 128, 384)
    assert wsd >= 2 * 384 * 128 + 4 * 384 * 256 and lib.dbf_residual_workspace_size(256, 100, 384) == 0
    args = [good] * 6
    assert d(None, *args[1:], 256, 128, 384, None, good, good, wsd, None) == _lib.W1_ERR_NULL
    assert d(*args, 256, 100, 384, None, good, good, wsd, None) == _lib.W1_ERR_SHAPE
    assert d(*args, 256 * 128, 128, 256 * 128, None, good, good, 1 << 40, None) == _lib.W1_ERR_SHAPE  # too many tiles
    assert d(*args, 256, 128, 384, None, good, good, wsd - 8, None) == _lib.W1_ERR_WORKSPACE
    assert d(*args, 256, 128, 384, None, odd, good, wsd, None) == _lib.W1_ERR_ALIGN  # sums not 8-aligned
    pi = lib.w1_power_iteration
    assert pi(None, 64, 64, good, 32, good, good, ws, None) == _lib.W1_ERR_NULL
    assert pi(good, 64, 66, good, 32, good, good, ws, None) == _lib.W1_ERR_SHAPE
    assert pi(good, 64, 64, good, -1, good, good, ws, None) == _lib.W1_ERR_SHAPE
    assert pi(good, 64, 64, good, 32, good, None, ws, None) == _lib.W1_ERR_WORKSPACE
    assert pi(odd, 64, 64, good, 32, good, good, ws, None) == _lib.W1_ERR_ALIGN


def test_stream_probe_host_side_argument_errors(lib):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    f = lib.w1_stream_probe
    assert f(None, 1024, None, 0, 148, 0, good, None) == _lib.W1_ERR_NULL
    assert f(good, 1024, None, 16, 148, 0, good, None) == _lib.W1_ERR_NULL   # b missing for bbytes > 0
    assert f(good, 1024, good, 16, 148, 0, None, None) == _lib.W1_ERR_NULL
    assert f(good, 0, None, 0, 148, 0, good, None) == _lib.W1_ERR_SHAPE
    assert f(good, 1000, None, 0, 148, 0, good, None) == _lib.W1_ERR_SHAPE
    assert f(good, 1024, good, 8, 148, 0, good, None) == _lib.W1_ERR_SHAPE
    assert f(good, 1024, None, 0, 0, 0, good, None) == _lib.W1_ERR_SHAPE
    assert f(good, 1024, None, 0, 148, 2, good, None) == _lib.W1_ERR_SHAPE
    assert f(odd, 1024, None, 0, 148, 0, good, None) == _lib.W1_ERR_ALIGN
    assert f(good, 1024, good, 16, 148, 1, odd, None) == _lib.W1_ERR_ALIGN


def test_reproject_host_side_argument_errors(lib):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    ws = lib.dbf_reproject_mid_workspace_size(256, 128, 384)
    assert ws >= 8 * 128 * 128
    assert lib.dbf_reproject_mid_workspace_size(256, 100, 384) == 0
    assert lib.dbf_reproject_mid_workspace_size(256, 16384 + 128, 384) == 0
    assert lib.dbf_reproject_mid_workspace_size(0, 128, 384) == 0
    f = lib.dbf_reproject_mid
    ops5 = [good] * 5

    def call(*, W=good, m=256, r=128, n=384, it=50, tol=1e-13, mid=good, mid64=None, info=None, wsp=good, wsb=ws):
        return f(W, *ops5[1:], m, r, n, it, tol, mid, mid64, info, wsp, wsb, None)

    assert call(W=None) == _lib.W1_ERR_NULL
    assert call(mid=None) == _lib.W1_ERR_NULL
    assert call(r=100) == _lib.W1_ERR_SHAPE
    assert call(n=200) == _lib.W1_ERR_SHAPE
    assert call(m=0) == _lib.W1_ERR_SHAPE
    assert call(r=16384 + 128) == _lib.W1_ERR_SHAPE
    assert call(it=-1) == _lib.W1_ERR_SHAPE
    assert call(tol=-1.0) == _lib.W1_ERR_SHAPE
    assert call(tol=float("nan")) == _lib.W1_ERR_SHAPE
    assert call(wsp=None) == _lib.W1_ERR_WORKSPACE
    assert call(wsb=ws - 1) == _lib.W1_ERR_WORKSPACE
    assert call(W=odd) == _lib.W1_ERR_ALIGN
    assert call(mid64=odd) == _lib.W1_ERR_ALIGN
    assert call(info=ctypes.c_void_p((1 << 20) + 2)) == _lib.W1_ERR_ALIGN


def test_binding_shape_checks_run_before_any_device_work():
    """The torch binding rejects mismatched shapes before marshalling pointers
    (CPU tensors: the shape error must come first, not the CUDA-tensor check)."""
    import torch
    from pack_sign_g128_b200 import ops
    x = torch.zeros((1, 4096), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="is not K"):
        ops.w1_okt_rotate(torch.zeros((64, 64)), torch.zeros((32, 32)), x)
    with pytest.raises(ValueError, match="square"):
        ops.w1_okt_rotate(torch.zeros((64, 32)), torch.zeros((64, 64)), x)
    signs = torch.zeros((16, 64), dtype=torch.int32)
    scales = torch.zeros((16, 16), dtype=torch.float16)
    with pytest.raises(ValueError, match="columns, the packed weights"):
        ops.w1_okt_gemv(signs, scales, torch.zeros((64, 64)), torch.zeros((64, 64)), x)
    with pytest.raises(ValueError, match="do not match"):
        ops.w1_residual(torch.zeros((16, 4096)), signs, scales)
    with pytest.raises(ValueError, match="entries"):
        ops.w1_power_iteration(torch.zeros((8, 16)), torch.zeros(12))
    h16 = lambda k: torch.zeros(k, dtype=torch.float16)
    w = lambda r, c: torch.zeros((r, c), dtype=torch.int32)
    with pytest.raises(ValueError, match="DBF operands"):
        ops.dbf_residual(torch.zeros((128, 256)), h16(128), w(128, 4), h16(128), w(128, 4), h16(256))
    with pytest.raises(ValueError, match="CUDA"):  # well-formed CPU tensors reach the device check
        ops.w1_power_iteration(torch.zeros((8, 16)), torch.zeros(16))

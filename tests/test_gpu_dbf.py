"""dbf_apply on the GPU vs the fp64 oracle chain.

Every test runs with each small-batch chain form -- the fused chain kernel and
two launches of a GEMV core (the dbf_path knob; groups of 1-4 rows take the
register-fed core, or the direct core with dbf_core=direct) -- forced to 8
and to 16 warps per CTA (the dbf_warps knob).  Batches of 64 and more take the
tensor-core path either way."""
import functools

import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import assert_within, bf16_dev, fp16_dev, words_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["fused8", "fused16", "twostep8", "twostep16", "twostepdirect8"])
def dbf_path(request, knob):
    form, warps = (request.param[:-2], request.param[-2:]) if request.param.endswith("16") else (request.param[:-1], "8")
    if form == "twostepdirect":
        form = "twostep"
        knob("dbf_core", "direct")  # the direct GEMV core for 1-4 rows too
    knob("dbf_path", form)
    knob("dbf_warps", warps)
    return request.param


def run_dbf(case, ws=None):
    a, B1, mid, B2, b, x = case
    dv = [fp16_dev(a), words_dev(B1), fp16_dev(mid), words_dev(B2), fp16_dev(b), bf16_dev(x)]
    m, r, n, B = a.shape[0], mid.shape[0], b.shape[0], x.shape[0]
    if ws is None:
        ws = ops.dbf_workspace(m, r, n, B)
    y = ops.dbf_apply(*dv, workspace=ws)
    st = ops.sync_status()
    return y.cpu().numpy().astype(np.float64), ws, st


def check(case, what, stage1=True):
    a, B1, mid, B2, b, x = case
    m, r, n, B = a.shape[0], mid.shape[0], b.shape[0], x.shape[0]
    y, ws, st = run_dbf(case)
    assert st == _lib.W1_OK
    ref = O.dbf_ref(a, B1, mid, B2, b, O.bf16_bits_to_f64(x), m, r, n)
    assert_within(y, ref["y"], ref["bound"], what=what)
    if stage1 and B < 64:
        # workspace holds mid * h of the last group of <= 8 batch rows
        b0 = ((B - 1) // 8) * 8
        nb = B - b0
        hw = ws[256:256 + 4 * nb * r].view(torch.float32).cpu().numpy().reshape(nb, r).astype(np.float64)
        midv = O.fp16_bits_to_f64(mid)
        assert_within(hw, ref["h_scaled"][b0:], np.abs(midv)[None, :] * ref["h_bound"][b0:], what=what + " stage 1")
    return y


@pytest.mark.parametrize("B", [1, 8])
def test_dbf_config(B):
    check(synth.dbf_case(B=B), f"4096^3 B={B}")


def _tensor_path_once(dbf_path):
    if dbf_path != "fused8":
        pytest.skip("batches of 64 and more take the tensor-core path under every small-batch form")


def test_dbf_config_batch512(dbf_path):
    _tensor_path_once(dbf_path)
    check(synth.dbf_case(B=512), "4096^3 B=512")


@pytest.mark.parametrize("m,r,n,B", [(300, 384, 256, 64), (4096, 1024, 2048, 200), (129, 128, 128, 65)])
def test_dbf_tensor_path_ragged(m, r, n, B, dbf_path):
    _tensor_path_once(dbf_path)
    check(synth.dbf_case(m=m, r=r, n=n, B=B, seed=m + r + n + B), f"tensor path {m}x{r}x{n} B={B}")


def test_dbf_tensor_path_extreme_scales(dbf_path):
    """Inputs spanning many binades: the per-row fp16 scalings must not overflow."""
    _tensor_path_once(dbf_path)
    a, B1, mid, B2, b, x = synth.dbf_case(m=512, r=512, n=512, B=96, seed=77)
    xf = synth.normal_f32(synth.rng(78), (96, 512))
    xf[0] *= 1e30
    xf[1] *= 1e-30
    xf[2, :] = 0.0
    check((a, B1, mid, B2, b, synth.f32_to_bf16_bits(xf)), "tensor path extreme x")


@pytest.mark.parametrize("m,r,n,B", [(200, 384, 256, 3), (1, 128, 128, 1), (1000, 640, 1152, 5),
                                     (4096, 1024, 2048, 2), (33, 256, 128, 7),
                                     # long K in either product: the GEMV cores split K over a cluster
                                     (128, 512, 32768, 1), (128, 32768, 256, 2), (300, 12288, 12288, 1),
                                     (300, 512, 32768, 3), (128, 32768, 256, 4), (1000, 640, 1152, 4)])
def test_dbf_ragged(m, r, n, B):
    check(synth.dbf_case(m=m, r=r, n=n, B=B, seed=m + r + n + B), f"{m}x{r}x{n} B={B}")


def _sylvester_words(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return O.pack_bits_lsb_first((H < 0).astype(np.uint8))


def test_dbf_hadamard_closed_form():
    n = 1024
    Hw = _sylvester_words(n)
    ones = np.full(n, 0x3C00, np.uint16)
    x = synth.activations_bf16(synth.rng(5), 4, n)
    y, _, st = run_dbf((ones, Hw, ones, Hw, ones, x))
    assert st == _lib.W1_OK
    exact = n * O.bf16_bits_to_f64(x)
    assert np.max(np.abs(y - exact)) <= 1e-5 * np.max(np.abs(exact))


def test_dbf_workspace_reuse_and_determinism():
    case = synth.dbf_case(m=512, r=1024, n=768, B=4, seed=9)
    y1, ws, st = run_dbf(case)
    assert st == _lib.W1_OK
    assert int(ws[:4].view(torch.int32).item()) == 0        # barrier count back at zero
    y2, _, st = run_dbf(case, ws)
    assert st == _lib.W1_OK
    assert np.array_equal(y1, y2)


def test_dbf_barrier_timeout_reports_status(dbf_path):
    """A barrier count that no arrival can complete: every CTA's bounded wait
    runs out, the call reports W1_ERR_TIMEOUT and the context stays usable."""
    if dbf_path.startswith("twostep"):
        pytest.skip("the two-launch form has no grid barrier")
    case = synth.dbf_case(m=256, r=256, n=256, B=1, seed=10)
    a, B1, mid, B2, b, x = case
    ws = ops.dbf_workspace(256, 256, 256, 1)
    ws[:4].view(torch.int32).fill_(-(2 ** 31))
    _, _, st = run_dbf(case, ws)
    assert st == _lib.W1_ERR_TIMEOUT
    ws.zero_()
    y, _, st = run_dbf(case, ws)
    assert st == _lib.W1_OK
    ref = O.dbf_ref(a, B1, mid, B2, b, O.bf16_bits_to_f64(x), 256, 256, 256)
    assert_within(y, ref["y"], ref["bound"], what="after timeout")


@pytest.mark.parametrize("split", [1, 2, 4, 8])
@pytest.mark.parametrize("m,r,n,B", [(4096, 4096, 4096, 1), (1000, 640, 1152, 5), (512, 2048, 256, 8)])
def test_dbf_twostep_rank_split(m, r, n, B, split, dbf_path, knob):
    """The two-launch form with r split over 1-8 CTAs of a cluster in U . h
    (DBF post, section 5 item 5, "Split rank"); splits whose plan does not
    fit the shape report W1_ERR_UNSUPPORTED before any launch."""
    if dbf_path != "twostep8":
        pytest.skip("one form is enough: the split applies to the two-launch chain")
    knob("dbf_rank_split", str(split))
    case = synth.dbf_case(m=m, r=r, n=n, B=B, seed=m + r + n + B + split)
    try:
        check(case, f"{m}x{r}x{n} B={B} rank split {split}")
    except _lib.W1Error as e:
        assert e.status == _lib.W1_ERR_UNSUPPORTED and split > 1

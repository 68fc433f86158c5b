"""w1_moe_grouped on the GPU vs the fp64 oracle: routing exact, every stage
within its bound, end to end with the bf16 intermediate propagated.  Batches
of up to 8 tokens take the decode path (per-route products), 9 to 16 the
decode path grouped by expert (one product per touched expert, its routes as
the batch rows), larger ones the expert-sorted tile pipeline; the moe_path
knob forces any of them."""
import functools

import numpy as np
import pytest
import torch

from oracle import w1_oracle as O
from pack_sign_g128_b200 import ops, synth, _lib
from gpu_helpers import assert_within, bf16_dev, fp16_dev, words_dev, f32_dev, bits16_host

pytestmark = pytest.mark.gpu


def _pack_experts(Wt):
    E, rows, K = Wt.shape
    s, c = O.pack_ref_fast(Wt.reshape(E * rows, K))
    return s.reshape(E, rows, K // 32), c.reshape(E, rows, K // 128)


def shared_logits(T, E, K, seed):
    """Every token prefers the same K experts (decreasing with the expert
    index), so each of them is routed by all T tokens."""
    g = np.random.default_rng(seed)
    L = g.normal(size=(T, E)).astype(np.float32) - 8.0
    L[:, :K] = np.float32(4.0) + np.linspace(1.0, 0.0, K, dtype=np.float32)[None, :] + \
        np.float32(0.01) * g.normal(size=(T, K)).astype(np.float32)
    return L


def tied_logits(T, E, seed):
    """Router logits full of exact ties: all-zero rows, constant rows, rows of
    values that each appear twice, and rows whose top value is unique but
    whose next values tie.  Ties in the logits are ties in the probabilities,
    which the routing breaks toward the lower expert index."""
    g = np.random.default_rng(seed)
    L = np.empty((T, E), dtype=np.float32)
    for t in range(T):
        kind = t % 4
        if kind == 0:
            L[t] = 0.0
        elif kind == 1:
            L[t] = np.float32(g.normal())
        elif kind == 2:
            vals = g.normal(size=(E + 1) // 2).astype(np.float32)
            L[t] = np.repeat(vals, 2)[:E][g.permutation(E)]
        else:
            L[t] = g.normal(size=E).astype(np.float32) - 4.0
            L[t, g.integers(0, E)] = 3.0
            L[t, g.choice(E, size=min(E - 1, 6), replace=False)[:5]] = 1.25
    return L


@functools.lru_cache(maxsize=None)
def moe_case(T, H, I, E, seed, skew=0.0, ties=False, shared_k=0):
    x, logits, gate, up, down = synth.moe_case(T=T, H=H, I=I, E=E, seed=seed)
    if skew:
        logits = logits + np.float32(skew) * np.linspace(1.0, 0.0, E, dtype=np.float32)[None, :]
    if ties:
        logits = tied_logits(T, E, seed)
    if shared_k:
        logits = shared_logits(T, E, shared_k, seed)
    return x, logits, _pack_experts(gate), _pack_experts(up), _pack_experts(down)


def run_and_check(T, H, I, E, K, seed, skew=0.0, ties=False, shared=False):
    x, logits, G, U, D = moe_case(T, H, I, E, seed, skew, ties, K if shared else 0)
    dev = lambda p: (words_dev(p[0].reshape(-1, p[0].shape[-1])).view(p[0].shape[0], p[0].shape[1], -1),
                     fp16_dev(p[1].reshape(-1, p[1].shape[-1])).view(p[1].shape[0], p[1].shape[1], -1))
    ws = ops.moe_workspace(T, H, I, E, K)
    out = ops.w1_moe_grouped(bf16_dev(x), f32_dev(logits), dev(G), dev(U), dev(D), K, workspace=ws)
    assert ops.sync_status() == _lib.W1_OK
    out = out.cpu().numpy().astype(np.float64)
    v = ops.moe_workspace_views(ws, T, H, I, E, K)
    xf = O.bf16_bits_to_f64(x)
    ref = O.moe_ref(xf, logits, G, U, D, H, I, E, K)

    # 1. routing: identical experts, fp32 weights
    ids = v["ids"].cpu().numpy().reshape(T, K)
    assert np.array_equal(ids, ref["ids"])
    w = v["wts"].cpu().numpy().reshape(T, K).astype(np.float64)
    assert np.all(np.abs(w - ref["w"]) <= 2e-6 * ref["w"] + 1e-9)

    # 2. gate/up stage: h = bf16(silu(g) u); bound from the g, u bounds + bf16 rounding
    pos = v["pos"].cpu().numpy().reshape(T, K)
    hs = O.bf16_bits_to_f64(v["h"].cpu().view(torch.int16).numpy().view(np.uint16))
    h_gpu = hs[pos]                                   # [T, K, I]
    g, u = ref["g"], ref["u"]
    sg = 1.0 / (1.0 + np.exp(-g))
    silu = g * sg
    dsilu = np.abs(sg * (1.0 + g * (1.0 - sg)))
    h_lim = 2.0 ** -8 * np.abs(ref["h"]) + 1e-3 * (dsilu * ref["g_bound"] * np.abs(u) + np.abs(silu) * ref["u_bound"])
    err = np.abs(h_gpu - ref["h"])
    assert np.all(err <= h_lim + 1e-30), f"h stage: {int((err > h_lim).sum())} elements out"

    # 3. down + combine, fed the device's own h
    ref2 = O.moe_ref(xf, logits, G, U, D, H, I, E, K, h_override=h_gpu)
    w_err = np.abs(w - ref["w"])                      # fp32 route weights
    d_abs = np.abs(ref2["d"])
    lim = 1e-3 * ref2["out_bound"] + (w_err[:, :, None] * d_abs).sum(1) + 1e-30
    assert_within(out, ref2["out"], lim / 1e-3, what=f"MoE T={T} E={E} k={K} down stage")

    # 4. end to end against the unrounded chain, the h error propagated exactly
    dh = np.abs(h_gpu - ref["h"])
    prop = np.zeros((T, H))
    for e in range(E):
        sel = np.argwhere(ref["ids"] == e)
        if sel.size == 0:
            continue
        Dabs = np.abs(O.dequant_ref(D[0][e], D[1][e], I))
        prop[sel[:, 0]] += ref["w"][sel[:, 0], sel[:, 1]][:, None] * (dh[sel[:, 0], sel[:, 1]] @ Dabs.T)
    lim_e2e = 1e-3 * ref["out_bound"] + prop * 1.001 + (w_err[:, :, None] * np.abs(ref["d"])).sum(1) + 1e-30
    assert_within(out, ref["out"], lim_e2e / 1e-3, what="MoE end to end")
    return out


def test_moe_config_olmoe_like():
    run_and_check(512, 2048, 1024, 64, 8, synth.SEEDS["moe"])


@pytest.mark.parametrize("T,H,I,E,K,seed,skew", [
    (16, 256, 128, 8, 2, 1, 0.0),      # tiny, ragged tiles
    (1, 2048, 1024, 64, 8, 2, 0.0),    # one token: decode regime (per-route products)
    (4, 2048, 1024, 64, 8, 5, 0.0),    # decode regime
    (8, 512, 384, 16, 4, 6, 0.0),      # decode regime, experts shared by tokens
    (300, 384, 256, 16, 4, 3, 6.0),    # skewed routing: empty experts, multi-tile experts
    (130, 512, 384, 32, 8, 4, 0.0),
])
def test_moe_small_and_skewed(T, H, I, E, K, seed, skew):
    run_and_check(T, H, I, E, K, seed, skew)


@pytest.mark.parametrize("path,T", [("tiles", 3), ("decode", 20)])
def test_moe_forced_path(path, T, knob):
    """Each path outside its default regime: the tile pipeline for a few
    tokens, the per-route decode products for a larger batch."""
    knob("moe_path", path)
    run_and_check(T, 512, 256, 16, 4, 7)


@pytest.mark.parametrize("tw", [2, 4])
@pytest.mark.parametrize("T,H,I", [(3, 512, 384), (8, 2048, 1024)])
def test_moe_decode_gateup_rows_per_warp(tw, T, H, I, knob):
    """The per-route gate/up kernel with 16 or 32 rows of each matrix per warp
    (64 or 128 per CTA; I = 384 leaves a ragged last block of 128)."""
    knob("moe_path", "decode")
    knob("moe_tw", tw)
    run_and_check(T, H, I, 16, 4, 12 + tw)


@pytest.mark.parametrize("T", [64, 4])
def test_moe_is_deterministic(T):
    H, I, E, K = 512, 256, 16, 4
    x, logits, G, U, D = moe_case(T, H, I, E, 7)
    dev = lambda p: (words_dev(p[0].reshape(-1, p[0].shape[-1])).view(p[0].shape[0], p[0].shape[1], -1),
                     fp16_dev(p[1].reshape(-1, p[1].shape[-1])).view(p[1].shape[0], p[1].shape[1], -1))
    args = (bf16_dev(x), f32_dev(logits), dev(G), dev(U), dev(D), K)
    a = ops.w1_moe_grouped(*args).cpu().numpy()
    b = ops.w1_moe_grouped(*args).cpu().numpy()
    assert ops.sync_status() == _lib.W1_OK
    assert np.array_equal(a, b)


@pytest.mark.parametrize("T,H,I,E,K,seed,skew,shared", [
    (1, 2048, 1024, 64, 8, 2, 0.0, False),    # one token: every count is 1
    (4, 2048, 1024, 64, 8, 5, 0.0, False),
    (8, 2048, 1024, 64, 8, 11, 0.0, False),   # the OLMoE-like layer at 8 tokens
    (8, 512, 384, 16, 4, 6, 0.0, False),      # experts shared by several tokens
    (16, 512, 256, 16, 4, 12, 0.0, False),    # the largest grouped batch
    (16, 512, 384, 8, 4, 13, 6.0, False),     # skewed: counts above 4 (several batches per expert)
    (16, 384, 256, 16, 4, 14, 0.0, True),     # every token on the same 4 experts: 16 routes each
    (11, 256, 128, 8, 2, 15, 0.0, True),      # 11 routes per expert: batches of 4, 4 and 3
])
def test_moe_grouped_decode(T, H, I, E, K, seed, skew, shared, knob):
    """The decode path grouped by expert (DBF post, section 7 item 1: products
    specialised to the observed expert counts), including forced shared
    experts whose routes exceed one 4-row batch."""
    knob("moe_path", "grouped")
    run_and_check(T, H, I, E, K, seed, skew, shared=shared)


@pytest.mark.parametrize("path", ["default", "tiles", "decode", "grouped"])
@pytest.mark.parametrize("T", [5, 24])
def test_moe_routing_ties_go_to_the_lower_expert(path, T, knob):
    """Exactly tied router logits on both paths (the decode path routes up to
    4 tokens inside its gate/up kernel, more in the router kernel): the expert
    ids must equal the oracle's, whose ties go to the lower expert index."""
    if path != "default":
        knob("moe_path", path)
    run_and_check(T, 512, 256, 16, 4, 9, ties=True)
    run_and_check(min(T, 3), 512, 256, 16, 4, 10, ties=True)

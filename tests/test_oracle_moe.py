"""Pins of the oracle's router, index build and MoE FFN (CPU only).

Independent references: brute-force sorts, scipy's softmax, closed-form
values of a hand-built layer, and a dense all-expert sum computed with numpy
matmuls of the dequantised weights.
"""
import math

import numpy as np
import pytest
from scipy.special import softmax

import oracle
import synth
from synth import workloads
from tests.helpers import oracle_layer, quantize_layer, rel_l2


# ----------------------------------------------------------------- routing
def test_topk_matches_bruteforce_sort():
    z = synth.normal(20, "logits", (50, 16), std=1.0).astype(np.float64)
    z[3, :] = 0.25            # all tied: lower indices first
    z[4, 5] = z[4, 9] = 3.0    # a tie inside the top-K
    for K in (1, 2, 4, 8, 16):
        idx, w = oracle.topk(z, K)
        for t in range(z.shape[0]):
            ref = sorted(range(16), key=lambda e: (-z[t, e], e))[:K]
            assert list(idx[t]) == ref
            p = softmax(z[t])
            assert np.allclose(w[t], p[ref] / p[ref].sum(), rtol=1e-13, atol=0)
        assert np.allclose(w.sum(axis=1), 1.0, rtol=1e-14)
    idx, w = oracle.topk(z, 1)
    assert np.all(w == 1.0)
    idx, w = oracle.topk(z, 16)  # K = E: the weights are the softmax itself
    for t in range(z.shape[0]):
        assert np.allclose(w[t], softmax(z[t])[idx[t]], rtol=1e-13)
    assert list(oracle.topk(z[3:4], 4)[0][0]) == [0, 1, 2, 3]


def test_router_logits_equal_dense_product():
    s = workloads.TINY
    w = workloads.moe_weights(s, seed=0)
    t = quantize_layer(w)
    L = oracle_layer(s, t)
    x, _ = workloads.moe_inputs(s)
    logits, gs = L.router(x)
    wr = oracle.dequant_affine(t["router_p"], t["router_s"], t["router_b"], s.H, 8).astype(np.float64)
    wsg = oracle.dequant_affine(t["sgate_p"], t["sgate_s"], t["sgate_b"], s.H, 8).astype(np.float64)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    assert np.allclose(logits, xf @ wr.T, rtol=1e-12, atol=1e-13)
    assert np.allclose(gs, (xf @ wsg.T)[:, 0], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------- index build
@pytest.mark.parametrize("n_adapters", [0, 1, 4])
def test_index_build_matches_bruteforce(n_adapters):
    T, K, E = 37, 4, 16
    z = synth.normal(21, "ib", (T, E)).astype(np.float64)
    idx, _ = oracle.topk(z, K)
    aid = None
    if n_adapters > 1:
        aid = synth.randint(21, "ib/a", (T,), -1, n_adapters - 1)
    counts, offsets, perm = oracle.index_build(idx, aid, E, n_adapters)
    jobs = []
    for t in range(T):
        a = (aid[t] if aid is not None else (0 if n_adapters > 0 else -1))
        ar = n_adapters if a < 0 else a
        for k in range(K + 1):
            e = idx[t, k] if k < K else E
            jobs.append((e, ar, t, k, a))
    jobs.sort()
    assert [list(r) for r in perm] == [[t, k, a, e] for (e, ar, t, k, a) in jobs]
    assert list(counts) == list(np.bincount([j[0] for j in jobs], minlength=E + 1))
    assert list(offsets) == [0] + list(np.cumsum(counts))
    assert counts[E] == T and offsets[-1] == T * (K + 1)


# ----------------------------------------------------------------- worked example
def _const_layer(E, K, H, I, vals, with_shared=True, shared_vals=None, sgate=None):
    """Layer whose groups are constants (bf16 exact, so dequantisation is exact)."""
    t = {}

    def q(name, arr, bits):
        p, s, b = oracle.quant_affine(arr.astype(np.float32), bits, 64)
        t[name + "_p"], t[name + "_s"], t[name + "_b"] = p, s, b

    q("router", np.stack([np.full(H, v, np.float32) for v in vals["router"]]), 8)
    q("gate", np.stack([np.full((I, H), v) for v in vals["gate"]]), 4)
    q("up", np.stack([np.full((I, H), v) for v in vals["up"]]), 4)
    q("down", np.stack([np.full((H, I), v) for v in vals["down"]]), 4)
    if with_shared:
        sv = shared_vals
        q("s_gate", np.full((1, I, H), sv["gate"]), 4)
        q("s_up", np.full((1, I, H), sv["up"]), 4)
        q("s_down", np.full((1, H, I), sv["down"]), 4)
        if sgate is not None:
            q("sgate", np.full((1, H), sgate, np.float32), 8)
    t["lora"] = []

    class S:
        pass
    s = S()
    s.H, s.E, s.K, s.I, s.Is, s.rank, s.alpha, s.group = H, E, K, I, I, 0, 0.0, 64
    return oracle_layer(s, t), t


def _silu(v):
    return v / (1.0 + math.exp(-v))


def _sigmoid(v):
    return 1.0 / (1.0 + math.exp(-v))


def test_worked_example_closed_form():
    # H = I = 64, x = 1: expert 0 has g = 64 * (1/64) = 1, u = 64 * (1/32) = 2,
    # so h = SiLU(1) * 2 and y = 64 * (1/64) * h = h.  The router sends the token
    # to expert 0 with weight 1 (K = 1); the shared gate logit is 1 and the shared
    # expert has g = 1, u = 1, down 1/64, so y_s = SiLU(1).
    H = I = 64
    vals = {"router": [1 / 64, -1 / 64], "gate": [1 / 64, 1 / 16], "up": [1 / 32, 1 / 16],
            "down": [1 / 64, 1 / 16]}
    L, _ = _const_layer(2, 1, H, I, vals, shared_vals={"gate": 1 / 64, "up": 1 / 64, "down": 1 / 64},
                        sgate=1 / 64)
    x = synth.bf16(np.ones((1, H), np.float32))
    y, idx, w, sg, logits = L.ffn(x)
    assert list(idx[0]) == [0] and w[0, 0] == 1.0
    assert logits[0, 0] == pytest.approx(1.0, abs=0) and logits[0, 1] == -1.0
    assert sg[0] == pytest.approx(_sigmoid(1.0), rel=1e-15)
    expect = _silu(1.0) * 2.0 + _sigmoid(1.0) * _silu(1.0)
    assert np.allclose(y, expect, rtol=1e-14, atol=0)
    # the same example must catch SiLU placed on the up branch
    oracle.set_mutation(oracle.MUTATION_SWAP_GATE_UP)
    try:
        ym = L.ffn(x)[0]
    finally:
        oracle.set_mutation(oracle.MUTATION_NONE)
    wrong = 1.0 * _silu(2.0) + _sigmoid(1.0) * _silu(1.0)
    assert np.allclose(ym, wrong, rtol=1e-14)
    assert not np.allclose(ym, expect, rtol=1e-3)


def test_worked_block_closed_form():
    # RMSNorm of an all-ones row is 1/sqrt(1 + 1e-6), which rounds to bf16 1.0,
    # so the block output is bf16(1 + y) with y from the worked example.
    H = I = 64
    vals = {"router": [1 / 64, -1 / 64], "gate": [1 / 64, 1 / 16], "up": [1 / 32, 1 / 16],
            "down": [1 / 64, 1 / 16]}
    L, _ = _const_layer(2, 1, H, I, vals, shared_vals={"gate": 1 / 64, "up": 1 / 64, "down": 1 / 64},
                        sgate=1 / 64)
    x = synth.bf16(np.ones((1, H), np.float32))
    assert np.all(oracle.rmsnorm_bf16(x, H) == 0x3F80)
    out = L.block(x)
    y = _silu(1.0) * 2.0 + _sigmoid(1.0) * _silu(1.0)
    assert np.all(out == oracle.bf16_round_nearest(1.0 + y))


def test_rmsnorm_closed_form():
    x = synth.bf16(np.array([[1.0, 7.0], [-2.0, 2.0]], np.float32))
    xn = oracle.rmsnorm_bf16(x, 2, eps=1e-6)
    r0 = 1.0 / math.sqrt(25.0 + 1e-6)
    r1 = 1.0 / math.sqrt(4.0 + 1e-6)
    assert list(xn[0]) == [oracle.bf16_round_nearest(1.0 * r0), oracle.bf16_round_nearest(7.0 * r0)]
    assert list(xn[1]) == [oracle.bf16_round_nearest(-2.0 * r1), oracle.bf16_round_nearest(2.0 * r1)]


# ----------------------------------------------------------------- dense special case
def _dense_expert(Wg, Wu, Wd, x, lora=None, scale=0.0):
    g = x @ Wg.T
    u = x @ Wu.T
    if lora is not None:
        Ag, Bg, Au, Bu, Ad, Bd = lora
        g = g + scale * (x @ Ag.T) @ Bg.T
        u = u + scale * (x @ Au.T) @ Bu.T
    h = g / (1.0 + np.exp(-g)) * u
    y = h @ Wd.T
    if lora is not None:
        y = y + scale * (h @ Ad.T) @ Bd.T
    return y


def _deq(t, name, in_, bits=4):
    return oracle.dequant_affine(t[name + "_p"], t[name + "_s"], t[name + "_b"], in_, bits).astype(np.float64)


def _lora_f64(ad, proj):
    return [synth.bf16_to_f32(ad[proj + "_A"]).astype(np.float64),
            synth.bf16_to_f32(ad[proj + "_B"]).astype(np.float64)]


def test_all_experts_uniform_gates_equal_dense_sum():
    # K = E and an all-zero router give every expert the weight 1/E, so the
    # routed FFN must equal a dense sum over all experts plus the gated shared expert.
    s = workloads.TINY
    w = workloads.moe_weights(s, seed=1)
    w["router"][:] = 0.0
    t = quantize_layer(w)
    import dataclasses
    sK = dataclasses.replace(s, K=s.E)
    L = oracle_layer(sK, t)
    x, _ = workloads.moe_inputs(s, seed=1)
    y, idx, wts, sg, _ = L.ffn(x)
    assert np.allclose(wts, 1.0 / s.E, rtol=1e-14)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    Wg, Wu, Wd = _deq(t, "gate", s.H), _deq(t, "up", s.H), _deq(t, "down", s.I)
    Sg, Su, Sd = _deq(t, "s_gate", s.H)[0], _deq(t, "s_up", s.H)[0], _deq(t, "s_down", s.Is)[0]
    ad = t["lora"][0]
    scale = s.alpha / s.rank
    ref = np.zeros_like(y)
    for e in range(s.E):
        lo = []
        for proj in ("gate", "up", "down"):
            A, B = _lora_f64(ad, proj)
            lo += [A[e], B[e]]
        ref += _dense_expert(Wg[e], Wu[e], Wd[e], xf, lo, scale) / s.E
    lo = []
    for proj in ("s_gate", "s_up", "s_down"):
        A, B = _lora_f64(ad, proj)
        lo += [A[0], B[0]]
    wsg = _deq(t, "sgate", s.H, 8)
    gsig = 1.0 / (1.0 + np.exp(-(xf @ wsg.T)))
    ref += gsig * _dense_expert(Sg, Su, Sd, xf, lo, scale)
    assert rel_l2(y, ref) < 1e-12
    # the planted up/gate swap must fail this comparison by a wide margin
    oracle.set_mutation(oracle.MUTATION_SWAP_GATE_UP)
    try:
        ym = L.ffn(x)[0]
    finally:
        oracle.set_mutation(oracle.MUTATION_NONE)
    assert rel_l2(ym, ref) > 0.1


def test_routed_equals_dense_on_selected_experts():
    s = workloads.TINY
    w = workloads.moe_weights(s, seed=2)
    t = quantize_layer(w)
    L = oracle_layer(s, t)
    x, _ = workloads.moe_inputs(s, seed=2)
    y, idx, wts, sg, logits = L.ffn(x)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    Wg, Wu, Wd = _deq(t, "gate", s.H), _deq(t, "up", s.H), _deq(t, "down", s.I)
    Sg, Su, Sd = _deq(t, "s_gate", s.H)[0], _deq(t, "s_up", s.H)[0], _deq(t, "s_down", s.Is)[0]
    ad = t["lora"][0]
    scale = s.alpha / s.rank
    for tok in range(s.T):
        p = softmax(logits[tok])
        ref_idx = sorted(range(s.E), key=lambda e: (-logits[tok, e], e))[:s.K]
        assert list(idx[tok]) == ref_idx
        ref = np.zeros(s.H)
        for k, e in enumerate(ref_idx):
            lo = []
            for proj in ("gate", "up", "down"):
                A, B = _lora_f64(ad, proj)
                lo += [A[e], B[e]]
            ref += p[e] / p[ref_idx].sum() * _dense_expert(Wg[e], Wu[e], Wd[e], xf[tok:tok + 1], lo, scale)[0]
        lo = []
        for proj in ("s_gate", "s_up", "s_down"):
            A, B = _lora_f64(ad, proj)
            lo += [A[0], B[0]]
        ref += sg[tok] * _dense_expert(Sg, Su, Sd, xf[tok:tok + 1], lo, scale)[0]
        assert rel_l2(y[tok], ref) < 1e-12


def test_zero_B_reproduces_base_output():
    s = workloads.TINY
    w0 = workloads.moe_weights(s, seed=3, lora_zero_B=True)
    t = quantize_layer(w0)
    x, _ = workloads.moe_inputs(s, seed=3)
    y_b0 = oracle_layer(s, t).ffn(x)[0]
    y_base = oracle_layer(s, t, n_adapters=0).ffn(x)[0]
    assert np.array_equal(y_b0, y_base)
    w1 = workloads.moe_weights(s, seed=3)
    y_lora = oracle_layer(s, quantize_layer(w1)).ffn(x)[0]
    assert rel_l2(y_lora, y_base) > 1e-3


def test_down_delta_is_linear_in_alpha_and_sparse():
    # A rank-1 down adapter with A = e_i and B = e_o changes only output row o,
    # and its change is linear in alpha (the down delta feeds no nonlinearity).
    s = workloads.TINY
    w = workloads.moe_weights(s, seed=4)
    t = quantize_layer(w)
    r = s.rank
    lo = {}
    for proj, (n, out, in_) in {"gate": (s.E, s.I, s.H), "up": (s.E, s.I, s.H), "down": (s.E, s.H, s.I),
                                "s_gate": (1, s.Is, s.H), "s_up": (1, s.Is, s.H),
                                "s_down": (1, s.H, s.Is)}.items():
        lo[proj + "_A"] = np.zeros((n, r, in_), np.uint16)
        lo[proj + "_B"] = np.zeros((n, out, r), np.uint16)
    lo["down_A"][:, 0, 5] = 0x3F80
    lo["down_B"][:, 17, 0] = 0x3F80
    t["lora"] = [lo]
    x, _ = workloads.moe_inputs(s, seed=4)
    import dataclasses
    y0 = oracle_layer(dataclasses.replace(s, alpha=0.0), t).ffn(x)[0]
    y1 = oracle_layer(dataclasses.replace(s, alpha=8.0), t).ffn(x)[0]
    y2 = oracle_layer(dataclasses.replace(s, alpha=16.0), t).ffn(x)[0]
    d1, d2 = y1 - y0, y2 - y0
    assert np.all(d1[:, np.arange(s.H) != 17] == 0.0)
    assert np.all(np.abs(d1[:, 17]) > 0)
    assert np.allclose(d2, 2 * d1, rtol=1e-12, atol=1e-15)


def test_adapter_selection_per_token():
    # A token routed through adapter a equals the same token on a layer that
    # holds adapter a alone; adapter -1 means the base alone.
    s = workloads.TINY
    import dataclasses
    s4 = dataclasses.replace(s, n_adapters=3)
    w = workloads.moe_weights(s4, seed=5)
    t = quantize_layer(w)
    x, _ = workloads.moe_inputs(s, seed=5)
    aid = np.array([2, -1, 0, 1], dtype=np.int32)
    y = oracle_layer(s4, t).ffn(x, aid)[0]
    for tok, a in enumerate(aid):
        tt = dict(t)
        tt["lora"] = [] if a < 0 else [t["lora"][a]]
        ya = oracle_layer(s4, tt).ffn(x[tok:tok + 1])[0]
        assert np.array_equal(y[tok], ya[0])


def test_select_override_renormalises():
    s = workloads.TINY
    t = quantize_layer(workloads.moe_weights(s, seed=6))
    L = oracle_layer(s, t)
    x, _ = workloads.moe_inputs(s, seed=6)
    y, idx, w, sg, logits = L.ffn(x)
    y2, idx2, w2, _, _ = L.ffn(x, select=idx[:, ::-1].copy())
    assert np.array_equal(idx2, idx[:, ::-1])
    assert np.allclose(w2, w[:, ::-1], rtol=1e-15)
    assert rel_l2(y2, y) < 1e-14

"""Pins of the oracle's EdgeRazor mixed-layout MLP and block (CPU only)."""
import numpy as np

import oracle
import synth
from synth import workloads
from tests.helpers import rel_l2


def _mlp_case(seed=30, H=128, I=192, T=3, rho=0.25):
    W = {n: synth.normal(seed, "mm/" + n, shp, std=0.02)
         for n, shp in (("gate", (I, H)), ("up", (I, H)), ("down", (H, I)))}
    q = {n: oracle.quant_mixed(W[n], rho) for n in W}
    x = synth.normal_bf16(seed, "mm/x", (T, H))
    return q, x, H, I, rho


def _dense(q, x, H, I, rho, swap=False):
    deq = {n: oracle.dequant_mixed(q[n][0], q[n][1], *((I, H) if n != "down" else (H, I)), rho).astype(np.float64)
           for n in q}
    xf = synth.bf16_to_f32(x).astype(np.float64)
    g = xf @ deq["gate"].T
    u = xf @ deq["up"].T
    if swap:
        g, u = u, g
    h = g / (1 + np.exp(-g)) * u
    return h @ deq["down"].T


def test_mixed_mlp_equals_dense_swiglu():
    q, x, H, I, rho = _mlp_case()
    y = oracle.mixed_mlp(q["gate"], q["up"], q["down"], H, I, rho, x)
    ref = _dense(q, x, H, I, rho)
    assert rel_l2(y, ref) < 1e-12
    oracle.set_mutation(oracle.MUTATION_SWAP_GATE_UP)
    try:
        ym = oracle.mixed_mlp(q["gate"], q["up"], q["down"], H, I, rho, x)
    finally:
        oracle.set_mutation(oracle.MUTATION_NONE)
    assert rel_l2(ym, ref) > 0.1
    assert rel_l2(ym, _dense(q, x, H, I, rho, swap=True)) < 1e-12


def test_mixed_block_is_residual_of_normed_mlp():
    q, x, H, I, rho = _mlp_case(seed=31)
    out = oracle.mixed_block(q["gate"], q["up"], q["down"], H, I, rho, x, eps=1e-6)
    xn = oracle.rmsnorm_bf16(x, H, eps=1e-6)
    y = _dense(q, xn, H, I, rho)
    ref = synth.bf16(synth.bf16_to_f32(x).astype(np.float64) + y)
    # the oracle rounds x + y from fp64 once; the reference rounds fp64 -> fp32 -> bf16
    diff = np.abs(synth.bf16_to_f32(out).astype(np.float64) - synth.bf16_to_f32(ref).astype(np.float64))
    ulp = np.abs(synth.bf16_to_f32(ref).astype(np.float64)) * 2.0 ** -7
    assert np.all(diff <= ulp + 1e-30)
    assert np.mean(out == ref) > 0.99


def test_mixed_qwen_shape_words():
    s = workloads.MIXED_B1
    G = oracle.mixed_group(s.rho)
    words = oracle.mixed_words(s.I, s.H, s.rho)
    assert words == (s.I // G) * (s.H // 8 + (G - 1) * s.H // 16)
    # bytes of one layer: three matrices of packed words plus one bf16 scale per row
    layer = 2 * (words * 4 + s.I * 2) + oracle.mixed_words(s.H, s.I, s.rho) * 4 + s.H * 2
    assert layer == 2963456

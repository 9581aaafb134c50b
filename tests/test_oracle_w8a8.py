"""Pins of the oracle's weight-activation form of the EdgeRazor mixed layer ("EDGERAZOR 深度解读"
section 2.1 量化公式 and 矩阵乘法分解; the 1.88-8-8 / 1.58-8-8 rows of the W/A table in
section 3.1): the 8-bit activation quantiser and Y = sum s_W s_X Q(W)^T Q(X)."""
import numpy as np
import pytest

import oracle
import synth
from synth import workloads


def test_act8_codes_and_scale():
    x = synth.normal(1, "a8/x", (6, 256)).astype(np.float32)
    x[2] *= 1e-3
    x[3] = 0.0
    q, s = oracle.quant_act8(x)
    assert q.dtype == np.int8 and np.all(np.abs(q.astype(int)) <= 127)
    for t in range(6):
        m = np.max(np.abs(x[t]))
        if m == 0.0:
            assert s[t] == np.float32(1e-5) and not q[t].any()
            continue
        assert s[t] == np.float32(m) / np.float32(127.0)  # one fp32 division
        j = int(np.argmax(np.abs(x[t])))
        assert abs(int(q[t, j])) == 127 and np.sign(q[t, j]) == np.sign(x[t, j])
        # every element within half a step (fp32 rounding of x / s allowed)
        err = np.abs(x[t].astype(np.float64) - s[t] * q[t].astype(np.float64))
        assert np.all(err <= 0.5 * s[t] * (1 + 1e-6))


def test_act8_integer_rows_are_exact():
    x = np.array([[127, -3, 0, 5, -127, 64, 1, -1]], np.float32)
    q, s = oracle.quant_act8(x)
    assert s[0] == 1.0 and np.array_equal(q[0], x[0].astype(np.int8))
    # round half to even on exact halves: 254 -> scale 2, codes 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    q2, s2 = oracle.quant_act8(np.array([[254.0, 1.0, 3.0, 5.0, -3.0]], np.float32))
    assert s2[0] == 2.0 and q2[0].tolist() == [127, 0, 2, 2, -2]


@pytest.fixture(scope="module")
def mixed():
    s = workloads.MIXED_B1
    W = workloads.mixed_weights(s, seed=2)
    return s, W, {n: oracle.quant_mixed(W[n], s.rho) for n in W}


def test_decomposition_equals_dequantised_dot(mixed):
    """s_W s_X Q(W)^T Q(X) equals the dot of the dequantised weights and the dequantised
    activations (the page's factorisation, checked with numpy)."""
    s, W, q = mixed
    x = workloads.mixed_inputs(s, seed=3, T=5)
    y = oracle.mixed_linear_a8(q["gate"][0], q["gate"][1], s.I, s.H, s.rho, x)
    qx, sx = oracle.quant_act8(synth.bf16_to_f32(x))
    Wd = oracle.dequant_mixed(q["gate"][0], q["gate"][1], s.I, s.H, s.rho).astype(np.float64)
    ref = (qx.astype(np.float64) * sx[:, None].astype(np.float64)) @ Wd.T
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_activation_error_bound_against_weight_only(mixed):
    """|y_a8 - y_weight_only| <= sum_j |w_hat_j| s_X / 2 per output (each activation code is
    within half a step of its input)."""
    s, W, q = mixed
    x = workloads.mixed_inputs(s, seed=4, T=3)
    ya8 = oracle.mixed_linear_a8(q["up"][0], q["up"][1], s.I, s.H, s.rho, x)
    ywo = oracle.mixed_linear(q["up"][0], q["up"][1], s.I, s.H, s.rho, x)
    _, sx = oracle.quant_act8(synth.bf16_to_f32(x))
    Wd = oracle.dequant_mixed(q["up"][0], q["up"][1], s.I, s.H, s.rho).astype(np.float64)
    bound = np.abs(Wd).sum(axis=1)[None, :] * (0.5 * sx.astype(np.float64))[:, None] * (1 + 1e-6)
    assert np.all(np.abs(ya8 - ywo) <= bound)
    assert np.linalg.norm(ya8 - ywo) > 0  # the activation codes do change the result


def test_mlp_a8_tracks_weight_only_mlp(mixed):
    s, W, q = mixed
    x = workloads.mixed_inputs(s, seed=5, T=4)
    ya8 = oracle.mixed_mlp_a8(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, x)
    ywo = oracle.mixed_mlp(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, x)
    rel = np.linalg.norm(ya8 - ywo) / np.linalg.norm(ywo)
    assert 1e-4 < rel < 5e-2
    # the residual block adds x to the a8 MLP of the normalised input
    xo = oracle.mixed_block_a8(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, x)
    xn = oracle.rmsnorm_bf16(x, s.H, 1e-6)
    ym = oracle.mixed_mlp_a8(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, xn)
    exp = synth.bf16(synth.bf16_to_f32(x).astype(np.float64) + ym)
    assert np.mean(xo == exp) > 0.99

"""Pins of the oracle's prerouter head ("Edge0 项目推荐" review, 亮点一): fp16 decoding,
the exact erf GELU, the feature layout [h, onehot(executed top-K), onehot(previous
token's top-K)], the linear_init skip and the full head against dense numpy algebra."""
import math

import numpy as np
import pytest
import scipy.special

import oracle
import synth
from synth import workloads


def test_fp16_decoding_matches_numpy_on_every_pattern():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    got = np.array([oracle.fp16_value(int(v)) for v in h])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isinf(got), np.isinf(ref)) and np.array_equal(np.isnan(got), np.isnan(ref))


def test_gelu_erf_closed_forms():
    assert oracle.gelu_erf(0.0) == 0.0
    for x in (0.1, 0.5, 1.0, 2.0, 3.5):  # x Phi(x) - (-x) Phi(-x) = x since Phi(x) + Phi(-x) = 1
        assert oracle.gelu_erf(x) - oracle.gelu_erf(-x) == pytest.approx(x, rel=1e-15, abs=1e-15)
    assert oracle.gelu_erf(10.0) == pytest.approx(10.0, rel=1e-15)
    assert abs(oracle.gelu_erf(-10.0)) < 1e-20
    # slope at 0 is Phi(0) = 1/2; x Phi(x) against scipy's normal CDF
    assert (oracle.gelu_erf(1e-6) - oracle.gelu_erf(-1e-6)) / 2e-6 == pytest.approx(0.5, rel=1e-9)
    xs = np.linspace(-6, 6, 97)
    assert np.allclose([oracle.gelu_erf(x) for x in xs], xs * scipy.special.ndtr(xs), rtol=1e-13, atol=1e-15)
    # not the tanh approximation: they differ by ~1e-4 near x = 2
    tanh_form = 0.5 * 2.0 * (1 + math.tanh(math.sqrt(2 / math.pi) * (2.0 + 0.044715 * 8.0)))
    assert abs(oracle.gelu_erf(2.0) - tanh_form) > 1e-5


def _zero_head(H, E, K, D):
    F = H + 2 * E
    z16 = lambda *s: np.zeros(s, np.uint16)  # noqa: E731 (fp16 +0.0)
    return {"w1": z16(D, F), "b1": z16(D), "w2": z16(E, D), "b2": z16(E), "wl": z16(E, F), "bl": z16(E)}


def test_feature_layout():
    """linear_init as a selector: row e reads h[e], row e reads onehot_exec[e] at H + e
    and onehot_prev[e] at H + E + e (with fc1 and fc2 zero, GELU(0) = 0)."""
    H, E, K, D = 16, 8, 3, 4
    F = H + 2 * E
    one = np.float16(1.0).view(np.uint16)
    h = synth.bf16(synth.normal(1, "pl/h", (2, H)))
    ex = np.array([[1, 4, 6], [0, 2, 7]], np.int32)
    pv = np.array([[3, 4, 5], [7, 6, 1]], np.int32)
    for block in range(3):
        w = _zero_head(H, E, K, D)
        wl = np.zeros((E, F), np.uint16)
        for e in range(E):
            wl[e, [e, H + e, H + E + e][block]] = one
        w["wl"] = wl
        z = oracle.prerouter(H, E, K, D, w, h, ex, pv)
        if block == 0:
            assert np.array_equal(z, synth.bf16_to_f32(h)[:, :E].astype(np.float64))
        else:
            sel = ex if block == 1 else pv
            exp = np.zeros((2, E))
            for t in range(2):
                exp[t, sel[t]] = 1.0
            assert np.array_equal(z, exp)
    # no previous token: its one-hot is all zero
    w = _zero_head(H, E, K, D)
    wl = np.zeros((E, F), np.uint16)
    wl[:, H + E:] = one
    w["wl"] = wl
    assert np.array_equal(oracle.prerouter(H, E, K, D, w, h, ex, None), np.zeros((2, E)))


def _dense(shape, w, h, ex, pv):
    """The head by dense numpy algebra (features materialised, scipy's normal CDF)."""
    H, E, D = shape.H, shape.E, shape.D
    f16 = lambda a: a.view(np.float16).astype(np.float64)  # noqa: E731
    T = h.shape[0]
    f = np.zeros((T, H + 2 * E))
    f[:, :H] = synth.bf16_to_f32(h)
    for t in range(T):
        f[t, H + ex[t]] = 1.0
        if pv is not None:
            f[t, H + E + pv[t]] = 1.0
    a = f @ f16(w["w1"]).T + f16(w["b1"])
    g = a * scipy.special.ndtr(a)
    return f @ f16(w["wl"]).T + f16(w["bl"]) + g @ f16(w["w2"]).T + f16(w["b2"])


def test_head_against_dense_algebra():
    s = workloads.PREROUTER_TINY
    w = workloads.prerouter_weights(s, seed=3)
    h, ex, pv = workloads.prerouter_inputs(s, seed=3)
    z = oracle.prerouter(s.H, s.E, s.K, s.D, w, h, ex, pv)
    assert np.allclose(z, _dense(s, w, h, ex, pv), rtol=1e-12, atol=1e-12)
    assert np.allclose(oracle.prerouter(s.H, s.E, s.K, s.D, w, h, ex, None), _dense(s, w, h, ex, None),
                       rtol=1e-12, atol=1e-12)


def test_linear_init_skip_alone():
    """With fc2 zeroed the head is exactly linear_init(f): linear in h and in the one-hots."""
    s = workloads.PREROUTER_TINY
    w = workloads.prerouter_weights(s, seed=4)
    w["w2"] = np.zeros_like(w["w2"])
    w["b2"] = np.zeros_like(w["b2"])
    h, ex, pv = workloads.prerouter_inputs(s, seed=4)
    z = oracle.prerouter(s.H, s.E, s.K, s.D, w, h, ex, pv)
    f16 = lambda a: a.view(np.float16).astype(np.float64)  # noqa: E731
    zero_h = np.zeros_like(h)
    z0 = oracle.prerouter(s.H, s.E, s.K, s.D, w, zero_h, ex, pv)
    # the h part alone: Wl[:, :H] h
    assert np.allclose(z - z0, synth.bf16_to_f32(h) @ f16(w["wl"])[:, :s.H].T, rtol=1e-12, atol=1e-12)


def test_planted_gelu_mistake_is_caught():
    """The head's nonlinearity matters: replacing GELU by identity moves the logits far."""
    s = workloads.PREROUTER_TINY
    w = workloads.prerouter_weights(s, seed=5)
    h, ex, pv = workloads.prerouter_inputs(s, seed=5)
    z = oracle.prerouter(s.H, s.E, s.K, s.D, w, h, ex, pv)
    H, E = s.H, s.E
    f16 = lambda a: a.view(np.float16).astype(np.float64)  # noqa: E731
    f = np.zeros((h.shape[0], H + 2 * E))
    f[:, :H] = synth.bf16_to_f32(h)
    for t in range(h.shape[0]):
        f[t, H + ex[t]] = 1.0
        f[t, H + E + pv[t]] = 1.0
    lin = f @ f16(w["wl"]).T + f16(w["bl"]) + (f @ f16(w["w1"]).T + f16(w["b1"])) @ f16(w["w2"]).T + f16(w["b2"])
    assert np.linalg.norm(z - lin) > 0.05 * np.linalg.norm(z)


def test_prerouter_inputs_are_distinct_top_k():
    s = workloads.PREROUTER
    h, ex, pv = workloads.prerouter_inputs(s, seed=0, T=64)
    assert ex.shape == (64, s.K) and all(len(set(r)) == s.K for r in ex) and ex.min() >= 0 and ex.max() < s.E

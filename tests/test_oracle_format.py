"""Pins of the oracle's storage formats and quantisers (CPU only).

Each check compares the oracle with something other than itself: the printed
numbers of the pages (tests/golden), exact rational arithmetic over the bf16
grid, closed forms, or hand-built bit patterns.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth
from tests.helpers import bf16_grid

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- bf16 rounding
def test_bf16_directed_rounding_against_grid():
    grid = bf16_grid()
    vals = np.concatenate([synth.normal(1, "bf16probe", (4000,), std=3.0).astype(np.float64),
                           synth.normal(2, "bf16probe2", (1000,), std=1e-3).astype(np.float64) * 1.0000001,
                           np.array([0.0, 1.0, -1.0, 1.0 + 2.0 ** -8, -(1.0 + 2.0 ** -8), 3.0e-39, 1e30])])
    for v in vals:
        i = np.searchsorted(grid, v, side="right")
        down = grid[i - 1]
        j = np.searchsorted(grid, v, side="left")
        up = grid[j]
        assert oracle.bf16_value(oracle.bf16_round_down(v)) == down
        assert oracle.bf16_value(oracle.bf16_round_up(v)) == up


def test_bf16_nearest_even_matches_independent_bit_trick():
    # For values that are exactly fp32, double->bf16 nearest-even must equal the
    # classic fp32 bit trick used by the input generator.
    f = synth.normal(3, "rne", (20000,), std=2.0)
    ref = synth.bf16(f)
    got = np.array([oracle.bf16_round_nearest(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, ref)
    # Exact ties go to the even pattern: 1 + 2^-8 lies halfway between 1.0 and 1 + 2^-7.
    assert oracle.bf16_round_nearest(1.0 + 2.0 ** -8) == 0x3F80
    assert oracle.bf16_round_nearest(1.0 + 3 * 2.0 ** -8) == 0x3F82


# ----------------------------------------------------------------- packing layout
def test_packing_field_order_golden():
    g = _gold("packing.json")
    # Constant-per-group weights that land exactly on the codes: w = s*q + b with
    # s = 1, b = 0 needs each group to span 0..15, so build rows whose first group
    # holds the codes of interest and the rest of the range.
    codes4 = list(g["int4_codes"]) + [0, 15] + [0] * 54
    W = np.array([codes4], dtype=np.float32)
    p, s, b = oracle.quant_affine(W, 4, 64)
    assert oracle.bf16_value(int(s[0, 0])) == 1.0 and oracle.bf16_value(int(b[0, 0])) == 0.0
    assert int(p[0, 0]) == g["int4_word"]
    codes8 = list(g["int8_codes"]) + [0, 255] + [0] * 58
    p8, s8, b8 = oracle.quant_affine(np.array([codes8], dtype=np.float32), 8, 64)
    assert int(p8[0, 0]) == g["int8_word"]
    assert oracle.bf16_value(int(s8[0, 0])) == 1.0


def test_unpack_repack_round_trip_bit_exact():
    W = synth.normal(4, "rt", (6, 256), std=0.02, outlier_prob=0.01, outlier_factor=20.0)
    for bits in (4, 8):
        p, s, b = oracle.quant_affine(W, bits, 64)
        q = oracle.unpack_codes(p, 256, bits)
        per = 32 // bits
        rep = np.zeros_like(p)
        for j in range(256):
            rep[:, j // per] |= (q[:, j].astype(np.uint32) << np.uint32((j % per) * bits))
        assert np.array_equal(rep, p)
        assert q.min() >= 0 and q.max() <= (1 << bits) - 1


# ----------------------------------------------------------------- affine quantiser
def _bruteforce_affine(wg, bits, grid):
    """Exact-rational restatement of the quantiser rule for one group."""
    qmax = (1 << bits) - 1
    lo, hi = float(min(wg)), float(max(wg))
    b = grid[np.searchsorted(grid, lo, side="right") - 1]
    d = Fraction(hi) - Fraction(b)
    if d == 0:
        return 0.0, b, [0] * len(wg)
    target = d / qmax
    j = np.searchsorted(grid, float(target), side="left")
    while Fraction(grid[j]) < target:
        j += 1
    while j > 0 and Fraction(grid[j - 1]) >= target:
        j -= 1
    s = grid[j]
    qs = [min(max(round((Fraction(float(w)) - Fraction(b)) / Fraction(s)), 0), qmax) for w in wg]
    return s, b, qs


@pytest.mark.parametrize("bits", [4, 8])
def test_affine_quantiser_matches_exact_rational_rule(bits):
    grid = bf16_grid()
    W = synth.normal(5, "q%d" % bits, (3, 192), std=0.02, outlier_prob=0.02, outlier_factor=20.0)
    p, s, b = oracle.quant_affine(W, bits, 64)
    q = oracle.unpack_codes(p, 192, bits)
    for r in range(3):
        for g in range(3):
            es, eb, eq = _bruteforce_affine(W[r, g * 64:(g + 1) * 64], bits, grid)
            assert oracle.bf16_value(int(s[r, g])) == es
            assert oracle.bf16_value(int(b[r, g])) == eb
            assert list(q[r, g * 64:(g + 1) * 64]) == eq


@pytest.mark.parametrize("bits", [4, 8])
def test_affine_error_at_most_half_step(bits):
    W = synth.normal(6, "err%d" % bits, (64, 512), std=0.02, outlier_prob=1e-3, outlier_factor=20.0)
    p, s, b = oracle.quant_affine(W, bits, 64)
    wh = oracle.dequant_affine(p, s, b, 512, bits, 64)
    sv = synth.bf16_to_f32(s).astype(np.float64).repeat(64, axis=1)
    err = np.abs(W.astype(np.float64) - wh.astype(np.float64))
    # s/2 plus the one fp32 rounding of the stored dequantised value.
    slack = np.abs(wh.astype(np.float64)) * 2.0 ** -24
    assert np.all(err <= sv / 2 * (1 + 1e-12) + slack)
    bv = synth.bf16_to_f32(b).astype(np.float64)
    gmin = W.reshape(64, 8, 64).min(axis=2)
    gmax = W.reshape(64, 8, 64).max(axis=2)
    assert np.all(bv <= gmin)
    assert np.all(synth.bf16_to_f32(s) * ((1 << bits) - 1) + bv >= gmax)


def test_constant_groups_are_exact():
    vals = [0.0, 0.5, -1.25, 2.0 ** -6, 3.0]
    W = np.concatenate([np.full((1, 64), v, dtype=np.float32) for v in vals], axis=1)
    for bits in (4, 8):
        p, s, b = oracle.quant_affine(W, bits, 64)
        wh = oracle.dequant_affine(p, s, b, W.shape[1], bits, 64)
        assert np.array_equal(wh, W)
        assert np.all(s == 0)


def test_dequant_hand_example():
    # s = 0.5 (0x3F00), b = -1.0 (0xBF80): codes 0, 3, 15 -> -1.0, 0.5, 6.5.
    packed = np.zeros((1, 8), dtype=np.uint32)
    packed[0, 0] = 0 | (3 << 4) | (15 << 8)
    s = np.array([[0x3F00]], dtype=np.uint16)
    b = np.array([[0xBF80]], dtype=np.uint16)
    wh = oracle.dequant_affine(packed, s, b, 64, 4, 64)
    assert list(wh[0, :3]) == [-1.0, 0.5, 6.5]
    assert np.all(wh[0, 3:] == -1.0)


def test_verbatim_ingest_zero_dequant_error():
    # Packed words, scales and biases copied byte for byte give exactly the
    # same dequantised weights (0.0 error), whatever produced them.
    W = synth.normal(7, "ingest", (8, 128), std=0.02)
    p, s, b = oracle.quant_affine(W, 4, 64)
    p2, s2, b2 = (np.frombuffer(a.tobytes(), dtype=a.dtype).reshape(a.shape) for a in (p, s, b))
    assert np.max(np.abs(oracle.dequant_affine(p, s, b, 128, 4, 64) - oracle.dequant_affine(p2, s2, b2, 128, 4, 64))) == 0.0


def test_storage_cost_golden():
    g = _gold("storage_cost.json")
    W = synth.normal(8, "cost", (1, g["group"]), std=0.02)
    p, s, b = oracle.quant_affine(W, 4, g["group"])
    assert p.nbytes == g["int4_bytes"]
    assert s.nbytes + b.nbytes == g["param_bytes"]
    assert W.size * 2 == g["bf16_bytes"]
    ratio = (p.nbytes + s.nbytes + b.nbytes) / g["bf16_bytes"]
    assert abs(ratio - g["approx_ratio"]) < 0.03


# ----------------------------------------------------------------- mixed layout
def test_mixed_bits_per_weight_labels():
    g = _gold("edgerazor_bits.json")
    for case in g["cases"]:
        rho = case["rho"]
        G = oracle.mixed_group(rho)
        out, in_ = 8 * G, 64
        W = synth.normal(9, "bits", (out, in_), std=0.02)
        packed, scales = oracle.quant_mixed(W, rho)
        q = oracle.mixed_codes(packed, out, in_, rho)
        four = np.array([np.any(np.abs(q[o]) > 1) or (o % G == 0) for o in range(out)])
        frac4 = np.mean([o % G == 0 for o in range(out)])
        assert frac4 == pytest.approx(rho)
        eff = frac4 * 4 + (1 - frac4) * g["ternary_bits"]
        # the printed label is the closed form rounded to two decimals
        assert abs(eff - case["label"]) <= 0.005 + 1e-12
        assert four.sum() == out // G


def test_mixed_codes_scales_and_super_groups():
    grid = bf16_grid()
    out, in_, rho = 10, 96, 0.25  # G = 4, trailing partial super-group of 2 rows
    G = oracle.mixed_group(rho)
    assert G == 4
    W = synth.normal(10, "mixed", (out, in_), std=0.02, outlier_prob=0.02, outlier_factor=20.0)
    packed, scales = oracle.quant_mixed(W, rho)
    w4, w2 = in_ // 8, in_ // 16
    assert packed.size == 2 * (w4 + 3 * w2) + (w4 + w2)
    q = oracle.mixed_codes(packed, out, in_, rho)
    for o in range(out):
        s = oracle.bf16_value(int(scales[o]))
        wrow = [Fraction(float(v)) for v in W[o]]
        if o % G == 0:
            m = max(abs(v) for v in wrow)
            target = max(m / 7, Fraction(1e-5))
            assert s == _nearest_bf16(target, grid)
            assert q[o].min() >= -7 and q[o].max() <= 7
            exp = [min(max(round(v / Fraction(s)), -7), 7) for v in wrow]
        else:
            mean = sum(abs(v) for v in wrow) / in_
            target = max(2 * mean, Fraction(1e-5))
            assert s == _nearest_bf16(target, grid)
            assert set(np.unique(q[o])) <= {-1, 0, 1}
            exp = [min(max(round(v / Fraction(s)), -1), 1) for v in wrow]
        assert list(q[o]) == exp
    # exactly one 4-bit row per super-group, the first one
    rows4 = [o for o in range(out) if o % G == 0]
    assert rows4 == [0, 4, 8]


def _nearest_bf16(target, grid):
    j = np.searchsorted(grid, float(target))
    cands = [grid[k] for k in (j - 1, j, j + 1) if 0 <= k < len(grid)]
    best = min(cands, key=lambda c: (abs(Fraction(c) - target), int(np.float32(c).view(np.uint32) >> 16) & 1))
    return best


def test_mixed_field_order_golden():
    g = _gold("packing.json")
    out, in_, rho = 2, 16, 0.5  # row 0 four-bit, row 1 ternary
    s4 = 0.25
    W = np.zeros((out, in_), dtype=np.float32)
    W[0, :8] = np.array(g["int4sym_codes"], dtype=np.float32) * s4
    W[0, 8] = 7 * s4  # pins max|w|/7 = s4
    W[1] = np.array(g["ternary_codes"], dtype=np.float32) * 0.5
    packed, scales = oracle.quant_mixed(W, rho)
    word0 = 0
    for j, c in enumerate(g["int4sym_codes"]):
        word0 |= (c + 8) << (4 * j)
    assert int(packed[0]) == word0
    # ternary row starts after the 4-bit row's in/8 = 2 words
    mean = np.mean(np.abs(W[1].astype(np.float64)))
    assert oracle.bf16_value(int(scales[1])) == pytest.approx(2 * mean, rel=2 ** -8)
    word_t = 0
    for j, c in enumerate(g["ternary_codes"]):
        word_t |= (c + 1) << (2 * j)
    assert int(packed[2]) == word_t


def test_mixed_matmul_decomposition():
    # [EdgeRazor 2.1]: the scale times the integer-code dot equals the dot with
    # dequantised weights (here with an independent numpy matmul).
    out, in_, rho = 12, 256, 0.25
    W = synth.normal(11, "dec", (out, in_), std=0.02)
    packed, scales = oracle.quant_mixed(W, rho)
    x = synth.normal_bf16(11, "decx", (5, in_))
    y = oracle.mixed_linear(packed, scales, out, in_, rho, x)
    wh = oracle.dequant_mixed(packed, scales, out, in_, rho).astype(np.float64)
    ref = synth.bf16_to_f32(x).astype(np.float64) @ wh.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_mixed_all_ternary_and_all_four_bit():
    W = synth.normal(12, "edge", (8, 64), std=0.02)
    p0, s0 = oracle.quant_mixed(W, 0.0)
    assert p0.size == 8 * 64 // 16
    assert set(np.unique(oracle.mixed_codes(p0, 8, 64, 0.0))) <= {-1, 0, 1}
    p1, s1 = oracle.quant_mixed(W, 1.0)
    assert p1.size == 8 * 64 // 8
    assert oracle.mixed_codes(p1, 8, 64, 1.0).max() == 7 or oracle.mixed_codes(p1, 8, 64, 1.0).min() == -7

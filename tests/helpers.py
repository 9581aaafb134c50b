"""Test helpers: quantise synthetic weights with the oracle and describe a layer."""
from __future__ import annotations

import numpy as np

import oracle


def quantize_layer(w: dict, group: int = 64) -> dict:
    """fp32 weights (from synth.workloads.moe_weights) -> packed tensors, via the oracle."""
    t = {}
    for name, bits, key in (("router", 8, "router"), ("sgate", 8, "sgate"), ("gate", 4, "gate"),
                            ("up", 4, "up"), ("down", 4, "down"), ("s_gate", 4, "s_gate"),
                            ("s_up", 4, "s_up"), ("s_down", 4, "s_down")):
        if w.get(key) is None:
            continue
        p, s, b = oracle.quant_affine(w[key], bits, group)
        t[name + "_p"], t[name + "_s"], t[name + "_b"] = p, s, b
    t["logit_bias"] = w.get("logit_bias")
    t["lora"] = w.get("lora") or []
    return t


def oracle_layer(shape, tensors: dict, n_adapters: int | None = None) -> oracle.OracleLayer:
    t = dict(tensors)
    if n_adapters is not None:
        t["lora"] = t["lora"][:n_adapters]
    return oracle.OracleLayer(shape.H, shape.E, shape.K, shape.I, shape.Is, t,
                              rank=shape.rank, alpha=shape.alpha, group=shape.group)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def bf16_grid() -> np.ndarray:
    """Every finite bf16 value, sorted, as float64 (for brute-force rounding checks)."""
    h = np.arange(65536, dtype=np.uint32)
    f32 = (h << 16).view(np.float32)
    f = f32[np.isfinite(f32)].astype(np.float64)
    return np.unique(f)

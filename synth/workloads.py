"""Synthetic workload recipes: shapes and value distributions only.

The shapes follow the Edge0-35B-A3B MoE layer (40 layers, 256 experts,
hidden 2048, expert and shared-expert intermediate 512, router and
shared_expert_gate at 8 bits, experts at int4 group 64, Recover-LoRA on every
projection) and the EdgeRazor Qwen3-0.6B MLP (hidden 1024, intermediate 3072,
28 layers, rho = 1/4).  No trained weights exist here, so every tensor is drawn
from the seeded generator in ``synth``: weights N(0, 0.02), LoRA factors
N(0, 0.01), activations N(0, 1) rounded to bf16.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import bf16, fp16, normal, randint, uniform


@dataclasses.dataclass(frozen=True)
class MoEShape:
    name: str
    H: int
    E: int
    K: int
    I: int
    Is: int
    T: int
    rank: int = 16
    alpha: float = 32.0
    n_adapters: int = 1
    layers: int = 1
    w_std: float = 0.02
    outlier_prob: float = 0.0
    outlier_factor: float = 20.0
    lora_std: float = 0.01
    logit_bias_std: float = 0.0
    random_adapters: bool = False
    group: int = 64


@dataclasses.dataclass(frozen=True)
class MixedShape:
    name: str
    H: int
    I: int
    T: int
    rho: float = 0.25
    layers: int = 1
    w_std: float = 0.02


# Tiny single layer: the case the oracle finishes in milliseconds.
TINY = MoEShape("tiny", H=256, E=8, K=2, I=128, Is=128, T=4, rank=8, alpha=16.0)
# Edge0-35B-shaped single layer, decode (one token), 0.1% of weights x20.
DECODE_K4 = MoEShape("decode_k4", H=2048, E=256, K=4, I=512, Is=512, T=1, outlier_prob=1e-3)
DECODE_K8 = dataclasses.replace(DECODE_K4, name="decode_k8", K=8)
# Multi-tenant decode: 64 tokens, 4 adapter sets over one base, per-expert logit offset N(0,1).
MULTI_TENANT = dataclasses.replace(DECODE_K4, name="multi_tenant", T=64, n_adapters=4,
                                   random_adapters=True, logit_bias_std=1.0)
# 40-layer prefill stack, 2048-token prompt.
PREFILL = MoEShape("prefill", H=2048, E=256, K=4, I=512, Is=512, T=2048, layers=40)
# EdgeRazor mixed-precision MLP stack (weight-only), decode batch 1 and 16.
MIXED_B1 = MixedShape("mixed_b1", H=1024, I=3072, T=1, layers=28)
MIXED_B16 = dataclasses.replace(MIXED_B1, name="mixed_b16", T=16)

# The same two workloads with the weights packed at group 32 (the d1a MLX port's group size).
DECODE_K4_G32 = dataclasses.replace(DECODE_K4, name="decode_k4_g32", group=32)
MULTI_TENANT_G32 = dataclasses.replace(MULTI_TENANT, name="multi_tenant_g32", group=32)

MOE_SHAPES = {s.name: s for s in (TINY, DECODE_K4, DECODE_K8, MULTI_TENANT, PREFILL, DECODE_K4_G32,
                                  MULTI_TENANT_G32)}
MIXED_SHAPES = {s.name: s for s in (MIXED_B1, MIXED_B16)}


def moe_weights(shape: MoEShape, seed: int = 0, layer: int = 0, lora_zero_B: bool = False):
    """Host fp32 weights of one MoE layer, plus bf16 LoRA factors.

    Returns a dict: router [E,H], sgate [1,H], gate/up [E,I,H], down [E,H,I],
    s_gate/s_up [1,Is,H], s_down [1,H,Is] (fp32), logit_bias [E] (fp32 or None)
    and lora: one dict per adapter with bf16 {proj}_A [n,r,in] / {proj}_B [n,out,r].
    """
    H, E, I, Is = shape.H, shape.E, shape.I, shape.Is
    p = "L%d/" % layer
    kw = dict(std=shape.w_std, outlier_prob=shape.outlier_prob, outlier_factor=shape.outlier_factor)
    w = {
        "router": normal(seed, p + "router", (E, H), **kw),
        "sgate": normal(seed, p + "sgate", (1, H), **kw),
        "gate": normal(seed, p + "gate", (E, I, H), **kw),
        "up": normal(seed, p + "up", (E, I, H), **kw),
        "down": normal(seed, p + "down", (E, H, I), **kw),
        "s_gate": normal(seed, p + "s_gate", (1, Is, H), **kw),
        "s_up": normal(seed, p + "s_up", (1, Is, H), **kw),
        "s_down": normal(seed, p + "s_down", (1, H, Is), **kw),
        "logit_bias": (normal(seed, p + "logit_bias", (E,), std=shape.logit_bias_std)
                       if shape.logit_bias_std > 0 else None),
    }
    lora = []
    r = shape.rank
    dims = {"gate": (E, I, H), "up": (E, I, H), "down": (E, H, I),
            "s_gate": (1, Is, H), "s_up": (1, Is, H), "s_down": (1, H, Is)}
    for a in range(shape.n_adapters):
        ad = {}
        for proj, (n, out, in_) in dims.items():
            q = p + "lora%d/%s" % (a, proj)
            ad[proj + "_A"] = bf16(normal(seed, q + "/A", (n, r, in_), std=shape.lora_std))
            Bv = normal(seed, q + "/B", (n, out, r), std=shape.lora_std)
            if lora_zero_B:
                Bv = np.zeros_like(Bv)
            ad[proj + "_B"] = bf16(Bv)
        lora.append(ad)
    w["lora"] = lora
    return w


def moe_inputs(shape: MoEShape, seed: int = 0, T: int | None = None, tag: str = "x"):
    """bf16 activations [T,H] and adapter ids [T] (None when one adapter serves all)."""
    T = shape.T if T is None else T
    x = bf16(normal(seed, tag, (T, shape.H)))
    aid = None
    if shape.random_adapters and shape.n_adapters > 0:
        aid = randint(seed, tag + "/adapter", (T,), 0, shape.n_adapters - 1)
    return x, aid


def mixed_weights(shape: MixedShape, seed: int = 0, layer: int = 0):
    p = "M%d/" % layer
    return {
        "gate": normal(seed, p + "gate", (shape.I, shape.H), std=shape.w_std),
        "up": normal(seed, p + "up", (shape.I, shape.H), std=shape.w_std),
        "down": normal(seed, p + "down", (shape.H, shape.I), std=shape.w_std),
    }


def mixed_inputs(shape: MixedShape, seed: int = 0, T: int | None = None, tag: str = "mx"):
    T = shape.T if T is None else T
    return bf16(normal(seed, tag, (T, shape.H)))


@dataclasses.dataclass(frozen=True)
class PrerouterShape:
    """One prerouter head: layer input width H, experts E, top-K, head hidden width D."""
    name: str
    H: int
    E: int
    K: int
    D: int = 512
    T: int = 1


# The Edge0-35B heads: hidden 2048, 256 experts, top-4, head width 512, fp16.
PREROUTER = PrerouterShape("prerouter", H=2048, E=256, K=4, D=512)
PREROUTER_TINY = PrerouterShape("prerouter_tiny", H=64, E=8, K=2, D=16, T=5)


def prerouter_weights(shape: PrerouterShape, seed: int = 0, layer: int = 0):
    """fp16 bit patterns of one head: fc1 w1 [D, H+2E], b1 [D]; fc2 w2 [E, D], b2 [E];
    linear_init wl [E, H+2E], bl [E].  Weights N(0, 1/fan_in), biases N(0, 0.1)."""
    H, E, D = shape.H, shape.E, shape.D
    F = H + 2 * E
    p = "P%d/" % layer
    return {
        "w1": fp16(normal(seed, p + "w1", (D, F), std=F ** -0.5)),
        "b1": fp16(normal(seed, p + "b1", (D,), std=0.1)),
        "w2": fp16(normal(seed, p + "w2", (E, D), std=D ** -0.5)),
        "b2": fp16(normal(seed, p + "b2", (E,), std=0.1)),
        "wl": fp16(normal(seed, p + "wl", (E, F), std=F ** -0.5)),
        "bl": fp16(normal(seed, p + "bl", (E,), std=0.1)),
    }


def prerouter_inputs(shape: PrerouterShape, seed: int = 0, T: int | None = None, tag: str = "pr"):
    """The head's layer input h (bf16 N(0,1) [T, H]) and two top-K expert lists [T, K]
    (K distinct experts per token, uniformly at random): the token's own executed
    routing and the previous token's."""
    T = shape.T if T is None else T
    h = bf16(normal(seed, tag + "/h", (T, shape.H)))
    ex = np.argsort(uniform(seed, tag + "/exec", (T, shape.E)), axis=1, kind="stable")[:, :shape.K].astype(np.int32)
    pv = np.argsort(uniform(seed, tag + "/prev", (T, shape.E)), axis=1, kind="stable")[:, :shape.K].astype(np.int32)
    return h, ex, pv

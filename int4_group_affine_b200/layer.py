"""Device-side holders of layer weights for the C ABI (torch used for memory only).

``DeviceLayer`` owns the torch tensors of one MoE layer (packed words, bf16
scales/biases as int16 bit patterns, LoRA factors) and exposes the ``moe_layer``
descriptor that libmoeq's entry points take.  ``DeviceMixed`` does the same for
one EdgeRazor mixed-layout matrix.  Quantisation and every forward computation
happen in libmoeq's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (FMT_AFFINE_INT4, FMT_AFFINE_INT8, FMT_MIXED_TERNARY_INT4, Layer, LoraPtrs, MixedTensor, QTensor,
               lora_set_adapters, moe_ffn_forward, moe_ffn_workspace_bytes, moe_mixed_words, moe_quant_pack,
               moe_workspace_init)

PROJ_DIMS = ("gate", "up", "down", "s_gate", "s_up", "s_down")


def to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    """Host array -> device tensor with the same bits (uint32 as int32, uint16 as int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    elif a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


def to_host(t: torch.Tensor, dtype) -> np.ndarray:
    """Device tensor -> host array reinterpreted as `dtype` (same bits)."""
    return t.detach().cpu().contiguous().numpy().view(dtype)


def _q(p, s, b, n, out, in_, bits, group) -> QTensor:
    q = QTensor()
    if p is None:
        return q
    q.packed, q.scales, q.biases = p.data_ptr(), s.data_ptr(), b.data_ptr()
    q.n, q.out, q.in_, q.bits, q.group = n, out, in_, bits, group
    return q


class DeviceLayer:
    """One MoE layer resident in device memory."""

    SPEC = {  # name -> (bits, n, out, in) as functions of (H, E, I, Is)
        "router": lambda H, E, I, Is: (8, 1, E, H),
        "sgate": lambda H, E, I, Is: (8, 1, 1, H),
        "gate": lambda H, E, I, Is: (4, E, I, H),
        "up": lambda H, E, I, Is: (4, E, I, H),
        "down": lambda H, E, I, Is: (4, E, H, I),
        "s_gate": lambda H, E, I, Is: (4, 1, Is, H),
        "s_up": lambda H, E, I, Is: (4, 1, Is, H),
        "s_down": lambda H, E, I, Is: (4, 1, H, Is),
    }

    def __init__(self, H, E, K, I, Is, rank=0, alpha=0.0, group=64):
        self.H, self.E, self.K, self.I, self.Is = H, E, K, I, Is
        self.rank, self.alpha, self.group = rank, alpha, group
        self.t: dict[str, torch.Tensor] = {}
        self.lora: list[dict[str, torch.Tensor]] = []
        self.L = Layer()

    # ------------------------------------------------------------ builders
    @classmethod
    def from_host(cls, shape, tensors: dict, device="cuda", n_adapters=None):
        """Upload pre-packed host tensors ({name}_p/_s/_b, logit_bias, lora) verbatim."""
        d = cls(shape.H, shape.E, shape.K, shape.I, shape.Is, shape.rank, shape.alpha, shape.group)
        for name in cls.SPEC:
            if tensors.get(name + "_p") is None:
                continue
            for suf in ("_p", "_s", "_b"):
                d.t[name + suf] = to_device(tensors[name + suf], device)
        if tensors.get("logit_bias") is not None:
            d.t["logit_bias"] = to_device(np.asarray(tensors["logit_bias"], np.float32), device)
        lora = tensors.get("lora") or []
        if n_adapters is not None:
            lora = lora[:n_adapters]
        d.lora = [{k: to_device(v, device) for k, v in ad.items()} for ad in lora]
        d._build()
        return d

    @classmethod
    def from_fp32(cls, shape, weights: dict, lora=None, stream=None):
        """Quantise device fp32 weights with libmoeq's pack kernel (router/sgate int8, experts int4).

        `weights` maps router/sgate/gate/up/down/s_gate/s_up/s_down to CUDA fp32
        tensors and optionally logit_bias; `lora` is a list of dicts of CUDA int16
        (bf16 bit) tensors."""
        d = cls(shape.H, shape.E, shape.K, shape.I, shape.Is, shape.rank, shape.alpha, shape.group)
        g = shape.group
        for name, spec in cls.SPEC.items():
            W = weights.get(name)
            if W is None:
                continue
            bits, n, out, in_ = spec(shape.H, shape.E, shape.I, shape.Is)
            dev = W.device
            rows = n * out
            p = torch.empty((n, out, in_ * bits // 32), dtype=torch.int32, device=dev)
            s = torch.empty((n, out, in_ // g), dtype=torch.int16, device=dev)
            b = torch.empty((n, out, in_ // g), dtype=torch.int16, device=dev)
            moe_quant_pack(FMT_AFFINE_INT4 if bits == 4 else FMT_AFFINE_INT8, W.contiguous(), rows, in_, g, 0.0,
                           p, s, b, stream)
            d.t[name + "_p"], d.t[name + "_s"], d.t[name + "_b"] = p, s, b
        if weights.get("logit_bias") is not None:
            d.t["logit_bias"] = weights["logit_bias"].float().contiguous()
        d.lora = list(lora or [])
        d._build()
        return d

    def _build(self):
        L = Layer()
        H, E, I, Is = self.H, self.E, self.I, self.Is
        L.hidden, L.n_experts, L.top_k, L.inter, L.shared_inter = H, E, self.K, I, Is
        for name, spec in self.SPEC.items():
            bits, n, out, in_ = spec(H, E, I, Is)
            q = _q(self.t.get(name + "_p"), self.t.get(name + "_s"), self.t.get(name + "_b"), n, out, in_, bits,
                   self.group)
            setattr(L, "shared_gate" if name == "sgate" else name, q)
        lb = self.t.get("logit_bias")
        L.logit_bias = lb.data_ptr() if lb is not None else None
        self.L = L
        sets = []
        for ad in self.lora:
            ps = LoraPtrs()
            for proj in PROJ_DIMS:
                A, B = ad.get(proj + "_A"), ad.get(proj + "_B")
                if A is not None and B is not None:
                    lp = getattr(ps, proj)
                    lp.A, lp.B = A.data_ptr(), B.data_ptr()
            sets.append(ps)
        lora_set_adapters(self.L, len(sets), self.rank if sets else 0, float(self.alpha) if sets else 0.0, sets)

    # ------------------------------------------------------------ helpers
    def workspace(self, T, device="cuda", stream=None):
        nbytes = moe_ffn_workspace_bytes(self.L, T)
        if nbytes == 0:
            raise ValueError("layer rejected by moe_ffn_workspace_bytes")
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        moe_workspace_init(ws, nbytes, stream)
        return ws, nbytes

    def forward(self, x: torch.Tensor, adapter_id=None, out=None, ws=None, stream=None) -> torch.Tensor:
        """y = FFN(x); x is a CUDA int16 (bf16 bits) or bfloat16 tensor [T, H]."""
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        if ws is None:
            ws = self.workspace(T, x.device, stream)
        moe_ffn_forward(self.L, x, adapter_id, T, out, ws[0], ws[1], stream)
        return out

    def nbytes(self) -> int:
        n = sum(t.numel() * t.element_size() for t in self.t.values())
        n += sum(t.numel() * t.element_size() for ad in self.lora for t in ad.values())
        return n


class DeviceMixed:
    """One EdgeRazor mixed ternary/4-bit matrix resident in device memory."""

    def __init__(self, out, in_, rho, packed: torch.Tensor, scales: torch.Tensor):
        self.out, self.in_, self.rho = out, in_, rho
        self.packed, self.scales = packed, scales
        self.T = MixedTensor()
        self.T.packed, self.T.scales = packed.data_ptr(), scales.data_ptr()
        self.T.out, self.T.in_, self.T.rho = out, in_, rho

    @classmethod
    def from_host(cls, out, in_, rho, packed: np.ndarray, scales: np.ndarray, device="cuda"):
        return cls(out, in_, rho, to_device(packed, device), to_device(scales, device))

    @classmethod
    def from_fp32(cls, W: torch.Tensor, rho, stream=None):
        out, in_ = W.shape
        words = moe_mixed_words(out, in_, rho)
        p = torch.empty(words, dtype=torch.int32, device=W.device)
        s = torch.empty(out, dtype=torch.int16, device=W.device)
        moe_quant_pack(FMT_MIXED_TERNARY_INT4, W.contiguous(), out, in_, 0, rho, p, s, None, stream)
        return cls(out, in_, rho, p, s)

    def nbytes(self) -> int:
        return self.packed.numel() * 4 + self.scales.numel() * 2

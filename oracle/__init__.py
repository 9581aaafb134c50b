"""ctypes front end of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this package.  Functions take and return numpy arrays; bf16 values
travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

MAX_ADAPTERS = 16
MUTATION_NONE = 0
MUTATION_SWAP_GATE_UP = 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, fp64, no FMA contraction, OpenMP)."""
    src = os.path.join(_HERE, "oracle.c")
    hdr = os.path.join(_HERE, "oracle.h")
    newest = max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                               "-shared", "-o", tmp, src, "-lm"])
        os.replace(tmp, _SO)
    return _SO


class QMat(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p),
                ("n", ctypes.c_int32), ("out", ctypes.c_int32), ("in_", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("group", ctypes.c_int32)]


class LoraProj(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("B", ctypes.c_void_p)]


class Adapter(ctypes.Structure):
    _fields_ = [(n, LoraProj) for n in ("gate", "up", "down", "s_gate", "s_up", "s_down")]


class Layer(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("E", ctypes.c_int32), ("K", ctypes.c_int32),
                ("I", ctypes.c_int32), ("Is", ctypes.c_int32),
                ("router", QMat), ("shared_gate", QMat),
                ("gate", QMat), ("up", QMat), ("down", QMat),
                ("s_gate", QMat), ("s_up", QMat), ("s_down", QMat),
                ("logit_bias", ctypes.c_void_p),
                ("n_adapters", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("alpha", ctypes.c_double),
                ("adapters", Adapter * MAX_ADAPTERS)]


def _get():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        sig = {
            "orc_set_mutation": (None, [I]),
            "orc_quant_affine": (I, [P, I64, I, I, I, P, P, P]),
            "orc_dequant_affine": (None, [P, P, P, I64, I, I, I, P]),
            "orc_unpack_codes": (None, [P, I64, I, I, P]),
            "orc_mixed_group": (I, [D]),
            "orc_mixed_words": (I64, [I, I, D]),
            "orc_mixed_row_offset": (I64, [I, I, I]),
            "orc_quant_mixed": (I, [P, I, I, D, P, P]),
            "orc_mixed_codes": (None, [P, I, I, D, P]),
            "orc_dequant_mixed": (None, [P, P, I, I, D, P]),
            "orc_mixed_linear": (None, [P, P, I, I, D, P, I, P]),
            "orc_mixed_mlp": (I, [P, P, P, P, P, P, I, I, D, P, I, P]),
            "orc_mixed_block": (I, [P, P, P, P, P, P, I, I, D, D, P, I, P]),
            "orc_router": (None, [P, P, I, P, P]),
            "orc_topk": (None, [P, I, I, I, P, P]),
            "orc_index_build": (I, [P, P, I, I, I, I, P, P, P]),
            "orc_moe_ffn": (I, [P, P, P, I, P, P, P, P, P, P]),
            "orc_rmsnorm_bf16": (None, [P, I, I, D, P]),
            "orc_moe_block": (I, [P, P, P, I, D, P]),
            "orc_bf16_round_down": (ctypes.c_uint16, [D]),
            "orc_bf16_round_up": (ctypes.c_uint16, [D]),
            "orc_bf16_round_nearest": (ctypes.c_uint16, [D]),
            "orc_bf16_value": (D, [ctypes.c_uint16]),
            "orc_threads": (I, []),
            "orc_fp16_value": (D, [ctypes.c_uint16]),
            "orc_gelu_erf": (D, [D]),
            "orc_prerouter": (I, [P, P, P, P, I, P]),
            "orc_quant_act8": (None, [P, I, I, P, P]),
            "orc_mixed_linear_a8": (None, [P, P, I, I, D, P, I, P]),
            "orc_mixed_mlp_a8": (I, [P, P, P, P, P, P, I, I, D, P, I, P]),
            "orc_mixed_block_a8": (I, [P, P, P, P, P, P, I, I, D, D, P, I, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def threads() -> int:
    return int(_get().orc_threads())


def set_mutation(m: int) -> None:
    _get().orc_set_mutation(int(m))


def bf16_round_down(v: float) -> int:
    return int(_get().orc_bf16_round_down(float(v)))


def bf16_round_up(v: float) -> int:
    return int(_get().orc_bf16_round_up(float(v)))


def bf16_round_nearest(v: float) -> int:
    return int(_get().orc_bf16_round_nearest(float(v)))


def bf16_value(h: int) -> float:
    return float(_get().orc_bf16_value(int(h)))


# ------------------------------------------------------------------ affine
def quant_affine(W: np.ndarray, bits: int, group: int = 64):
    """W fp32 [..., out, in] -> (packed uint32 [..., out, in*bits/32], scales, biases uint16 [..., out, in/group])."""
    W = _c(W, np.float32)
    in_ = W.shape[-1]
    rows = W.size // in_
    lead = W.shape[:-1]
    packed = np.empty(lead + (in_ * bits // 32,), dtype=np.uint32)
    scales = np.empty(lead + (in_ // group,), dtype=np.uint16)
    biases = np.empty(lead + (in_ // group,), dtype=np.uint16)
    rc = _get().orc_quant_affine(_p(W), rows, in_, bits, group, _p(packed), _p(scales), _p(biases))
    if rc != 0:
        raise ValueError("orc_quant_affine rejected the shape (rc=%d)" % rc)
    return packed, scales, biases


def dequant_affine(packed, scales, biases, in_: int, bits: int, group: int = 64) -> np.ndarray:
    packed = _c(packed, np.uint32)
    scales = _c(scales, np.uint16)
    biases = _c(biases, np.uint16)
    rows = packed.size // (in_ * bits // 32)
    out = np.empty(packed.shape[:-1] + (in_,), dtype=np.float32)
    _get().orc_dequant_affine(_p(packed), _p(scales), _p(biases), rows, in_, bits, group, _p(out))
    return out


def unpack_codes(packed, in_: int, bits: int) -> np.ndarray:
    packed = _c(packed, np.uint32)
    rows = packed.size // (in_ * bits // 32)
    q = np.empty(packed.shape[:-1] + (in_,), dtype=np.int32)
    _get().orc_unpack_codes(_p(packed), rows, in_, bits, _p(q))
    return q


# ------------------------------------------------------------------- mixed
def mixed_group(rho: float) -> int:
    return int(_get().orc_mixed_group(float(rho)))


def mixed_words(out: int, in_: int, rho: float) -> int:
    return int(_get().orc_mixed_words(out, in_, float(rho)))


def mixed_row_offset(row: int, in_: int, G: int) -> int:
    return int(_get().orc_mixed_row_offset(row, in_, G))


def quant_mixed(W: np.ndarray, rho: float):
    W = _c(W, np.float32)
    out, in_ = W.shape
    packed = np.empty(mixed_words(out, in_, rho), dtype=np.uint32)
    scales = np.empty(out, dtype=np.uint16)
    rc = _get().orc_quant_mixed(_p(W), out, in_, float(rho), _p(packed), _p(scales))
    if rc != 0:
        raise ValueError("orc_quant_mixed rejected the shape (rc=%d)" % rc)
    return packed, scales


def mixed_codes(packed, out: int, in_: int, rho: float) -> np.ndarray:
    q = np.empty((out, in_), dtype=np.int32)
    _get().orc_mixed_codes(_p(_c(packed, np.uint32)), out, in_, float(rho), _p(q))
    return q


def dequant_mixed(packed, scales, out: int, in_: int, rho: float) -> np.ndarray:
    w = np.empty((out, in_), dtype=np.float32)
    _get().orc_dequant_mixed(_p(_c(packed, np.uint32)), _p(_c(scales, np.uint16)), out, in_, float(rho), _p(w))
    return w


def mixed_linear(packed, scales, out: int, in_: int, rho: float, x_bf16) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    T = x.size // in_
    y = np.empty((T, out), dtype=np.float64)
    _get().orc_mixed_linear(_p(_c(packed, np.uint32)), _p(_c(scales, np.uint16)), out, in_, float(rho),
                            _p(x), T, _p(y))
    return y


def mixed_mlp(gate, up, down, H: int, I: int, rho: float, x_bf16) -> np.ndarray:
    """gate/up/down: (packed, scales) pairs in the mixed layout."""
    x = _c(x_bf16, np.uint16)
    T = x.size // H
    y = np.empty((T, H), dtype=np.float64)
    g, u, d = [(_c(p, np.uint32), _c(s, np.uint16)) for p, s in (gate, up, down)]
    rc = _get().orc_mixed_mlp(_p(g[0]), _p(g[1]), _p(u[0]), _p(u[1]), _p(d[0]), _p(d[1]), H, I, float(rho),
                              _p(x), T, _p(y))
    if rc:
        raise ValueError("orc_mixed_mlp rc=%d" % rc)
    return y


def mixed_block(gate, up, down, H: int, I: int, rho: float, x_bf16, eps: float = 1e-6) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    T = x.size // H
    out = np.empty((T, H), dtype=np.uint16)
    g, u, d = [(_c(p, np.uint32), _c(s, np.uint16)) for p, s in (gate, up, down)]
    rc = _get().orc_mixed_block(_p(g[0]), _p(g[1]), _p(u[0]), _p(u[1]), _p(d[0]), _p(d[1]), H, I,
                                float(rho), float(eps), _p(x), T, _p(out))
    if rc:
        raise ValueError("orc_mixed_block rc=%d" % rc)
    return out


# ------------------------------------------------------------------- layer
class OracleLayer:
    """Owns the numpy arrays of one MoE layer and the ctypes descriptor over them.

    ``tensors`` maps names to arrays:
      router_{p,s,b}, sgate_{p,s,b} (optional), {gate,up,down}_{p,s,b},
      {s_gate,s_up,s_down}_{p,s,b} (optional), logit_bias (optional),
      lora: list (one per adapter) of dicts with keys
      {gate,up,down,s_gate,s_up,s_down}_{A,B} (bf16 uint16 arrays).
    """

    def __init__(self, H, E, K, I, Is, tensors, rank=0, alpha=0.0, group=64):
        self.keep = []
        L = Layer()
        L.H, L.E, L.K, L.I, L.Is = H, E, K, I, Is

        def qm(prefix, n, out, in_, bits):
            q = QMat()
            if tensors.get(prefix + "_p") is None:
                return q
            arrs = [_c(tensors[prefix + "_p"], np.uint32), _c(tensors[prefix + "_s"], np.uint16),
                    _c(tensors[prefix + "_b"], np.uint16)]
            self.keep += arrs
            q.packed, q.scales, q.biases = [a.ctypes.data for a in arrs]
            q.n, q.out, q.in_, q.bits, q.group = n, out, in_, bits, group
            return q

        L.router = qm("router", 1, E, H, 8)
        L.shared_gate = qm("sgate", 1, 1, H, 8)
        L.gate = qm("gate", E, I, H, 4)
        L.up = qm("up", E, I, H, 4)
        L.down = qm("down", E, H, I, 4)
        L.s_gate = qm("s_gate", 1, Is, H, 4)
        L.s_up = qm("s_up", 1, Is, H, 4)
        L.s_down = qm("s_down", 1, H, Is, 4)
        lb = tensors.get("logit_bias")
        if lb is not None:
            lb = _c(lb, np.float32)
            self.keep.append(lb)
            L.logit_bias = lb.ctypes.data
        lora = tensors.get("lora") or []
        L.n_adapters = len(lora)
        L.rank = rank
        L.alpha = alpha
        for a, ad in enumerate(lora):
            for proj in ("gate", "up", "down", "s_gate", "s_up", "s_down"):
                A = ad.get(proj + "_A")
                B = ad.get(proj + "_B")
                if A is None or B is None:
                    continue
                A = _c(A, np.uint16)
                B = _c(B, np.uint16)
                self.keep += [A, B]
                lp = getattr(L.adapters[a], proj)
                lp.A, lp.B = A.ctypes.data, B.ctypes.data
        self.L = L
        self.H, self.E, self.K = H, E, K

    def ffn(self, x_bf16, adapter_id=None, select=None):
        """Returns (y fp64 [T,H], idx [T,K], w [T,K], sg [T], logits [T,E])."""
        x = _c(x_bf16, np.uint16)
        T = x.size // self.H
        y = np.empty((T, self.H), dtype=np.float64)
        idx = np.empty((T, self.K), dtype=np.int32)
        w = np.empty((T, self.K), dtype=np.float64)
        sg = np.empty(T, dtype=np.float64)
        logits = np.empty((T, self.E), dtype=np.float64)
        aid = None if adapter_id is None else _c(adapter_id, np.int32)
        sel = None if select is None else _c(select, np.int32)
        rc = _get().orc_moe_ffn(ctypes.byref(self.L), _p(x), _p(aid), T, _p(sel), _p(y), _p(idx), _p(w),
                                _p(sg), _p(logits))
        if rc != 0:
            raise ValueError("orc_moe_ffn rc=%d" % rc)
        return y, idx, w, sg, logits

    def router(self, x_bf16):
        x = _c(x_bf16, np.uint16)
        T = x.size // self.H
        logits = np.empty((T, self.E), dtype=np.float64)
        gs = np.empty(T, dtype=np.float64)
        _get().orc_router(ctypes.byref(self.L), _p(x), T, _p(logits), _p(gs))
        return logits, gs

    def block(self, x_bf16, adapter_id=None, eps=1e-6):
        x = _c(x_bf16, np.uint16)
        T = x.size // self.H
        out = np.empty((T, self.H), dtype=np.uint16)
        aid = None if adapter_id is None else _c(adapter_id, np.int32)
        rc = _get().orc_moe_block(ctypes.byref(self.L), _p(x), _p(aid), T, float(eps), _p(out))
        if rc != 0:
            raise ValueError("orc_moe_block rc=%d" % rc)
        return out


def topk(logits: np.ndarray, K: int):
    z = _c(logits, np.float64)
    T, E = z.shape
    idx = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float64)
    _get().orc_topk(_p(z), T, E, K, _p(idx), _p(w))
    return idx, w


def index_build(idx, adapter_id, E: int, n_adapters: int):
    idx = _c(idx, np.int32)
    T, K = idx.shape
    aid = None if adapter_id is None else _c(adapter_id, np.int32)
    counts = np.empty(E + 1, dtype=np.int32)
    offsets = np.empty(E + 2, dtype=np.int32)
    perm = np.empty((T * (K + 1), 4), dtype=np.int32)
    rc = _get().orc_index_build(_p(idx), _p(aid), T, K, E, n_adapters, _p(counts), _p(offsets), _p(perm))
    if rc != 0:
        raise ValueError("orc_index_build rc=%d" % rc)
    return counts, offsets, perm


def rmsnorm_bf16(x_bf16, H: int, eps: float = 1e-6) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    T = x.size // H
    out = np.empty((T, H), dtype=np.uint16)
    _get().orc_rmsnorm_bf16(_p(x), T, H, float(eps), _p(out))
    return out


class Prerouter(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("E", ctypes.c_int32), ("K", ctypes.c_int32), ("D", ctypes.c_int32),
                ("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p),
                ("wl", ctypes.c_void_p), ("bl", ctypes.c_void_p)]


def fp16_value(h: int) -> float:
    return float(_get().orc_fp16_value(int(h)))


def gelu_erf(v: float) -> float:
    return float(_get().orc_gelu_erf(float(v)))


def prerouter(H, E, K, D, w, h_bf16, exec_idx, prev_idx=None):
    """Predicted next-layer logits [T, E] of one prerouter head.  `w` maps w1 [D, H+2E],
    b1 [D], w2 [E, D], b2 [E], wl [E, H+2E], bl [E] to fp16 bit patterns (uint16); a
    missing bias is zero."""
    keep = {k: (None if w.get(k) is None else _c(w[k], np.uint16)) for k in ("w1", "b1", "w2", "b2", "wl", "bl")}
    P = Prerouter(H, E, K, D, *[_p(keep[k]) for k in ("w1", "b1", "w2", "b2", "wl", "bl")])
    h = _c(h_bf16, np.uint16)
    T = h.size // H
    ex = _c(exec_idx, np.int32)
    pv = None if prev_idx is None else _c(prev_idx, np.int32)
    z = np.empty((T, E), dtype=np.float64)
    rc = _get().orc_prerouter(ctypes.byref(P), _p(h), _p(ex), _p(pv), T, _p(z))
    if rc != 0:
        raise ValueError("orc_prerouter rc=%d" % rc)
    return z


def quant_act8(x: np.ndarray):
    """Per-row symmetric 8-bit codes (int8 [T, n]) and scales (fp32 [T]) of fp32 rows."""
    x = _c(x, np.float32)
    T, n = x.shape
    q = np.empty((T, n), dtype=np.int8)
    s = np.empty(T, dtype=np.float32)
    _get().orc_quant_act8(_p(x), T, n, _p(q), _p(s))
    return q, s


def mixed_linear_a8(packed, scales, out: int, in_: int, rho: float, x_bf16) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    T = x.size // in_
    y = np.empty((T, out), dtype=np.float64)
    _get().orc_mixed_linear_a8(_p(_c(packed, np.uint32)), _p(_c(scales, np.uint16)), out, in_, float(rho), _p(x), T,
                               _p(y))
    return y


def mixed_mlp_a8(gate, up, down, H: int, I: int, rho: float, x_bf16) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    T = x.size // H
    y = np.empty((T, H), dtype=np.float64)
    arrs = [_c(a, np.uint32 if i % 2 == 0 else np.uint16) for i, a in enumerate((*gate, *up, *down))]
    rc = _get().orc_mixed_mlp_a8(*[_p(a) for a in arrs], H, I, float(rho), _p(x), T, _p(y))
    if rc != 0:
        raise ValueError("orc_mixed_mlp_a8 rc=%d" % rc)
    return y


def mixed_block_a8(gate, up, down, H: int, I: int, rho: float, x_bf16, eps: float = 1e-6) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    T = x.size // H
    out = np.empty((T, H), dtype=np.uint16)
    arrs = [_c(a, np.uint32 if i % 2 == 0 else np.uint16) for i, a in enumerate((*gate, *up, *down))]
    rc = _get().orc_mixed_block_a8(*[_p(a) for a in arrs], H, I, float(rho), float(eps), _p(x), T, _p(out))
    if rc != 0:
        raise ValueError("orc_mixed_block_a8 rc=%d" % rc)
    return out

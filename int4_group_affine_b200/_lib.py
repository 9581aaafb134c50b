"""ctypes declarations of libmoeq's C ABI (include/moeq.h).

Loading fails with an ImportError when the shared library has not been built;
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoeq.so")

MAX_ADAPTERS = 16

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
                4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_DEVICE_INDEX", 6: "MOE_ERR_TIMEOUT"}
FMT_AFFINE_INT4, FMT_AFFINE_INT8, FMT_MIXED_TERNARY_INT4 = 0, 1, 2

# Every function the header declares, with (restype, argtypes).
P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class QTensor(ctypes.Structure):
    _fields_ = [("packed", P), ("scales", P), ("biases", P), ("n", I32), ("out", I32), ("in_", I32),
                ("bits", I32), ("group", I32)]


class MixedTensor(ctypes.Structure):
    _fields_ = [("packed", P), ("scales", P), ("out", I32), ("in_", I32), ("rho", F32)]


class LoraProj(ctypes.Structure):
    _fields_ = [("A", P), ("B", P)]


class LoraPtrs(ctypes.Structure):
    _fields_ = [(n, LoraProj) for n in ("gate", "up", "down", "s_gate", "s_up", "s_down")]


class Layer(ctypes.Structure):
    _fields_ = [("hidden", I32), ("n_experts", I32), ("top_k", I32), ("inter", I32), ("shared_inter", I32),
                ("router", QTensor), ("shared_gate", QTensor), ("gate", QTensor), ("up", QTensor),
                ("down", QTensor), ("s_gate", QTensor), ("s_up", QTensor), ("s_down", QTensor),
                ("logit_bias", P), ("n_adapters", I32), ("rank", I32), ("alpha", F32),
                ("lora", LoraPtrs * MAX_ADAPTERS)]


class Prerouter(ctypes.Structure):
    _fields_ = [("hidden", I32), ("n_experts", I32), ("top_k", I32), ("head_dim", I32), ("w1", P), ("b1", P),
                ("w2", P), ("b2", P), ("wl", P), ("bl", P)]


PQ, PM, PL, PLP = (ctypes.POINTER(QTensor), ctypes.POINTER(MixedTensor), ctypes.POINTER(Layer),
                   ctypes.POINTER(LoraPtrs))

SIGNATURES = {
    "moe_version": (ctypes.c_int, []),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_quant_pack": (ctypes.c_int, [ctypes.c_int, P, I64, I32, I32, F32, P, P, P, P]),
    "moe_mixed_words": (I64, [I32, I32, F32]),
    "moe_dequant": (ctypes.c_int, [PQ, P, P]),
    "moe_mixed_dequant": (ctypes.c_int, [PM, P, P]),
    "moe_router_topk": (ctypes.c_int, [P, PQ, PQ, P, I32, I32, I32, I32, P, P, P, P, P]),
    "moe_index_workspace_bytes": (SZ, [I32, I32, I32, I32]),
    "moe_index_build": (ctypes.c_int, [P, P, I32, I32, I32, I32, P, P, P, P, SZ, P]),
    "lora_set_adapters": (ctypes.c_int, [PL, I32, I32, F32, PLP]),
    "moe_ffn_workspace_bytes": (SZ, [PL, I32]),
    "moe_workspace_init": (ctypes.c_int, [P, SZ, P]),
    "moe_ffn_forward": (ctypes.c_int, [PL, P, P, I32, P, P, SZ, P]),
    "moe_ffn_forward_host": (ctypes.c_int, [PL, P, P, I32, P, P, SZ, P]),
    "moe_ffn_forward_static": (ctypes.c_int, [PL, P, P, I32, P, P]),
    "moe_block_forward": (ctypes.c_int, [PL, P, P, I32, F32, P, P, SZ, P]),
    "moe_rmsnorm": (ctypes.c_int, [P, I32, I32, F32, P, P]),
    "moe_get_device_status": (ctypes.c_int, [P, P, ctypes.POINTER(I32)]),
    "moe_mixed_linear": (ctypes.c_int, [PM, P, I32, P, P]),
    "moe_mixed_mlp_workspace_bytes": (SZ, [I32, I32, I32]),
    "moe_mixed_mlp_forward": (ctypes.c_int, [PM, PM, PM, P, I32, I32, F32, P, P, SZ, P]),
    "moe_ffn_static_device_status": (ctypes.c_int, [P, ctypes.POINTER(I32)]),
    "moe_ffn_routing": (ctypes.c_int, [PL, I32, P, SZ, P, P, P]),
    "moe_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
    "moe_set_decode_path": (ctypes.c_int, [ctypes.c_int]),
    "moe_decode_path": (ctypes.c_int, []),
    "moe_wait_limit_ns": (ctypes.c_uint64, []),
    "moe_ffn_forward_select": (ctypes.c_int, [PL, P, P, P, I32, P, P, SZ, P]),
    "moe_prerouter_workspace_bytes": (SZ, [ctypes.POINTER(Prerouter), I32]),
    "moe_prerouter_forward": (ctypes.c_int, [ctypes.POINTER(Prerouter), P, P, P, I32, P, P, P, SZ, P]),
    "moe_act8_quant": (ctypes.c_int, [P, I32, I32, P, P, P]),
    "moe_mixed_linear_a8_workspace_bytes": (SZ, [I32, I32]),
    "moe_mixed_linear_a8": (ctypes.c_int, [PM, P, I32, P, P, SZ, P]),
    "moe_mixed_mlp_a8_workspace_bytes": (SZ, [I32, I32, I32]),
    "moe_mixed_mlp_forward_a8": (ctypes.c_int, [PM, PM, PM, P, I32, I32, F32, P, P, SZ, P]),
    "moe_experts_workspace_bytes": (SZ, [PL, I32]),
    "moe_experts_forward": (ctypes.c_int, [PL, P, P, P, I32, P, P, SZ, P]),
    "moe_ep_dispatch": (ctypes.c_int, [P, P, P, I32, I32, I32, I32, I32, I32, P, P, P, P, P, P]),
    "moe_ep_combine": (ctypes.c_int, [P, P, P, P, P, I32, I32, I32, P, P]),
    "moe_timing_kinds": (ctypes.c_int, []),
    "moe_timing_kind_name": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_timing_enable": (ctypes.c_int, [ctypes.c_int]),
    "moe_timing_collect": (ctypes.c_int, [P, P, I32]),
}

_lib = None


def lib():
    """The loaded libmoeq (raises ImportError if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libmoeq.so is not built: run `python -m int4_group_affine_b200.build` "
                              "(nvcc, sm_100a); there is no CPU implementation")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib

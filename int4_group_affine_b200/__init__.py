"""Python binding of libmoeq, the sm_100a int4 group-affine MoE expert FFN library.

Functions carry the names of the C entry points (include/moeq.h) and only
marshal arguments: torch tensors become device pointers, ``stream=None`` means
torch's current CUDA stream, and a non-zero status raises ``MoeError``.
Every computation runs in the CUDA kernels of libmoeq.so.
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import (FMT_AFFINE_INT4, FMT_AFFINE_INT8, FMT_MIXED_TERNARY_INT4, Layer, LoraProj, LoraPtrs,
                   MixedTensor, Prerouter, QTensor, STATUS_NAMES)

__all__ = [
    "MoeError", "QTensor", "MixedTensor", "LoraProj", "LoraPtrs", "Layer",
    "FMT_AFFINE_INT4", "FMT_AFFINE_INT8", "FMT_MIXED_TERNARY_INT4",
    "moe_version", "moe_quant_pack", "moe_mixed_words", "moe_dequant", "moe_mixed_dequant", "moe_router_topk",
    "moe_index_workspace_bytes", "moe_index_build", "lora_set_adapters", "moe_ffn_workspace_bytes",
    "moe_workspace_init", "moe_ffn_forward", "moe_block_forward", "moe_rmsnorm", "moe_get_device_status",
    "moe_mixed_linear", "moe_mixed_mlp_workspace_bytes", "moe_mixed_mlp_forward",
    "moe_timing_enable", "moe_timing_collect", "moe_ffn_forward_static", "moe_ffn_static_device_status",
    "moe_ffn_routing", "moe_set_wait_limit_ns", "moe_wait_limit_ns", "Prerouter", "moe_ffn_forward_select",
    "moe_prerouter_workspace_bytes", "moe_prerouter_forward", "moe_act8_quant",
    "moe_mixed_linear_a8_workspace_bytes", "moe_mixed_linear_a8", "moe_mixed_mlp_a8_workspace_bytes",
    "moe_mixed_mlp_forward_a8", "moe_experts_workspace_bytes", "moe_experts_forward", "moe_ep_dispatch",
    "moe_ep_combine", "moe_ffn_forward_host", "moe_set_decode_path", "moe_decode_path", "DECODE_AUTO", "DECODE_CHAIN", "DECODE_BARRIER", "DECODE_CLUSTER",
]

DECODE_AUTO, DECODE_CHAIN, DECODE_BARRIER, DECODE_CLUSTER = 0, 1, 2, 3


class MoeError(RuntimeError):
    def __init__(self, name, status):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (name, STATUS_NAMES.get(status, "?"), status))


def _check(name, st):
    if st != 0:
        raise MoeError(name, st)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ref(s):
    return None if s is None else ctypes.byref(s)


def moe_version() -> int:
    return _lib.lib().moe_version()


def moe_quant_pack(fmt, W, rows, in_, group, rho, packed, scales, biases, stream=None):
    _check("moe_quant_pack", _lib.lib().moe_quant_pack(fmt, _ptr(W), rows, in_, group, rho, _ptr(packed),
                                                       _ptr(scales), _ptr(biases), _stream(stream)))


def moe_mixed_words(out, in_, rho) -> int:
    return int(_lib.lib().moe_mixed_words(out, in_, rho))


def moe_dequant(t: QTensor, w_hat, stream=None):
    _check("moe_dequant", _lib.lib().moe_dequant(ctypes.byref(t), _ptr(w_hat), _stream(stream)))


def moe_mixed_dequant(t: MixedTensor, w_hat, stream=None):
    _check("moe_mixed_dequant", _lib.lib().moe_mixed_dequant(ctypes.byref(t), _ptr(w_hat), _stream(stream)))


def moe_router_topk(x, router: QTensor, shared_gate, logit_bias, T, H, E, K, topk_idx, topk_w, shared_scale,
                    logits, stream=None):
    _check("moe_router_topk", _lib.lib().moe_router_topk(
        _ptr(x), ctypes.byref(router), _ref(shared_gate), _ptr(logit_bias), T, H, E, K, _ptr(topk_idx),
        _ptr(topk_w), _ptr(shared_scale), _ptr(logits), _stream(stream)))


def moe_index_workspace_bytes(T, K, E, n_adapters) -> int:
    return int(_lib.lib().moe_index_workspace_bytes(T, K, E, n_adapters))


def moe_index_build(topk_idx, adapter_id, T, K, E, n_adapters, counts, offsets, perm, workspace, ws_bytes,
                    stream=None):
    _check("moe_index_build", _lib.lib().moe_index_build(
        _ptr(topk_idx), _ptr(adapter_id), T, K, E, n_adapters, _ptr(counts), _ptr(offsets), _ptr(perm),
        _ptr(workspace), ws_bytes, _stream(stream)))


def lora_set_adapters(layer: Layer, n_adapters, rank, alpha, sets):
    arr = None
    if n_adapters > 0:
        arr = (LoraPtrs * n_adapters)(*sets)
    _check("lora_set_adapters", _lib.lib().lora_set_adapters(ctypes.byref(layer), n_adapters, rank, alpha, arr))


def moe_ffn_workspace_bytes(layer: Layer, T) -> int:
    return int(_lib.lib().moe_ffn_workspace_bytes(ctypes.byref(layer), T))


def moe_workspace_init(workspace, ws_bytes, stream=None):
    _check("moe_workspace_init", _lib.lib().moe_workspace_init(_ptr(workspace), ws_bytes, _stream(stream)))


def moe_ffn_forward(layer: Layer, x, adapter_id, T, y, workspace, ws_bytes, stream=None):
    _check("moe_ffn_forward", _lib.lib().moe_ffn_forward(ctypes.byref(layer), _ptr(x), _ptr(adapter_id), T,
                                                         _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)))


def _hptr(t):
    """Address of a page-locked host tensor (or a raw address)."""
    if isinstance(t, int):
        return t
    if t.is_cuda or not t.is_pinned():
        raise ValueError("expected a pinned host tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def moe_ffn_forward_host(layer: Layer, x_host, adapter_id, T, y_host, workspace, ws_bytes, stream=None):
    """moe_ffn_forward with x and y in mapped page-locked host memory (pinned torch tensors or
    raw host addresses); 1 to 8 tokens."""
    _check("moe_ffn_forward_host", _lib.lib().moe_ffn_forward_host(ctypes.byref(layer), _hptr(x_host),
                                                                   _ptr(adapter_id), T, _hptr(y_host),
                                                                   _ptr(workspace), ws_bytes, _stream(stream)))


def moe_block_forward(layer: Layer, x, adapter_id, T, eps, x_out, workspace, ws_bytes, stream=None):
    _check("moe_block_forward", _lib.lib().moe_block_forward(ctypes.byref(layer), _ptr(x), _ptr(adapter_id), T,
                                                             eps, _ptr(x_out), _ptr(workspace), ws_bytes,
                                                             _stream(stream)))


def moe_rmsnorm(x, T, H, eps, xn, stream=None):
    _check("moe_rmsnorm", _lib.lib().moe_rmsnorm(_ptr(x), T, H, eps, _ptr(xn), _stream(stream)))


def moe_get_device_status(workspace, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("moe_get_device_status", _lib.lib().moe_get_device_status(_ptr(workspace), _stream(stream),
                                                                     ctypes.byref(v)))
    return int(v.value)


def moe_mixed_linear(W: MixedTensor, x, T, y, stream=None):
    _check("moe_mixed_linear", _lib.lib().moe_mixed_linear(ctypes.byref(W), _ptr(x), T, _ptr(y),
                                                           _stream(stream)))


def moe_mixed_mlp_workspace_bytes(H, I, T) -> int:
    return int(_lib.lib().moe_mixed_mlp_workspace_bytes(H, I, T))


def moe_mixed_mlp_forward(gate: MixedTensor, up: MixedTensor, down: MixedTensor, x, T, residual, eps, y,
                          workspace, ws_bytes, stream=None):
    _check("moe_mixed_mlp_forward", _lib.lib().moe_mixed_mlp_forward(
        ctypes.byref(gate), ctypes.byref(up), ctypes.byref(down), _ptr(x), T, residual, eps, _ptr(y),
        _ptr(workspace), ws_bytes, _stream(stream)))


def moe_timing_enable(enable: bool):
    _check("moe_timing_enable", _lib.lib().moe_timing_enable(1 if enable else 0))


def moe_timing_collect() -> dict:
    """{kernel kind: (total ms, launches)} recorded since the last collect (synchronises)."""
    L = _lib.lib()
    n = L.moe_timing_kinds()
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_int32 * n)()
    _check("moe_timing_collect", L.moe_timing_collect(ms, cnt, n))
    return {L.moe_timing_kind_name(k).decode(): (float(ms[k]), int(cnt[k])) for k in range(n) if cnt[k]}


def moe_ffn_forward_static(layer: Layer, x, adapter_id, T, y, stream=None):
    """moe_ffn_forward with the library's built-in device workspace (no allocation anywhere)."""
    _check("moe_ffn_forward_static", _lib.lib().moe_ffn_forward_static(ctypes.byref(layer), _ptr(x),
                                                                       _ptr(adapter_id), T, _ptr(y),
                                                                       _stream(stream)))


def moe_ffn_static_device_status(stream=None) -> int:
    """Read and clear the status word of the built-in workspace (synchronises)."""
    v = ctypes.c_int32(0)
    _check("moe_ffn_static_device_status", _lib.lib().moe_ffn_static_device_status(_stream(stream),
                                                                                   ctypes.byref(v)))
    return int(v.value)


def moe_ffn_routing(layer: Layer, T, workspace, ws_bytes, topk_idx, topk_w, stream=None):
    """Copy the routing (indices, weights) the last forward on this workspace used."""
    _check("moe_ffn_routing", _lib.lib().moe_ffn_routing(ctypes.byref(layer), T, _ptr(workspace), ws_bytes,
                                                         _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def moe_set_wait_limit_ns(ns: int):
    _check("moe_set_wait_limit_ns", _lib.lib().moe_set_wait_limit_ns(int(ns)))


def moe_wait_limit_ns() -> int:
    return int(_lib.lib().moe_wait_limit_ns())


def moe_ffn_forward_select(layer: Layer, x, adapter_id, select, T, y, workspace, ws_bytes, stream=None):
    """moe_ffn_forward with each token's expert set given (select [T, K] int32)."""
    _check("moe_ffn_forward_select", _lib.lib().moe_ffn_forward_select(
        ctypes.byref(layer), _ptr(x), _ptr(adapter_id), _ptr(select), T, _ptr(y), _ptr(workspace), ws_bytes,
        _stream(stream)))


def moe_prerouter_workspace_bytes(head: Prerouter, T) -> int:
    return int(_lib.lib().moe_prerouter_workspace_bytes(ctypes.byref(head), T))


def moe_prerouter_forward(head: Prerouter, h, exec_idx, prev_idx, T, logits, pred_idx, workspace, ws_bytes,
                          stream=None):
    _check("moe_prerouter_forward", _lib.lib().moe_prerouter_forward(
        ctypes.byref(head), _ptr(h), _ptr(exec_idx), _ptr(prev_idx), T, _ptr(logits), _ptr(pred_idx),
        _ptr(workspace), ws_bytes, _stream(stream)))


def moe_act8_quant(x, T, n, q, s, stream=None):
    _check("moe_act8_quant", _lib.lib().moe_act8_quant(_ptr(x), T, n, _ptr(q), _ptr(s), _stream(stream)))


def moe_mixed_linear_a8_workspace_bytes(in_, T) -> int:
    return int(_lib.lib().moe_mixed_linear_a8_workspace_bytes(in_, T))


def moe_mixed_linear_a8(W: MixedTensor, x, T, y, workspace, ws_bytes, stream=None):
    _check("moe_mixed_linear_a8", _lib.lib().moe_mixed_linear_a8(ctypes.byref(W), _ptr(x), T, _ptr(y),
                                                                 _ptr(workspace), ws_bytes, _stream(stream)))


def moe_mixed_mlp_a8_workspace_bytes(H, I, T) -> int:
    return int(_lib.lib().moe_mixed_mlp_a8_workspace_bytes(H, I, T))


def moe_mixed_mlp_forward_a8(gate: MixedTensor, up: MixedTensor, down: MixedTensor, x, T, residual, eps, y,
                             workspace, ws_bytes, stream=None):
    _check("moe_mixed_mlp_forward_a8", _lib.lib().moe_mixed_mlp_forward_a8(
        ctypes.byref(gate), ctypes.byref(up), ctypes.byref(down), _ptr(x), T, residual, eps, _ptr(y),
        _ptr(workspace), ws_bytes, _stream(stream)))


def moe_experts_workspace_bytes(layer: Layer, N) -> int:
    return int(_lib.lib().moe_experts_workspace_bytes(ctypes.byref(layer), N))


def moe_experts_forward(layer: Layer, x, expert, adapter_id, N, y, workspace, ws_bytes, stream=None):
    """y[n] = expert[n]'s SwiGLU FFN (with its LoRA delta) of x[n]; no router, no shared expert."""
    _check("moe_experts_forward", _lib.lib().moe_experts_forward(
        ctypes.byref(layer), _ptr(x), _ptr(expert), _ptr(adapter_id), N, _ptr(y), _ptr(workspace), ws_bytes,
        _stream(stream)))


def moe_ep_dispatch(x, topk_idx, adapter_id, n_adapters, T, K, H, E, G, pos, counts, send_x, send_meta, status,
                    stream=None):
    _check("moe_ep_dispatch", _lib.lib().moe_ep_dispatch(
        _ptr(x), _ptr(topk_idx), _ptr(adapter_id), n_adapters, T, K, H, E, G, _ptr(pos), _ptr(counts), _ptr(send_x),
        _ptr(send_meta), _ptr(status), _stream(stream)))


def moe_ep_combine(ret, pos, topk_w, shared, shared_scale, T, K, H, y, stream=None):
    _check("moe_ep_combine", _lib.lib().moe_ep_combine(
        _ptr(ret), _ptr(pos), _ptr(topk_w), _ptr(shared), _ptr(shared_scale), T, K, H, _ptr(y), _stream(stream)))


def moe_set_decode_path(path: int):
    _check("moe_set_decode_path", _lib.lib().moe_set_decode_path(int(path)))


def moe_decode_path() -> int:
    return int(_lib.lib().moe_decode_path())

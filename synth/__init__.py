"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

Nothing here performs quantisation or MoE arithmetic: it only draws numbers.
Two generators are offered:

* ``normal`` / ``uniform`` / ``randint`` / ``bf16``: host arrays from the
  counter-based SplitMix64 + Box-Muller generator in ``synth.c`` (bit
  reproducible for a given seed and stream name, independent of thread count).
* ``device_normal``: bulk weights drawn directly on a CUDA device with torch's
  seeded Philox generator, for workloads too large to draw on the host (the
  multi-gigabyte layer copies of the benchmark).  Values a CPU check needs are
  copied back from the device.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _get():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_stream_key.restype = ctypes.c_uint64
        lib.synth_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_char_p]
        lib.synth_uniform_f64.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_double,
                                         ctypes.c_double, ctypes.c_void_p]
        lib.synth_outliers_f32.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_double,
                                           ctypes.c_double, ctypes.c_void_p]
        lib.synth_uniform_int.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_void_p]
        lib.synth_f32_to_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        _lib = lib
    return _lib


def key(seed: int, name: str) -> int:
    return int(_get().synth_stream_key(ctypes.c_uint64(seed), name.encode()))


def normal(seed: int, name: str, shape, mean: float = 0.0, std: float = 1.0,
           outlier_prob: float = 0.0, outlier_factor: float = 1.0) -> np.ndarray:
    """fp32 Normal(mean, std) array; optionally each element scaled by
    ``outlier_factor`` with probability ``outlier_prob`` (own stream)."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.float32)
    lib = _get()
    if n:
        lib.synth_normal_f32(key(seed, name), n, mean, std, out.ctypes.data)
        if outlier_prob > 0.0:
            lib.synth_outliers_f32(key(seed, name + "/outliers"), n, outlier_prob,
                                   outlier_factor, out.ctypes.data)
    return out.reshape(shape)


def uniform(seed: int, name: str, shape) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.float64)
    if n:
        _get().synth_uniform_f64(key(seed, name), n, out.ctypes.data)
    return out.reshape(shape)


def randint(seed: int, name: str, shape, lo: int, hi: int) -> np.ndarray:
    """int32 uniform on the closed range [lo, hi]."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.int32)
    if n:
        _get().synth_uniform_int(key(seed, name), n, lo, hi, out.ctypes.data)
    return out.reshape(shape)


def bf16(a: np.ndarray) -> np.ndarray:
    """Round an fp32 array to bf16 (nearest even); returns the uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    if a.size:
        _get().synth_f32_to_bf16(a.ctypes.data, a.size, out.ctypes.data)
    return out


def fp16(a: np.ndarray) -> np.ndarray:
    """Round to IEEE binary16 (numpy's nearest-even conversion); returns the uint16 bit patterns."""
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed: int, name: str, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    return bf16(normal(seed, name, shape, mean, std))


def device_normal(seed: int, name: str, shape, std: float, device, outlier_prob: float = 0.0,
                  outlier_factor: float = 1.0):
    """fp32 Normal(0, std) tensor drawn on ``device`` by torch's seeded Philox
    generator (stream chosen from ``seed`` and ``name``)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(key(seed, name) & 0x7FFFFFFFFFFFFFFF)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    if outlier_prob > 0.0:
        u = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
        t = torch.where(u < outlier_prob, t * outlier_factor, t)
    return t

"""Seeded synthetic inputs and the workload table for the temporal modules.

This package is the one piece shared by the fp64 oracle's tests and the CUDA
path's tests and benchmark.  It holds no arithmetic of the temporal modules:
only the workload shapes, the value distributions and a counter-based random
number generator (SplitMix64 + Box-Muller, defined in ``gen.c``), so that any
element of any input tensor can be regenerated from (seed, tensor id, index).

Shapes follow the Video-Infinity write-up ("Video-Infinity: Distributed Long
Video Generation", clip parallelism and experiment paragraphs): a 512x320
video at a /8 latent gives P = 40x64 = 2560 positions at the top U-Net level,
/2 and /4 of that at the lower levels with C = 320/640/1280 channels; F is the
frame count, cut into N clips of L = F/N frames.

Distributions: N(mean, var) with the second parameter a variance (the conv
weight's 1/(k C) is a fan-in variance).  All inputs are i.i.d.; bf16 workloads
round every input once, to nearest even, and both sides consume the rounded
values.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")

# Tensor ids: one independent random stream per input tensor.
TID = {"q": 1, "k": 2, "v": 3, "conv_x": 4, "conv_w": 5, "conv_b": 6,
       "gn_x": 7, "gn_gamma": 8, "gn_beta": 9,
       "attn_x": 10, "w_qkv": 11, "b_qkv": 12, "w_out": 13, "b_out": 14}


def build(force: bool = False) -> str:
    """Compile gen.c into libsynth.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.synth_splitmix64_at.restype = u64
        L.synth_splitmix64_at.argtypes = [u64, u64]
        L.synth_stream_key.restype = u64
        L.synth_stream_key.argtypes = [u64, u64]
        for name in ("synth_normal_f64", "synth_normal_f32", "synth_normal_bf16"):
            fn = getattr(L, name)
            fn.restype = None
            fn.argtypes = [vp, i64, i64, u64, u64, dbl, dbl]
        L.synth_f32_to_bf16.argtypes = [vp, vp, i64]
        L.synth_bf16_to_f32.argtypes = [vp, vp, i64]
        _lib = L
    return _lib


def splitmix64_at(seed: int, n: int) -> int:
    return int(lib().synth_splitmix64_at(seed, n))


def normal(shape, tid: int, mean: float = 0.0, std: float = 1.0, seed: int = 0,
           dtype: str = "f64", first: int = 0) -> np.ndarray:
    """Draw elements [first, first+prod(shape)) of stream (seed, tid).

    dtype "f64" returns unrounded doubles, "f32" float32 values, "bf16" the
    bf16 bit patterns as uint16 (use ``bf16_to_f32`` to read them).
    """
    n = int(np.prod(shape)) if len(shape) else 1
    if dtype == "f64":
        out = np.empty(n, np.float64)
        lib().synth_normal_f64(out.ctypes.data, n, first, seed, tid, mean, std)
    elif dtype == "f32":
        out = np.empty(n, np.float32)
        lib().synth_normal_f32(out.ctypes.data, n, first, seed, tid, mean, std)
    elif dtype == "bf16":
        out = np.empty(n, np.uint16)
        lib().synth_normal_bf16(out.ctypes.data, n, first, seed, tid, mean, std)
    else:
        raise ValueError(dtype)
    return out.reshape(shape)


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().synth_f32_to_bf16(a.ctypes.data, out.ctypes.data, a.size)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.uint16)
    out = np.empty(a.shape, np.float32)
    lib().synth_bf16_to_f32(a.ctypes.data, out.ctypes.data, a.size)
    return out


def values_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """The exact values an input array holds, as float64."""
    if dtype == "bf16":
        return bf16_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


@dataclass(frozen=True)
class Workload:
    """One temporal-module workload: latent [P positions][F frames][C channels]."""
    name: str
    dtype: str            # "f32" or "bf16" (I/O type; arithmetic is fp32 on the GPU)
    F: int                # frames
    N: int                # clips (L = F / N frames each)
    P: int                # spatial positions H' x W'
    C: int                # channels = heads * d
    heads: int
    d: int
    n_pre: int = 8
    n_post: int = 8
    n_global: int = 16
    k: int = 3            # temporal conv kernel size
    groups: int = 32
    eps: float = 1e-5
    seed: int = 0
    hw: tuple = field(default=(0, 0))   # latent H' x W' (documentation only)

    @property
    def L(self) -> int:
        return self.F // self.N

    @property
    def tokens(self) -> int:
        return self.F * self.P

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def act_shape(self):
        return (self.P, self.F, self.C)

    @property
    def act_bytes(self) -> int:
        return self.P * self.F * self.C * self.elem_bytes

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five workloads.  Sizes follow the write-up's 512x320 video at a /8 latent
# (P = 40x64) and two lower U-Net levels; every one uses d = 64, 8/8/16 context
# frames, k = 3 and 32 GroupNorm groups (8 for the tiny fp32 case).
WORKLOADS = [
    Workload("tiny_f32_F32_P64_C64", "f32", F=32, N=4, P=64, C=64, heads=1, d=64, groups=8,
             hw=(8, 8)),
    Workload("bf16_F128_P2560_C320", "bf16", F=128, N=8, P=2560, C=320, heads=5, d=64, hw=(40, 64)),
    Workload("bf16_F1024_P2560_C320", "bf16", F=1024, N=64, P=2560, C=320, heads=5, d=64,
             hw=(40, 64)),
    Workload("bf16_F1024_P640_C640", "bf16", F=1024, N=64, P=640, C=640, heads=10, d=64,
             hw=(20, 32)),
    Workload("bf16_F2304_P160_C1280", "bf16", F=2304, N=144, P=160, C=1280, heads=20, d=64,
             hw=(10, 16)),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def dist(w: Workload, tensor: str):
    """(mean, std) of each input tensor; the distributions are stated as N(mean, variance)."""
    return {
        "q": (0.0, 1.0), "k": (0.0, 1.0), "v": (0.0, 1.0),
        "conv_x": (0.0, 1.0),
        "conv_w": (0.0, math.sqrt(1.0 / (w.k * w.C))),
        "conv_b": (0.0, math.sqrt(0.01)),
        "gn_x": (0.5, math.sqrt(2.0)),
        "gn_gamma": (1.0, math.sqrt(0.1)),
        "gn_beta": (0.0, math.sqrt(0.1)),
        # temporal-attention module: input and Linear layers (fan-in variance)
        "attn_x": (0.0, 1.0),
        "w_qkv": (0.0, math.sqrt(1.0 / w.C)), "b_qkv": (0.0, math.sqrt(0.01)),
        "w_out": (0.0, math.sqrt(1.0 / w.C)), "b_out": (0.0, math.sqrt(0.01)),
    }[tensor]


def shape_of(w: Workload, tensor: str):
    if tensor in ("q", "k", "v", "conv_x", "gn_x", "attn_x"):
        return w.act_shape
    if tensor == "conv_w":
        return (w.C, w.C, w.k)        # [C_out][C_in][k], PyTorch Conv1d order
    if tensor == "w_qkv":
        return (3 * w.C, w.C)         # rows Wq, Wk, Wv; PyTorch Linear order
    if tensor == "b_qkv":
        return (3 * w.C,)
    if tensor == "w_out":
        return (w.C, w.C)
    return (w.C,)                     # conv_b, gn_gamma, gn_beta


def make(w: Workload, tensor: str, dtype: str | None = None) -> np.ndarray:
    """Generate one input tensor of workload w in its I/O dtype (uint16 = bf16 bits)."""
    mean, std = dist(w, tensor)
    return normal(shape_of(w, tensor), TID[tensor], mean, std, seed=w.seed,
                  dtype=dtype or w.dtype)

"""fp64 CPU oracle for the clip-parallel temporal modules (Video-Infinity).

TEST INFRASTRUCTURE ONLY: the plain, slow statement of what the temporal
modules compute, used to check the CUDA library.  Only ``tests/``, the
package's ``smoke()`` check and ``bench.py``'s CPU-baseline leg may import it;
the product path never does, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, OpenMP over
independent positions); this module marshals numpy arrays to it.  Inputs are
given in their I/O dtype (float32 values, or bf16 bit patterns as uint16) and
widened exactly; outputs are float64.

Parity status (each function is pinned by tests/test_oracle_*.py):
  - key_frames / dual_attn: pinned by hand-derived key lists
    (tests/golden/attn_key_frames.txt), the q = 0 multiset mean, the
    orthonormal-key membership probe, constant V, and library SDPA in the
    N = 1 / no-context special cases.
  - temporal_conv: pinned by library conv1d with zero padding, the identity
    and shift kernels, and linearity.
  - groupnorm_global: pinned by library group_norm on the whole tensor for
    several clip counts, a constant group, and the moment identities.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPE_CODE = {"f32": 0, "bf16": 1, "f64": 2}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
                               "-fno-fast-math", "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_key_frames.restype = i32
        L.oracle_key_frames.argtypes = [i32] * 6 + [vp]
        L.oracle_dual_attn.restype = None
        L.oracle_dual_attn.argtypes = [vp, vp, vp, i32, vp] + [i32] * 8 + [vp, i32, i32]
        L.oracle_temporal_conv.restype = None
        L.oracle_temporal_conv.argtypes = [vp, vp, vp, i32, vp] + [i32] * 5 + [vp, i32, i32, i32]
        L.oracle_groupnorm_global.restype = None
        L.oracle_groupnorm_global.argtypes = ([vp, vp, vp, i32, vp, vp, vp] + [i32] * 5 +
                                              [dbl, vp, i32, i32])
        L.oracle_max_threads.restype = i32
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _dtype_of(a: np.ndarray, allow_f64: bool = False) -> str:
    if a.dtype == np.uint16:
        return "bf16"
    if a.dtype == np.float32:
        return "f32"
    if allow_f64 and a.dtype == np.float64:
        return "f64"
    raise TypeError(f"oracle inputs are float32 values or bf16 bits (uint16), got {a.dtype}")


def _c(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a)


def _positions(P: int, positions) -> np.ndarray:
    if positions is None:
        positions = np.arange(P)
    pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int32))
    if pos.size and (pos.min() < 0 or pos.max() >= P):
        raise ValueError("position out of range")
    return pos


def key_frames(i: int, F: int, N: int, n_pre: int, n_post: int, n_global: int) -> list[int]:
    """Key/value frame list of clip i: own, C_pre, C_post, C_global (duplicates kept)."""
    L = F // N
    buf = np.zeros(L + n_pre + n_post + max(n_global, 0), np.int32)
    n = lib().oracle_key_frames(i, F, N, n_pre, n_post, n_global, buf.ctypes.data)
    return [int(t) for t in buf[:n]]


def _check_common(F, N):
    if F <= 0 or N <= 0 or F % N:
        raise ValueError("F must be a positive multiple of N")


def dual_attn(q, k, v, F, N, heads, d, n_pre=8, n_post=8, n_global=16, positions=None,
              nthreads=0) -> np.ndarray:
    """Dual-domain attention over [P][F][heads*d] inputs -> [n_pos][F][C] float64.

    Inputs may also be float64 (the exact output of another oracle module)."""
    q, k, v = _c(q), _c(k), _c(v)
    dt = _dtype_of(q, allow_f64=True)
    assert _dtype_of(k, allow_f64=True) == dt and _dtype_of(v, allow_f64=True) == dt
    _check_common(F, N)
    C = heads * d
    P = q.size // (F * C)
    assert q.size == P * F * C == k.size == v.size
    L = F // N
    # Neighbour context comes from the adjacent clip only, so it is at most L
    # frames; with one clip there are no neighbours and the sizes are unused.
    if n_pre < 0 or n_post < 0 or not 0 <= n_global <= F or (N > 1 and max(n_pre, n_post) > L):
        raise ValueError("context sizes out of range")
    pos = _positions(P, positions)
    out = np.zeros((pos.size, F, C), np.float64)
    lib().oracle_dual_attn(q.ctypes.data, k.ctypes.data, v.ctypes.data, DTYPE_CODE[dt],
                           out.ctypes.data, F, N, P, heads, d, n_pre, n_post, n_global,
                           pos.ctypes.data, pos.size, nthreads)
    return out


def temporal_conv(x, w, b, F, N, k=3, positions=None, nthreads=0) -> np.ndarray:
    """Clip-padded temporal conv over [P][F][C] -> [n_pos][F][C] float64.

    x may also be float64 (the exact output of another oracle module)."""
    x, w, b = _c(x), _c(w), _c(b)
    xdt = _dtype_of(x, allow_f64=True)
    dt = _dtype_of(w)
    assert _dtype_of(b) == dt
    _check_common(F, N)
    C = b.size
    P = x.size // (F * C)
    assert x.size == P * F * C and w.size == C * C * k
    if k % 2 == 0 or k // 2 > F // N:
        raise ValueError("k must be odd with k//2 <= L")
    pos = _positions(P, positions)
    y = np.zeros((pos.size, F, C), np.float64)
    lib().oracle_temporal_conv(x.ctypes.data, w.ctypes.data, b.ctypes.data, DTYPE_CODE[dt],
                               y.ctypes.data, F, N, P, C, k, pos.ctypes.data, pos.size, nthreads,
                               DTYPE_CODE[xdt])
    return y


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Values rounded to bf16 (via fp32, round to nearest even), as float64."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def groupnorm_conv(x, gamma, beta, w, b, F, N, groups, eps=1e-5, k=3, positions=None,
                   nthreads=0, intermediate="f64") -> np.ndarray:
    """Temporal conv of the global-statistics GroupNorm of x (the ResNet-module
    order: normalise, then convolve along frames), composed from the two
    modules above.  intermediate="f64" feeds the exact GroupNorm output to the
    conv; "bf16" rounds it to bf16 first, as a pipeline whose modules exchange
    bf16 tensors does.  -> [n_pos][F][C] float64."""
    P = x.size // (F * gamma.size)
    pos = _positions(P, positions)
    z, _, _ = groupnorm_global(x, gamma, beta, F, N, groups, eps, positions=pos,
                               nthreads=nthreads)
    if intermediate == "bf16":
        z = round_bf16(z)
    return temporal_conv(z, w, b, F, N, k, nthreads=nthreads)


def groupnorm_global(x, gamma, beta, F, N, groups, eps=1e-5, positions=None, nthreads=0,
                     want_y=True):
    """Global-statistics GroupNorm -> (y [n_pos][F][C] float64 or None, mean[G], var[G])."""
    x, gamma, beta = _c(x), _c(gamma), _c(beta)
    dt = _dtype_of(x)
    assert _dtype_of(gamma) == dt and _dtype_of(beta) == dt
    _check_common(F, N)
    C = gamma.size
    P = x.size // (F * C)
    assert x.size == P * F * C and C % groups == 0
    pos = _positions(P, positions)
    y = np.zeros((pos.size, F, C), np.float64) if want_y else None
    mean = np.zeros(groups, np.float64)
    var = np.zeros(groups, np.float64)
    lib().oracle_groupnorm_global(x.ctypes.data, gamma.ctypes.data, beta.ctypes.data,
                                  DTYPE_CODE[dt], y.ctypes.data if want_y else None,
                                  mean.ctypes.data, var.ctypes.data, F, N, P, C, groups,
                                  float(eps), pos.ctypes.data, pos.size, nthreads)
    return y, mean, var


def _as_f32_exact(a: np.ndarray) -> np.ndarray:
    """bf16-representable float64 values as float32 (exact)."""
    return np.ascontiguousarray(a, dtype=np.float32)


def temporal_attention(x, w_qkv, b_qkv, w_out, b_out, F, N, heads, d, n_pre=8, n_post=8,
                       n_global=16, positions=None, nthreads=0, intermediate="bf16"):
    """Temporal attention module: per-frame input projections (Linear layers,
    here single-tap temporal convs), dual-domain attention, output projection.
    intermediate="bf16" rounds q, k, v and the attention output to bf16 as the
    separate stages exchange them; "f64" keeps them exact.  -> [n_pos][F][C]."""
    C = heads * d
    P = x.size // (F * C)
    pos = _positions(P, positions)
    rnd = (lambda a: _as_f32_exact(round_bf16(a))) if intermediate == "bf16" else (lambda a: a)
    proj = []
    for i in range(3):
        wi = np.ascontiguousarray(w_qkv[i * C:(i + 1) * C]).reshape(C, C, 1)
        bi = np.ascontiguousarray(b_qkv[i * C:(i + 1) * C])
        proj.append(rnd(temporal_conv(x, wi, bi, F, N, 1, positions=pos, nthreads=nthreads)))
    a = rnd(dual_attn(*proj, F, N, heads, d, n_pre, n_post, n_global, nthreads=nthreads))
    wo = np.ascontiguousarray(w_out).reshape(C, C, 1)
    return temporal_conv(a, wo, np.ascontiguousarray(b_out), F, N, 1, nthreads=nthreads)


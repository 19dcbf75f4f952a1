"""Shared helpers of the GPU parity tests: seeded inputs, device upload through
torch, and the comparison rule against the fp64 oracle.

Tolerances (max abs error against the oracle's fp64 result):
  fp32 I/O : 1e-5.
  bf16 I/O : 2e-2.  For GroupNorm outputs with |y| >= 8 the bf16 grid itself
             is coarser than that (half an ulp is 2^-5 on [8, 16)), so there
             the bound is half an ulp of the oracle value plus 1e-3.  Attention
             outputs are convex combinations of |v| < 8 and conv outputs have
             sigma ~ 1, so the plain bound applies to them.
"""
from __future__ import annotations

import numpy as np
import torch

import synth

TOL_F32 = 1e-5
TOL_BF16 = 2e-2


def to_device(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.to("cuda")


def from_device(t: torch.Tensor) -> np.ndarray:
    """Exact float64 values of a CUDA tensor."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return synth.bf16_to_f32(t.view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    return t.numpy().astype(np.float64)


def half_ulp_bf16(y: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at |y| (8 significant bits)."""
    a = np.abs(y)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def tolerance(dtype: str, ref: np.ndarray, kind: str) -> np.ndarray | float:
    if dtype == "f32":
        return TOL_F32
    if kind == "gn":
        return np.maximum(TOL_BF16, half_ulp_bf16(ref) + 1e-3)
    return TOL_BF16


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, kind: str, what: str = ""):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = tolerance(dtype, ref, kind)
    bad = err > tol
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                             f"worst at {i}: got {got[i]!r} oracle {ref[i]!r} "
                             f"(max abs err {err.max():.3e})")
    return float(err.max())


def sample_positions(P: int, count: int = 4, seed: int = 0) -> list[int]:
    """First, last and a few seeded interior positions."""
    rng = np.random.default_rng(seed)
    inner = rng.choice(np.arange(1, max(P - 1, 2)), size=min(count, max(P - 2, 0)), replace=False)
    return sorted({0, P - 1, *[int(i) for i in inner]})

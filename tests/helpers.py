"""Shared helpers of the GPU parity tests (conversion and comparison only)."""

from __future__ import annotations

import math

import numpy as np

TOL = {"r32": 1e-4, "c64": 1e-4, "c32h": 2e-3, "r16": 2e-3}


def to_np(t):
    return t.detach().cpu().contiguous().numpy()


def as_complex(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "c32h":
        return a[..., 0].astype(np.float64) + 1j * a[..., 1].astype(np.float64)
    return a.astype(np.complex128)


def rel_err(w_gpu: np.ndarray, w_ref: np.ndarray, dtype: str) -> float:
    """max |W_gpu - W_ref| / max |W_ref| over the compared elements."""
    a, b = as_complex(w_gpu, dtype), as_complex(w_ref, dtype)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def projector_distance(U, V) -> float:
    U = np.asarray(U, np.complex128)
    V = np.asarray(V, np.complex128)
    return float(np.linalg.norm(U @ U.conj().T - V @ V.conj().T))


def eigengap(evals: np.ndarray, r: int) -> float:
    if r >= len(evals) or evals[0] <= 0:
        return math.inf
    return float((evals[r - 1] - evals[r]) / evals[0])


def random_moments(rng, info, cplx, scale=1e-2):
    """Non-zero moments (v >= 0) to exercise the moment arithmetic."""
    out = {}
    for key in ("core_m", "sparse_m"):
        out[key] = (rng.standard_normal(info[key + "_len"]) * scale).astype(np.float32)
    for key in ("core_v", "sparse_v"):
        out[key] = (rng.standard_normal(info[key + "_len"]) * scale) ** 2
        out[key] = out[key].astype(np.float32)
    return out

"""The seeded input generator follows its stated recipe (the only module the
oracle and the CUDA path share, and it holds none of the method's
arithmetic): an exact Tucker part, floor(p N) outliers, dense noise, fixed or
drifting orthonormal factors, storage layouts per dtype, reproducible seeds."""

import math

import numpy as np
import pytest
import torch

from rank_sparse_tensor_b200 import synth


def _c(x, dtype):
    a = x.numpy()
    if dtype == "c32h":
        return a[..., 0].astype(np.float64) + 1j * a[..., 1].astype(np.float64)
    return a.astype(np.complex128)


def _unfold(X, n):
    return np.moveaxis(X, n, 0).reshape(X.shape[n], -1)


@pytest.mark.parametrize("dtype", ["c64", "r32"])
def test_tucker_exact_has_the_generator_ranks(dtype):
    shape, ranks = (12, 10, 9, 7), (3, 4, 2, 3)
    g, Q = synth.tucker_exact(shape, ranks, dtype, seed=2)
    X = _c(g, dtype)
    for n, (q, r) in enumerate(zip(Q, ranks)):
        qn = q.numpy().astype(np.complex128)
        assert np.allclose(qn.conj().T @ qn, np.eye(r), atol=1e-5)
        s = np.linalg.svd(_unfold(X, n), compute_uv=False)
        assert s[r] / s[0] < 1e-5 and s[r - 1] / s[0] > 1e-3
        # the tensor lies in the span of Q_n along mode n
        P = qn @ qn.conj().T
        Xp = np.moveaxis(np.tensordot(P, np.moveaxis(X, n, 0), axes=1), 0, n)
        assert np.abs(Xp - X).max() <= 1e-5 * np.abs(X).max()


@pytest.mark.parametrize("dtype", ["c64", "r32"])
def test_outliers_are_floor_pN_entries(dtype):
    shape, ranks, p, scale = (16, 12, 10), (3, 3, 2), 0.013, 100.0
    N = math.prod(shape)
    base = synth.GradientStream(shape, ranks, dtype, 4, outlier_frac=0.0, noise=0.0).next()
    out = synth.GradientStream(shape, ranks, dtype, 4, outlier_frac=p, outlier_scale=scale,
                               noise=0.0).next()
    d = _c(out, dtype) - _c(base, dtype)
    nz = np.count_nonzero(np.abs(d) > 1e-3)
    assert nz == math.floor(p * N)
    assert 0.5 * scale < np.sqrt(np.mean(np.abs(d[np.abs(d) > 1e-3]) ** 2)) < 1.5 * scale


def test_noise_level():
    shape = (20, 16, 12)
    base = synth.GradientStream(shape, (2, 2, 2), "c64", 6, outlier_frac=0.0, noise=0.0).next()
    noisy = synth.GradientStream(shape, (2, 2, 2), "c64", 6, outlier_frac=0.0, noise=0.5).next()
    d = _c(noisy, "c64") - _c(base, "c64")
    assert abs(np.sqrt(np.mean(np.abs(d) ** 2)) - 0.5) < 0.05


def test_seeds_and_steps():
    a = synth.GradientStream((8, 6, 5), (2, 2, 2), "c64", 1)
    b = synth.GradientStream((8, 6, 5), (2, 2, 2), "c64", 1)
    c = synth.GradientStream((8, 6, 5), (2, 2, 2), "c64", 2)
    a0, a1 = a.next(), a.next()
    b0 = b.next()
    assert torch.equal(a0, b0) and not torch.equal(a0, a1)
    assert not torch.equal(a0, c.next())


def test_storage_layouts():
    shape = (4, 3, 5)
    want = {"r32": (torch.float32, shape), "r16": (torch.float16, shape),
            "c64": (torch.complex64, shape), "c32h": (torch.float16, shape + (2,))}
    for dt, (tdt, sh) in want.items():
        g = synth.GradientStream(shape, (2, 2, 2), dt, 0).next()
        w = synth.weights(shape, dt, 0)
        assert g.dtype == tdt and tuple(g.shape) == sh and g.is_contiguous()
        assert w.dtype == tdt and tuple(w.shape) == sh


def test_weight_scale():
    w = synth.weights((64, 64, 32), "c64", 3).numpy()
    for comp in (w.real, w.imag):
        assert abs(comp.std() - 0.02) < 0.001 and abs(comp.mean()) < 0.001


def test_drift_keeps_factors_orthonormal():
    s = synth.GradientStream((10, 8, 6), (3, 2, 2), "c64", 5, drift=0.05)
    q0 = [q.clone() for q in s.Q]
    s.next()
    assert all(torch.equal(a, b) for a, b in zip(q0, s.Q))   # the first step keeps them
    s.next()
    for a, b in zip(q0, s.Q):
        qb = b.numpy().astype(np.complex128)
        assert np.allclose(qb.conj().T @ qb, np.eye(qb.shape[1]), atol=1e-5)
        assert not torch.equal(a, b)
    fixed = synth.GradientStream((10, 8, 6), (3, 2, 2), "c64", 5)
    f0 = [q.clone() for q in fixed.Q]
    fixed.next()
    fixed.next()
    assert all(torch.equal(a, b) for a, b in zip(f0, fixed.Q))


def test_integer_ties():
    g = synth.integer_ties((6, 7), "c64", 3, levels=2).numpy()
    for comp in (g.real, g.imag):
        assert np.array_equal(comp, np.round(comp)) and np.abs(comp).max() <= 2


def test_workload_table():
    for name, wl in synth.WORKLOADS.items():
        assert wl.name == name
        assert all(1 <= r <= I for r, I in zip(wl.ranks, wl.shape))
        assert wl.k == math.floor(wl.sparse_ratio * wl.N)
    assert synth.WORKLOADS["spectral_c32h_256x256x128x65"].N == 545_259_520
    assert synth.WORKLOADS["spectral_c32h_256x256x128x65"].k == 27_262_976
    assert synth.WORKLOADS["fno4_c32h_128x128x64x33"].n_tensors == 4

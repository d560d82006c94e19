"""Pins for the oracle's DCT factor basis (the dynamic column selection of the
Trion / DCT-AdamW page, used as a cheap refresh): the basis vectors are the
columns of scipy's orthonormal DCT-II matrix, each mode keeps the r_n columns
with the largest alignment q_j^T Gram q_j (ties to the lower column), in
descending order; a step projects onto them like onto HOSVD factors."""

import math
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import scipy.fft

import oracle


def dct_matrix(n):
    """Orthonormal DCT-II matrix from scipy (row k = frequency k)."""
    return scipy.fft.dct(np.eye(n), type=2, norm="ortho", axis=0)


def unfold(X, n):
    return np.moveaxis(X, n, 0).reshape(X.shape[n], -1)


def mode_mul(X, M, n):
    return np.moveaxis(np.tensordot(M, np.moveaxis(X, n, 0), axes=1), 0, n)


def selection(X, n, r):
    """Columns of the DCT matrix by descending alignment, ties to the lower."""
    Q = dct_matrix(X.shape[n])
    score = np.sum(np.abs(unfold(X, n).conj().T @ Q) ** 2, axis=0)
    order = sorted(range(len(score)), key=lambda j: (-score[j], j))
    return order[:r], np.sort(score)[::-1]


def pin_span_recovered(make):
    """Mode-0 fibers in the span of DCT columns 3 and 7: exactly those two."""
    rng = np.random.default_rng(1)
    Q = dct_matrix(12)
    core = rng.standard_normal((2, 5, 4)) + 1j * rng.standard_normal((2, 5, 4))
    X = mode_mul(core, Q[:, [3, 7]], 0).astype(np.complex64)
    o = make((12, 5, 4), (2, 5, 4))
    o.refresh(X)
    U = o.get_U(0)
    assert sorted(int(np.argmax(np.abs(Q.T @ U[:, c]))) for c in range(2)) == [3, 7]
    P = U @ U.conj().T
    assert np.abs(P - Q[:, [3, 7]] @ Q[:, [3, 7]].T).max() < 1e-6


def pin_scores_match_numpy(make):
    """Random tensor: every mode's U is the numpy selection's columns, and the
    reported values are the sorted alignments."""
    rng = np.random.default_rng(2)
    X = (rng.standard_normal((9, 7, 6)) + 1j * rng.standard_normal((9, 7, 6))).astype(np.complex64)
    ranks = (3, 2, 4)
    o = make(X.shape, ranks)
    o.refresh(X)
    for n, r in enumerate(ranks):
        sel, sc = selection(X.astype(np.complex128), n, r)
        Q = dct_matrix(X.shape[n])
        assert np.abs(o.get_U(n) - Q[:, sel]).max() < 1e-6, n
        assert np.allclose(o.eigvals(n), sc, rtol=1e-9, atol=1e-12)


def pin_ties_to_lower_columns(make):
    """A zero gradient aligns equally with every column: the first r."""
    X = np.zeros((8, 5, 3), np.complex64)
    o = make(X.shape, (3, 2, 2))
    o.refresh(X)
    Q = dct_matrix(8)
    assert np.abs(o.get_U(0) - Q[:, :3]).max() < 1e-6


def pin_step_projects_onto_the_columns(make):
    """rho = 0, one step from zero moments: the weights move by the AdamW
    update of the core taken on the selected DCT columns."""
    rng = np.random.default_rng(3)
    shape, ranks, lr = (8, 6, 5), (3, 2, 2), 1e-2
    G = (rng.standard_normal(shape) + 1j * rng.standard_normal(shape)).astype(np.complex64)
    W = (0.02 * (rng.standard_normal(shape) + 1j * rng.standard_normal(shape))).astype(np.complex64)
    o = make(shape, ranks, lr=lr)
    o.refresh(G)
    w = W.copy()
    o.step(G, w)
    G64 = G.astype(np.complex128)
    Us = [dct_matrix(shape[n])[:, selection(G64, n, ranks[n])[0]] for n in range(3)]
    C = G64
    for n, U in enumerate(Us):
        C = mode_mul(C, U.conj().T, n)
    f32 = np.float32
    m = f32(0.1 * C.real).astype(np.float64) + 1j * f32(0.1 * C.imag).astype(np.float64)
    v = f32(0.001 * (C.real ** 2 + C.imag ** 2)).astype(np.float64)
    D = (m / 0.1) / (np.sqrt(v / 0.001) + 1e-8)
    for n, U in enumerate(Us):
        D = mode_mul(D, U, n)
    ref = (W.astype(np.complex128) - lr * D).astype(np.complex64)
    assert np.abs(w - ref).max() <= 1e-6 * np.abs(ref).max()


PINS = [pin_span_recovered, pin_scores_match_numpy, pin_ties_to_lower_columns,
        pin_step_projects_onto_the_columns]


def _make(shape, ranks, lr=1e-3):
    return oracle.Oracle(shape, ranks, 0.0, 0, lr=lr, grad_dtype="c64", auto_refresh=0, basis=1)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(_make)


def test_unknown_basis_rejected():
    with pytest.raises(ValueError):
        oracle.Oracle((4, 4, 4), (2, 2, 2), 0.1, 0, basis=2)


# (name, original text, mutated text): slips in the DCT basis
MUTANTS = [
    ("rows_for_columns", "h.U[n][2 * (i * rn + c)] = (float)dct_entry(i, ord[c], In);",
     "h.U[n][2 * (i * rn + c)] = (float)dct_entry(ord[c], i, In);"),
    ("row0_not_scaled", "return k == 0 ? v / std::sqrt(2.0) : v;", "return v;"),
    ("ascending_alignment", "[&](int64_t a, int64_t b) { return score[a] > score[b]; });",
     "[&](int64_t a, int64_t b) { return score[a] < score[b]; });"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "oracle", "tgd_oracle.cpp")).read()
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        mut, so = os.path.join(d, "mutant.cpp"), os.path.join(d, "mutant.so")
        open(mut, "w").write(src.replace(old, new))
        subprocess.run(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread",
                        "-ffp-contract=off", "-o", so, mut], check=True)
        env = dict(os.environ, TGD_ORACLE_LIB=so, TGD_ORACLE_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            "-k", "not planted_mistake", os.path.abspath(__file__)],
                           env=env, cwd=root, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"

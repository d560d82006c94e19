"""Pins for the oracle's ablated variants of the decomposition.

The method's free parameters include the decomposition order (sparse part
first is the chosen one; the ablation reverses it), and the pages compare it
with a matricized extension of GaLore. Each variant is checked here against an
independent numpy statement of its definition on small tensors (numpy SVD and
eigh for the factors, numpy tensordot for the mode products, FP32-stored Adam
moments). The only oracle routine reused is its top-k selection, which is
pinned against brute force on its own.
"""

import math

import numpy as np
import pytest

import oracle

B1, B2, EPS = 0.9, 0.999, 1e-8


# ------------------------------------------------------------ numpy reference
def unfold(X, n):
    return np.moveaxis(X, n, 0).reshape(X.shape[n], -1)


def mode_mul(X, M, n):
    """X x_n M for a matrix M of shape (J, I_n)."""
    return np.moveaxis(np.tensordot(M, np.moveaxis(X, n, 0), axes=1), 0, n)


def hosvd_factors(X, ranks):
    """Leading r_n eigenvectors of each mode-n Gram; None for full-rank modes."""
    Us = []
    for n, r in enumerate(ranks):
        if r == X.shape[n]:
            Us.append(None)
            continue
        Xn = unfold(X, n)
        _, V = np.linalg.eigh(Xn @ Xn.conj().T)
        Us.append(V[:, ::-1][:, :r])
    return Us


def project(X, Us):
    for n, U in enumerate(Us):
        if U is not None:
            X = mode_mul(X, U.conj().T, n)
    return X


def expand(C, Us):
    for n, U in enumerate(Us):
        if U is not None:
            C = mode_mul(C, U, n)
    return C


def adam_first_step(g, cplx):
    """One Adam step from zero moments at t = 0 (bias correction s = 1), with
    m and v rounded to FP32 storage before the update is formed; complex m,
    v = EMA of |g|^2."""
    f32 = np.float32
    if cplx:
        m = f32((1 - B1) * g.real).astype(np.float64) + 1j * f32((1 - B1) * g.imag).astype(np.float64)
        v = f32((1 - B2) * (g.real * g.real + g.imag * g.imag)).astype(np.float64)
    else:
        m = f32((1 - B1) * g).astype(np.float64)
        v = f32((1 - B2) * g * g).astype(np.float64)
    return (m / (1 - B1)) / (np.sqrt(v / (1 - B2)) + EPS)


def weight_update(W, D, lr, wd):
    out = W.astype(np.complex128 if np.iscomplexobj(W) else np.float64) * (1 - lr * wd) - lr * D
    return out.astype(W.dtype)


def lowrank_first_step(G, W, ranks, rho, lr, wd, lam):
    """Refresh and one step with the low-rank part first: factors from G
    itself, Omega = top-k of E = G - L (E in fp32), sparse values E at Omega."""
    cplx = np.iscomplexobj(G)
    G64 = G.astype(np.complex128 if cplx else np.float64)
    Us = hosvd_factors(G64, ranks)
    C = project(G64, Us)
    E = G64 - expand(C, Us)
    k = math.floor(rho * G.size)
    omega = oracle.topk(E.astype(np.complex64 if cplx else np.float32).reshape(-1),
                        "c64" if cplx else "r32", k)
    sparse = lam * adam_first_step(E.reshape(-1)[omega], cplx)
    D = expand(adam_first_step(C, cplx), Us).reshape(-1)
    D[omega] += sparse
    return omega, weight_update(W, D.reshape(G.shape), lr, wd), Us


def galore_step(G, W, d, r, lr, wd):
    """Matricized GaLore along mode d: P = leading r left singular vectors of
    G_(d); Adam on P^H G_(d); the update P Adam(P^H G_(d)) folded back."""
    cplx = np.iscomplexobj(G)
    G64 = G.astype(np.complex128 if cplx else np.float64)
    Gd = unfold(G64, d)
    P = np.linalg.svd(Gd, full_matrices=False)[0][:, :r]
    upd = P @ adam_first_step(P.conj().T @ Gd, cplx)
    moved = np.moveaxis(G64, d, 0).shape
    D = np.moveaxis(upd.reshape(moved), 0, d)
    return weight_update(W, D, lr, wd)


def rel(a, b):
    a = a.astype(np.complex128)
    b = b.astype(np.complex128)
    return float(np.abs(a - b).max() / np.abs(b).max())


def inputs(shape, gen_ranks, dtype, seed, outlier_frac=0.05):
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    G = GradientStream(shape, gen_ranks, dtype, seed, outlier_frac=outlier_frac,
                       outlier_scale=10.0).next().numpy()
    W = weights(shape, dtype, seed).numpy()
    return G, W


# ------------------------------------------------------------------- pins
@pytest.mark.parametrize("dtype,shape,ranks,rho", [
    ("c64", (6, 5, 8, 7), (2, 2, 3, 3), 0.1),
    ("c64", (4, 9, 6), (2, 3, 2), 0.05),
    ("r32", (7, 6, 9), (3, 2, 4), 0.1),
    ("r32", (5, 4, 6, 3), (2, 4, 3, 2), 0.2),   # one full-rank mode
])
def test_lowrank_first_matches_numpy(dtype, shape, ranks, rho):
    lr, wd, lam = 1e-2, 0.01, 0.5
    G, W = inputs(shape, ranks, dtype, seed=3)
    omega, W_ref, _ = lowrank_first_step(G, W, ranks, rho, lr, wd, lam)
    o = oracle.Oracle(shape, ranks, rho, 0, lr=lr, wd=wd, grad_dtype=dtype, sparse_scale=lam,
                      auto_refresh=0, order=1)
    o.refresh(G)
    assert np.array_equal(o.omega, omega)
    w = W.copy()
    assert o.step(G, w) == 0
    assert rel(w, W_ref) <= 1e-6


def test_lowrank_first_without_sparse_part_is_sparse_first():
    """rho = 0: both orders are the pure low-rank update."""
    shape, ranks = (6, 5, 8, 7), (2, 2, 3, 3)
    G, W = inputs(shape, ranks, "c64", seed=4)
    out = []
    for order in (0, 1):
        o = oracle.Oracle(shape, ranks, 0.0, 0, lr=1e-2, wd=0.01, grad_dtype="c64",
                          auto_refresh=0, order=order)
        o.refresh(G)
        w = W.copy()
        o.step(G, w)
        out.append(w)
    assert rel(out[1], out[0]) <= 1e-6


def test_lowrank_first_at_full_rank_is_adamw():
    """Full ranks: L = G, the sparse values are zero and contribute nothing;
    the step is AdamW on G."""
    shape = (4, 5, 6)
    G, W = inputs(shape, shape, "c64", seed=5)
    o = oracle.Oracle(shape, shape, 0.1, 0, lr=1e-2, wd=0.01, grad_dtype="c64",
                      auto_refresh=0, order=1)
    o.refresh(G)
    w = W.copy()
    o.step(G, w)
    W_ref = weight_update(W, adam_first_step(G.astype(np.complex128), True), 1e-2, 0.01)
    assert rel(w, W_ref) <= 1e-6


def test_outliers_perturb_the_lowrank_first_subspace():
    """The pages' reason for the order: outliers left in the gradient pull the
    Tucker subspace away from the low-rank signal. With large outliers and
    Omega big enough to hold them, the sparse-first factors sit closer to the
    generator's subspace than the low-rank-first ones."""
    from rank_sparse_tensor_b200.synth import GradientStream
    shape, ranks = (12, 10, 9), (3, 3, 2)
    gs = GradientStream(shape, ranks, "c64", 8, outlier_frac=0.01, outlier_scale=300.0)
    G = gs.next().numpy()
    # the generator's clean part: G with its outliers removed is exactly rank
    # (3, 3, 2) up to the noise, so its own HOSVD is the reference subspace
    Gc = G.astype(np.complex128)
    top = np.argsort(-np.abs(Gc).reshape(-1))[:int(0.01 * G.size)]
    clean = Gc.reshape(-1).copy()
    clean[top] = 0
    U_ref = hosvd_factors(clean.reshape(shape), ranks)
    dist = {}
    for order in (0, 1):
        o = oracle.Oracle(shape, ranks, 0.02, 0, grad_dtype="c64", auto_refresh=0, order=order)
        o.refresh(G)
        d = 0.0
        for n in range(3):
            U = o.get_U(n)
            d += np.linalg.norm(U @ U.conj().T - U_ref[n] @ U_ref[n].conj().T)
        dist[order] = d
    assert dist[0] < 0.5 * dist[1], dist


@pytest.mark.parametrize("dtype,shape,d,r", [
    ("c64", (6, 5, 8), 0, 2),
    ("c64", (6, 5, 8), 2, 3),
    ("r32", (7, 4, 5, 3), 1, 2),
])
def test_matricized_galore_is_a_one_mode_tucker_step(dtype, shape, d, r):
    """GaLore on the mode-d unfolding is the step with rank r on mode d, every
    other mode at full rank (the identity) and no sparse part."""
    lr, wd = 1e-2, 0.01
    G, W = inputs(shape, shape, dtype, seed=6)
    ranks = tuple(r if n == d else I for n, I in enumerate(shape))
    o = oracle.Oracle(shape, ranks, 0.0, 0, lr=lr, wd=wd, grad_dtype=dtype, auto_refresh=0)
    o.refresh(G)
    w = W.copy()
    o.step(G, w)
    assert rel(w, galore_step(G, W, d, r, lr, wd)) <= 1e-6


def test_unknown_order_rejected():
    with pytest.raises(ValueError):
        oracle.Oracle((4, 4, 4), (2, 2, 2), 0.1, 0, order=2)


# (name, original text, mutated text): slips in the low-rank-first code
MUTANTS = [
    ("sparse_values_from_gradient", "cd e = {G[i].re - L[i].re, G[i].im - L[i].im};", "cd e = G[i];"),
    ("keys_from_gradient", "Ef[i * comps] = (float)(G[i].re - L[i].re);", "Ef[i * comps] = (float)(G[i].re);"),
    ("sparse_update_not_scattered",
     "for (int64_t j = 0; j < h.k; ++j) D[h.omega[j]] = D[h.omega[j]] + sparse_upd[j];", ""),
    ("sparse_scale_dropped_in_lowrank_first",
     "    cd u = adam_update(e, &h.sp_m[j * mc], &h.sp_v[j * vc], h, bc1, bc2);\n"
     "    sparse_upd[j] = {h.o.sparse_scale * u.re, h.o.sparse_scale * u.im};",
     "    cd u = adam_update(e, &h.sp_m[j * mc], &h.sp_v[j * vc], h, bc1, bc2);\n"
     "    sparse_upd[j] = u;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    """A mutated copy of the oracle (compiled to a temporary directory; the
    shipped one is untouched) fails at least one of the pins above."""
    import os
    import subprocess
    import sys
    import tempfile
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

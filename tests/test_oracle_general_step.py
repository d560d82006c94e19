"""Pin of the oracle's general sparse-first step against a numpy restatement.

The other step pins reach the general case only through special cases (full
ranks, rho = 0 or 1, zero moments). Here one step runs with everything on at
once: a sparse part (rho = 0.05, Omega at random positions), partial Tucker
ranks with one full-rank mode, non-zero moments carried over from earlier
steps (t > 0, so the bias correction is not the first step's), weight decay,
a sparse scale lambda != 1, and both complex Adam variants.

The numpy side restates the step of the nullthought.net TensorGRaD summary
(section 三) and the paper text appended to the Pith review (Theorem 2: project
with the conjugate-transposed factors, Adam on the core, project back) with
numpy only: gather g_s = G[Omega]; residual R = G with Omega zeroed; core
C = R x_n U_n^H by tensordot; AdamW with FP32-stored moments on C and on g_s;
Delta = C~ x_n U_n with lambda S~ added at Omega; W <- W (1 - lr wd) - lr Delta
rounded once to the storage type. No oracle routine is used on that side;
the factors and Omega are inputs (any orthonormal factors and any index set
define the step), so no eigensolver or selection enters the comparison.
"""

import numpy as np
import pytest

import oracle

B1, B2, EPS = 0.9, 0.999, 1e-8


def mode_mul(X, M, n):
    """X x_n M for a matrix M of shape (J, I_n)."""
    return np.moveaxis(np.tensordot(M, np.moveaxis(X, n, 0), axes=1), 0, n)


def adam(g, m, v, t, cplx, cmode):
    """AdamW moments for step count s = t + 1, stored as FP32 before the
    update direction is formed. g: complex128 or float64 array; m, v the
    stored FP32 moments as float arrays laid out like the oracle's (complex m
    as (re, im) pairs; v one value per entry, or (re, im) pairs when cmode = 1).
    Returns (update, m_new, v_new)."""
    s = t + 1
    bc1, bc2 = 1 - B1 ** s, 1 - B2 ** s
    f32 = np.float32
    if not cplx:
        m1 = f32(B1 * m.astype(np.float64) + (1 - B1) * g)
        v1 = f32(B2 * v.astype(np.float64) + (1 - B2) * g * g)
        u = (m1 / bc1) / (np.sqrt(v1.astype(np.float64) / bc2) + EPS)
        return u, m1, v1
    mp = m.reshape(-1, 2).astype(np.float64)
    mr = f32(B1 * mp[:, 0] + (1 - B1) * g.real)
    mi = f32(B1 * mp[:, 1] + (1 - B1) * g.imag)
    m1 = np.stack([mr, mi], -1).reshape(-1)
    if cmode == 1:
        vp = v.reshape(-1, 2).astype(np.float64)
        vr = f32(B2 * vp[:, 0] + (1 - B2) * g.real * g.real)
        vi = f32(B2 * vp[:, 1] + (1 - B2) * g.imag * g.imag)
        u = ((mr / bc1) / (np.sqrt(vr.astype(np.float64) / bc2) + EPS)
             + 1j * (mi / bc1) / (np.sqrt(vi.astype(np.float64) / bc2) + EPS))
        return u, m1, np.stack([vr, vi], -1).reshape(-1)
    v1 = f32(B2 * v.astype(np.float64) + (1 - B2) * (g.real * g.real + g.imag * g.imag))
    den = np.sqrt(v1.astype(np.float64) / bc2) + EPS
    u = (mr.astype(np.float64) / bc1) / den + 1j * (mi.astype(np.float64) / bc1) / den
    return u, m1, v1


def numpy_step(G, W, Us, omega, moments, t, lr, wd, lam, cmode):
    """One sparse-first step; returns (W_new, new moments)."""
    cplx = np.iscomplexobj(G)
    G64 = G.astype(np.complex128 if cplx else np.float64)
    flat = G64.reshape(-1)
    g_s = flat[omega]
    R = flat.copy()
    R[omega] = 0
    C = R.reshape(G.shape)
    for n, U in enumerate(Us):
        if U is not None:
            C = mode_mul(C, U.conj().T if cplx else U.T, n)
    cu, cm, cv = adam(C.reshape(-1), moments["core_m"], moments["core_v"], t, cplx, cmode)
    su, sm, sv = adam(g_s, moments["sparse_m"], moments["sparse_v"], t, cplx, cmode)
    D = cu.reshape(C.shape)
    for n, U in enumerate(Us):
        if U is not None:
            D = mode_mul(D, U, n)
    D = D.reshape(-1).copy()
    D[omega] += lam * su
    W64 = W.astype(np.complex128 if cplx else np.float64).reshape(-1)
    Wn = (W64 * (1 - lr * wd) - lr * D).astype(W.dtype).reshape(W.shape)
    return Wn, {"core_m": cm, "core_v": cv, "sparse_m": sm, "sparse_v": sv}


def rand_orthonormal(rng, I, r, cplx):
    X = rng.standard_normal((I, r))
    if cplx:
        X = X + 1j * rng.standard_normal((I, r))
    Q, _ = np.linalg.qr(X)
    return Q.astype(np.complex64 if cplx else np.float32)


def rel(a, b):
    a = np.asarray(a).astype(np.complex128)
    b = np.asarray(b).astype(np.complex128)
    return float(np.abs(a - b).max() / np.abs(b).max())


CASES = [
    # dtype, shape, ranks (one mode at full rank), rho, complex Adam mode
    ("c64", (6, 5, 8, 7), (3, 5, 4, 3), 0.05, 0),
    ("c64", (6, 5, 8, 7), (3, 5, 4, 3), 0.05, 1),
    ("c64", (9, 4, 6), (4, 2, 6), 0.05, 0),
    ("r32", (7, 6, 9), (3, 6, 4), 0.05, 0),
    ("r32", (5, 4, 6, 3), (2, 3, 3, 3), 0.05, 0),
]


@pytest.mark.parametrize("dtype,shape,ranks,rho,cmode", CASES)
def test_general_step_matches_numpy(dtype, shape, ranks, rho, cmode):
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    rng = np.random.default_rng(11)
    cplx = dtype == "c64"
    lr, wd, lam, t = 3e-3, 0.05, 0.7, 7
    G = GradientStream(shape, ranks, dtype, 21, outlier_frac=0.03, outlier_scale=10.0).next().numpy()
    W = weights(shape, dtype, 22).numpy()
    o = oracle.Oracle(shape, ranks, rho, 0, lr=lr, wd=wd, grad_dtype=dtype, sparse_scale=lam,
                      complex_adam=cmode, auto_refresh=0)
    info = o.info
    N, k = info["N"], info["k"]
    assert k == int(np.floor(rho * N)) and k > 0
    omega = np.sort(rng.choice(N, size=k, replace=False)).astype(np.int64)
    Us = []
    for n, (I, r) in enumerate(zip(shape, ranks)):
        if r < I:
            U = rand_orthonormal(rng, I, r, cplx)
            o.set_U(n, U)
            Us.append(U.astype(np.complex128 if cplx else np.float64))
        else:
            Us.append(None)
    o.omega = omega
    o.set_counters(t, 1)
    moments = {}
    for which in ("core_m", "core_v", "sparse_m", "sparse_v"):
        size = o._msize(which)
        x = rng.standard_normal(size).astype(np.float32) * 0.3
        if which.endswith("_v"):
            x = np.abs(x) * 0.1 + 1e-3   # second moments are non-negative
        o.set_moment(which, x)
        moments[which] = x.copy()
    W_ref, mom_ref = numpy_step(G, W, Us, omega, moments, t, lr, wd, lam, cmode)
    w = W.copy()
    assert o.step(G, w) == 0
    # fp64 on both sides, FP32 moments rounded once each: agreement to a few
    # ulps of fp32 storage in the weights and moments
    assert rel(w, W_ref) <= 1e-6
    for which, ref in mom_ref.items():
        got = o.get_moment(which)
        assert np.allclose(got, ref, rtol=1e-6, atol=1e-12), which
    # the update itself, not just the weights: the weights' change agrees
    dW = w.astype(np.complex128) - W.astype(np.complex128)
    dW_ref = W_ref.astype(np.complex128) - W.astype(np.complex128)
    assert rel(dW, dW_ref) <= 1e-4


def test_general_step_sees_a_wrong_mode_product():
    """The comparison is sharp enough to catch a plausible slip on the numpy
    side: projecting with U_n instead of its conjugate changes the step."""
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    shape, ranks = (6, 5, 8, 7), (3, 5, 4, 3)
    rng = np.random.default_rng(12)
    G = GradientStream(shape, ranks, "c64", 31, outlier_frac=0.03).next().numpy()
    W = weights(shape, "c64", 32).numpy()
    o = oracle.Oracle(shape, ranks, 0.05, 0, lr=3e-3, grad_dtype="c64", auto_refresh=0)
    Us = []
    for n, (I, r) in enumerate(zip(shape, ranks)):
        if r < I:
            U = rand_orthonormal(rng, I, r, True)
            o.set_U(n, U)
            Us.append(U.astype(np.complex128))
        else:
            Us.append(None)
    k = o.info["k"]
    omega = np.sort(rng.choice(G.size, size=k, replace=False)).astype(np.int64)
    o.omega = omega
    o.set_counters(0, 1)
    zeros = {w: np.zeros(o._msize(w), np.float32) for w in ("core_m", "core_v", "sparse_m", "sparse_v")}
    w = W.copy()
    o.step(G, w)
    good, _ = numpy_step(G, W, Us, omega, zeros, 0, 3e-3, 0.0, 1.0, 0)
    bad, _ = numpy_step(G, W, [None if U is None else U.conj() for U in Us], omega, zeros, 0,
                        3e-3, 0.0, 1.0, 0)
    assert rel(w, good) <= 1e-6
    assert rel(w, bad) > 1e-4

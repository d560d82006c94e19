"""Pins of the CPU oracle to facts the pages and the mathematics fix.

Every check here compares the oracle against something other than itself:
published test vectors, textbook identities, library routines (numpy), brute
force on tiny inputs, or special cases where the method reduces to plain
AdamW. Planted mistakes (a dropped term, a wrong sign, a transposed operand, an
off-by-one index) fail at least one of them; ``test_oracle_planted.py`` checks
that claim for mistakes planted in copies of the oracle.
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ------------------------------------------------------------------ helpers
def rng(seed):
    return np.random.default_rng(seed)


def crandn(r, shape):
    return (r.standard_normal(shape) + 1j * r.standard_normal(shape)) / math.sqrt(2)


def orthonormal(r, I, c, complex_=True):
    a = crandn(r, (I, c)) if complex_ else r.standard_normal((I, c))
    q, _ = np.linalg.qr(a)
    return q


def np_mode_product(x, n, M):
    """Y = x x_n M with M of shape (J, I): contracts axis n of x with M's axis 1."""
    y = np.tensordot(M, x, axes=([1], [n]))  # J, ...rest
    return np.moveaxis(y, 0, n)


def projector_distance(U, V):
    return np.linalg.norm(U @ U.conj().T - V @ V.conj().T)


def f32_round_exact(q: Fraction) -> np.float32:
    """Round an exact rational to the nearest float32, ties to even."""
    f = np.float32(float(q))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - q),
                                     int(np.array(c, np.float32).view(np.uint32)) & 1))
    return np.float32(best)


# -------------------------------------------------------------- binary16
def test_binary16_golden(oracle_mod):
    rows = []
    for line in open(os.path.join(HERE, "golden", "binary16_rounding.txt")):
        line = line.split("#")[0].strip()
        if line:
            v, b = line.split()[:2]
            rows.append((float(v), int(b, 16)))
    bits = oracle_mod.f64_to_f16_bits(np.array([v for v, _ in rows]))
    assert [int(x) for x in bits] == [b for _, b in rows]


def test_binary16_matches_numpy(oracle_mod):
    r = rng(1)
    x = np.concatenate([
        r.standard_normal(20000) * 10.0 ** r.integers(-9, 5, 20000),
        (r.integers(-2048, 2048, 5000) + 0.5) * 2.0 ** r.integers(-24, 5, 5000),  # ties
        np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e6, -1e6, 2.0 ** -25, 2.0 ** -26]),
    ])
    ours = oracle_mod.f64_to_f16_bits(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    allbits = np.arange(65536, dtype=np.uint16)
    back = oracle_mod.f16_bits_to_f64(allbits)
    refb = allbits.view(np.float16).astype(np.float64)
    ok = np.isnan(refb) | (back == refb)
    assert ok.all() and np.array_equal(np.isnan(back), np.isnan(refb))


# -------------------------------------------------------------- keys, top-k
def _exact_key(dtype, g, i):
    if dtype in ("r32", "r16"):
        v = np.float32(g.reshape(-1)[i])
        return abs(Fraction(float(v)))
    if dtype == "c64":
        re, im = np.float32(g.reshape(-1)[i].real), np.float32(g.reshape(-1)[i].imag)
    else:
        pair = g.reshape(-1, 2)[i].astype(np.float32)
        re, im = pair[0], pair[1]
    im2 = f32_round_exact(Fraction(float(im)) ** 2)
    return Fraction(float(f32_round_exact(Fraction(float(re)) ** 2 + Fraction(float(im2)))))


def _gen(dtype, n, r, ties=False):
    if ties:
        re = r.integers(-3, 4, n).astype(np.float32)
        im = r.integers(-3, 4, n).astype(np.float32)
    else:
        re = r.standard_normal(n).astype(np.float32)
        im = r.standard_normal(n).astype(np.float32)
    if dtype == "r32":
        return re
    if dtype == "r16":
        return re.astype(np.float16)
    if dtype == "c64":
        return (re + 1j * im).astype(np.complex64)
    return np.stack([re, im], -1).astype(np.float16)


@pytest.mark.parametrize("dtype", ["r32", "c64", "c32h", "r16"])
def test_mag_keys_definition(oracle_mod, dtype):
    r = rng(2)
    g = _gen(dtype, 3000, r)
    keys = oracle_mod.mag_keys(g, dtype)
    exact = [_exact_key(dtype, g, i) for i in range(3000)]
    got = keys.view(np.float32).astype(np.float64)
    assert all(Fraction(float(a)) == b for a, b in zip(got, exact))


@pytest.mark.parametrize("dtype", ["r32", "c64", "c32h", "r16"])
@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("n,k", [(1, 1), (17, 0), (17, 17), (64, 3), (1000, 50), (4096, 204)])
def test_topk_brute_force(oracle_mod, dtype, ties, n, k):
    r = rng(n * 7 + k)
    g = _gen(dtype, n, r, ties)
    keys = [_exact_key(dtype, g, i) for i in range(n)]
    brute = sorted(sorted(range(n), key=lambda i: (-keys[i], i))[:k])
    got = oracle_mod.topk(g, dtype, k)
    assert list(got) == brute


def test_topk_all_equal(oracle_mod):
    g = np.ones(100, np.float32)
    assert list(oracle_mod.topk(g, "r32", 7)) == list(range(7))


# ---------------------------------------------------------- random Omega
def test_splitmix64_published_vector(oracle_mod):
    vals = [int(l, 16) for l in open(os.path.join(HERE, "golden", "splitmix64_seed0.txt"))
            if l.strip() and not l.startswith("#")]
    gamma = 0x9E3779B97F4A7C15
    got = [oracle_mod.splitmix64_mix((i * gamma) % 2 ** 64) for i in range(1, 5)]
    assert got == vals


def test_random_omega_brute_force_and_distinct(oracle_mod):
    for seed, ordinal, n, k in [(0, 0, 1000, 50), (7, 3, 513, 100), (123, 0, 64, 64), (5, 1, 10, 0)]:
        got = oracle_mod.random_omega(seed, ordinal, n, k)
        keys = [oracle_mod.random_key(seed, ordinal, i) for i in range(n)]
        brute = sorted(sorted(range(n), key=lambda i: (keys[i], i))[:k])
        assert list(got) == brute
        assert len(set(got.tolist())) == k and np.all(np.diff(got) > 0)


def test_random_omega_uniform(oracle_mod):
    n, k, trials = 200, 20, 2000
    counts = np.zeros(n)
    for t in range(trials):
        counts[oracle_mod.random_omega(99, t, n, k)] += 1
    expected = trials * k / n
    chi2 = ((counts - expected) ** 2 / expected).sum()
    # 199 degrees of freedom: mean 199, sd ~20; 300 is > 5 sd away.
    assert chi2 < 300
    # a different ordinal draws a different set
    assert not np.array_equal(oracle_mod.random_omega(99, 0, n, k), oracle_mod.random_omega(99, 1, n, k))


# ----------------------------------------------------------- tensor algebra
@pytest.mark.parametrize("shape", [(5, 6, 7), (3, 4, 5, 6), (2, 3, 2, 3, 4)])
def test_mode_product_matches_tensordot(oracle_mod, shape):
    r = rng(len(shape))
    x = crandn(r, shape)
    for n in range(len(shape)):
        I = shape[n]
        rr = max(1, I - 2)
        U = crandn(r, (I, rr))
        y = oracle_mod.mode_product(x, n, U, proj=True)
        assert np.allclose(y, np_mode_product(x, n, U.conj().T), atol=1e-12)
        z = oracle_mod.mode_product(y, n, U, proj=False)
        assert np.allclose(z, np_mode_product(y, n, U), atol=1e-12)


def test_mode_products_commute_and_identity(oracle_mod):
    r = rng(5)
    x = crandn(r, (4, 5, 6))
    A = crandn(r, (4, 2))
    B = crandn(r, (6, 3))
    ab = oracle_mod.mode_product(oracle_mod.mode_product(x, 0, A, True), 2, B, True)
    ba = oracle_mod.mode_product(oracle_mod.mode_product(x, 2, B, True), 0, A, True)
    assert np.allclose(ab, ba, atol=1e-12)
    eye = np.eye(5)
    assert np.allclose(oracle_mod.mode_product(x, 1, eye, True), x, atol=0)


@pytest.mark.parametrize("shape", [(6, 5, 4), (3, 4, 5, 2)])
def test_gram_definition_trace_psd(oracle_mod, shape):
    r = rng(11)
    x = crandn(r, shape)
    for n in range(len(shape)):
        G = oracle_mod.mode_gram(x, n)
        Xn = np.moveaxis(x, n, 0).reshape(shape[n], -1)
        assert np.allclose(G, Xn @ Xn.conj().T, atol=1e-10)
        assert np.isclose(np.trace(G).real, np.linalg.norm(x) ** 2)
        assert np.allclose(G, G.conj().T)
        assert np.linalg.eigvalsh(G).min() > -1e-10


def test_eigh_2x2_closed_form(oracle_mod):
    for a, c, b in [(2.0, 1.0, 0.5 + 0.25j), (1.0, 1.0, 1e-3j), (-3.0, 4.0, 2.0), (5.0, 5.0, 0.0)]:
        A = np.array([[a, b], [np.conj(b), c]], np.complex128)
        w, V = oracle_mod.eigh(A)
        disc = math.sqrt(((a - c) / 2) ** 2 + abs(b) ** 2)
        assert np.allclose(w, [(a + c) / 2 + disc, (a + c) / 2 - disc], atol=1e-13)
        assert np.allclose(A @ V, V * w, atol=1e-12)


@pytest.mark.parametrize("n,real", [(1, False), (7, False), (16, True), (33, False), (64, False)])
def test_eigh_against_numpy(oracle_mod, n, real):
    r = rng(n)
    M = r.standard_normal((n, n)) if real else crandn(r, (n, n))
    A = M @ M.conj().T
    w, V = oracle_mod.eigh(A)
    assert np.allclose(w, np.linalg.eigvalsh(A)[::-1], atol=1e-10 * max(1, abs(w).max()))
    assert np.all(np.diff(w) <= 1e-12)
    assert np.allclose(V.conj().T @ V, np.eye(n), atol=1e-11)
    assert np.allclose(A @ V, V * w, atol=1e-9 * max(1, abs(w).max()))
    # canonical phase: the largest-magnitude entry of each column is real > 0
    for c in range(n):
        i = int(np.argmax(np.abs(V[:, c]) ** 2))
        assert abs(V[i, c].imag) < 1e-14 and V[i, c].real > 0
    if real:
        assert np.abs(V.imag).max() == 0


def test_stable_rank_bounds(oracle_mod):
    """1 <= ||T||_F^2 / ||T_(k)||_2^2 <= rank(T_(k)) (the appendix's stable rank)."""
    r = rng(12)
    Q = [orthonormal(r, I, c) for I, c in [(8, 3), (9, 2), (7, 4)]]
    x = crandn(r, (3, 2, 4))
    for n, q in enumerate(Q):
        x = np_mode_product(x, n, q)
    for n, rk in enumerate([3, 2, 4]):
        w, _ = oracle_mod.eigh(oracle_mod.mode_gram(x, n))
        sr = np.linalg.norm(x) ** 2 / w[0]
        assert 1 - 1e-9 <= sr <= rk + 1e-9
        assert np.all(w[rk:] < 1e-9 * w[0])


# ------------------------------------------------------------- optimizer
def textbook_adamw(grads, w0, lr, b1, b2, eps, wd, complex_mode=0):
    """Plain AdamW (decoupled decay, bias correction, eps outside the sqrt)."""
    w = w0.astype(np.complex128).copy()
    m = np.zeros_like(w)
    v = np.zeros(w.shape, np.float64) if complex_mode == 0 else np.zeros_like(w)
    for t, g in enumerate(grads, start=1):
        g = g.astype(np.complex128)
        m = b1 * m + (1 - b1) * g
        if complex_mode == 0:
            v = b2 * v + (1 - b2) * np.abs(g) ** 2
            upd = (m / (1 - b1 ** t)) / (np.sqrt(v / (1 - b2 ** t)) + eps)
        else:
            v = b2 * v + (1 - b2) * (g.real ** 2 + 1j * g.imag ** 2)
            upd = ((m.real / (1 - b1 ** t)) / (np.sqrt(v.real / (1 - b2 ** t)) + eps)
                   + 1j * (m.imag / (1 - b1 ** t)) / (np.sqrt(v.imag / (1 - b2 ** t)) + eps))
        w = w * (1 - lr * wd) - lr * upd
    return w


def _as_storage(x, dtype):
    if dtype == "r32":
        return np.ascontiguousarray(x.real.astype(np.float32))
    if dtype == "c64":
        return np.ascontiguousarray(x.astype(np.complex64))
    if dtype == "c32h":
        return np.ascontiguousarray(np.stack([x.real, x.imag], -1).astype(np.float16))
    return np.ascontiguousarray(x.real.astype(np.float16))


def _from_storage(a, dtype):
    if dtype == "c32h":
        return a[..., 0].astype(np.float64) + 1j * a[..., 1].astype(np.float64)
    return a.astype(np.complex128)


@pytest.mark.parametrize("dtype", ["r32", "c64"])
@pytest.mark.parametrize("rho", [0.0, 0.1, 1.0])
@pytest.mark.parametrize("complex_mode", [0, 1])
def test_full_rank_reduces_to_adamw(oracle_mod, dtype, rho, complex_mode):
    """r_n = I_n for every mode: the core is the masked gradient itself and the
    sparse branch covers Omega, so from zero moments with a fixed Omega the
    step is textbook AdamW on every element, for any sparse ratio."""
    if dtype == "r32" and complex_mode == 1:
        pytest.skip("complex Adam mode only applies to complex tensors")
    shape = (3, 4, 5)
    r = rng(21)
    cplx = dtype == "c64"
    grads = [crandn(r, shape) if cplx else r.standard_normal(shape) for _ in range(4)]
    w0 = crandn(r, shape) * 0.02 if cplx else r.standard_normal(shape) * 0.02
    lr, b1, b2, eps, wd = 1e-2, 0.9, 0.999, 1e-8, 0.1
    o = oracle_mod.Oracle(shape, shape, rho, 100, lr, (b1, b2), eps, wd, dtype, dtype,
                          complex_adam=complex_mode)
    w = _as_storage(w0, dtype)
    gs = [_as_storage(g, dtype) for g in grads]
    for g in gs:
        assert o.step(g, w) == 0
    ref = textbook_adamw([_from_storage(g, dtype) for g in gs], _from_storage(_as_storage(w0, dtype), dtype),
                         lr, b1, b2, eps, wd, complex_mode if cplx else 0)
    got = _from_storage(w, dtype)
    assert np.abs(got - ref).max() <= 1e-6 * np.abs(ref).max()
    assert o.info["refreshes"] == 1 and o.info["k"] == math.floor(rho * 60)


def test_fp16_weights_rounded_once(oracle_mod):
    """c32h weights: one fp64 AdamW step rounded once to binary16 (numpy's
    float64 -> float16 conversion is the reference rounding)."""
    shape = (4, 3, 5)
    r = rng(3)
    g = crandn(r, shape)
    w0 = crandn(r, shape) * 0.02
    gs, ws = _as_storage(g, "c32h"), _as_storage(w0, "c32h")
    o = oracle_mod.Oracle(shape, shape, 0.0, 10, 1e-3, (0.9, 0.999), 1e-8, 0.01, "c32h", "c32h")
    w = ws.copy()
    o.step(gs, w)
    ref = textbook_adamw([_from_storage(gs, "c32h")], _from_storage(ws, "c32h"), 1e-3, 0.9, 0.999, 1e-8, 0.01)
    assert np.array_equal(w, _as_storage(ref, "c32h"))


def test_weight_decay_only(oracle_mod):
    shape = (4, 5, 3)
    r = rng(4)
    w0 = (r.standard_normal(shape) * 0.02).astype(np.float32)
    o = oracle_mod.Oracle(shape, (2, 2, 2), 0.05, 10, 1e-2, (0.9, 0.999), 1e-8, 0.5, "r32", "r32")
    w = w0.copy()
    o.step(np.zeros(shape, np.float32), w)
    assert np.array_equal(w, (w0.astype(np.float64) * (1 - 1e-2 * 0.5)).astype(np.float32))


@pytest.mark.parametrize("dtype", ["r32", "c64"])
def test_exact_tucker_recovered(oracle_mod, dtype):
    """An exactly Tucker-rank gradient with rho = 0 and the true ranks: the
    refreshed factors span the true mode subspaces and G x U^H x U = G."""
    shape, ranks = (10, 9, 8, 7), (3, 2, 4, 2)
    r = rng(8)
    cplx = dtype == "c64"
    Q = [orthonormal(r, I, c, cplx) for I, c in zip(shape, ranks)]
    x = crandn(r, ranks) if cplx else r.standard_normal(ranks)
    for n, q in enumerate(Q):
        x = np_mode_product(x, n, q)
    g = _as_storage(x, dtype)
    o = oracle_mod.Oracle(shape, ranks, 0.0, 1, grad_dtype=dtype, weight_dtype=dtype)
    o.refresh(g)
    Us = [o.get_U(n).astype(np.complex128) for n in range(4)]
    for n in range(4):
        assert projector_distance(Us[n], Q[n]) < 1e-5  # fp32-stored factors
        assert np.allclose(Us[n].conj().T @ Us[n], np.eye(ranks[n]), atol=1e-6)
    core = x.astype(np.complex128)
    xg = _from_storage(g, dtype)
    c = xg
    for n in range(4):
        c = oracle_mod.mode_product(c, n, Us[n], True)
    back = c
    for n in range(4):
        back = oracle_mod.mode_product(back, n, Us[n], False)
    assert np.abs(back - xg).max() < 1e-5 * np.abs(xg).max()
    # the fp64 tensor with its fp64 factors round-trips to fp64 rounding
    x64 = x.astype(np.complex128)
    c = x64
    for n in range(4):
        c = oracle_mod.mode_product(c, n, Q[n], True)
    back = c
    for n in range(4):
        back = oracle_mod.mode_product(back, n, Q[n], False)
    assert np.abs(back - x64).max() < 1e-12 * np.abs(x64).max()
    del core


def test_phase_flip_invariance(oracle_mod):
    """With zero moments, multiplying columns of U_n by unit phases leaves the
    step unchanged: Adam's first step is invariant to per-element phases."""
    shape, ranks = (6, 5, 4, 3), (3, 2, 2, 2)
    r = rng(9)
    g = _as_storage(crandn(r, shape), "c64")
    w0 = _as_storage(crandn(r, shape) * 0.02, "c64")
    a = oracle_mod.Oracle(shape, ranks, 0.1, 0, auto_refresh=0)
    a.refresh(g)
    b = oracle_mod.Oracle(shape, ranks, 0.1, 0, auto_refresh=0)
    b.refresh(g)
    for n in range(4):
        U = b.get_U(n)
        ph = np.exp(1j * r.uniform(0, 2 * np.pi, U.shape[1]))
        b.set_U(n, U * ph)
    wa, wb = w0.copy(), w0.copy()
    a.step(g, wa)
    b.step(g, wb)
    assert np.abs(wa - wb).max() < 1e-6 * np.abs(wa).max()


def test_sparse_scatter_positions(oracle_mod):
    """Low-rank branch switched off (U_n with zero-overlap is impossible, so use
    a gradient that vanishes off Omega): with G supported on Omega, R = 0, the
    core update is 0 and only Omega moves, by lambda * AdamW."""
    shape, ranks = (6, 5, 4), (2, 2, 2)
    r = rng(10)
    g = np.zeros(shape, np.complex128)
    idx = r.choice(120, 12, replace=False)
    g.reshape(-1)[idx] = crandn(r, 12) * 5
    gs = _as_storage(g, "c64")
    w0 = _as_storage(crandn(r, shape) * 0.02, "c64")
    lam = 0.5
    o = oracle_mod.Oracle(shape, ranks, 0.1, 10, 1e-2, sparse_scale=lam)
    w = w0.copy()
    o.step(gs, w)
    assert sorted(o.omega.tolist()) == sorted(idx.tolist())
    moved = np.flatnonzero(np.abs(w.reshape(-1) - w0.reshape(-1)) > 0)
    assert sorted(moved.tolist()) == sorted(idx.tolist())
    gi = g.reshape(-1)[idx]
    expect = w0.reshape(-1)[idx].astype(np.complex128) - 1e-2 * lam * gi / (np.abs(gi) + 1e-8)
    assert np.allclose(w.reshape(-1)[idx], expect, atol=1e-7)


def test_refresh_schedule(oracle_mod):
    shape = (4, 4, 3)
    r = rng(13)
    o = oracle_mod.Oracle(shape, (2, 2, 2), 0.1, 3, grad_dtype="r32", weight_dtype="r32")
    w = np.zeros(shape, np.float32)
    seen = []
    for t in range(7):
        o.step(r.standard_normal(shape).astype(np.float32), w)
        seen.append(o.info["refreshes"])
    assert seen == [1, 1, 1, 2, 2, 2, 3]
    o2 = oracle_mod.Oracle(shape, (2, 2, 2), 0.1, 0, auto_refresh=1, grad_dtype="r32", weight_dtype="r32")
    assert o2.step(np.ones(shape, np.float32), w) == 6  # never refreshed: state error


def test_moments_reset_option(oracle_mod):
    shape = (4, 4, 3)
    r = rng(14)
    g = r.standard_normal(shape).astype(np.float32)
    o = oracle_mod.Oracle(shape, (2, 2, 2), 0.1, 2, grad_dtype="r32", weight_dtype="r32",
                          moments_on_refresh=1)
    w = np.zeros(shape, np.float32)
    o.step(g, w)
    o.step(g, w)
    assert np.abs(o.get_moment("core_m")).max() > 0
    o.refresh(g)
    assert np.abs(o.get_moment("core_m")).max() == 0 and np.abs(o.get_moment("sparse_v")).max() == 0


def test_sampled_slabs_match_full_step(oracle_mod):
    shape, ranks = (5, 4, 6, 3), (2, 3, 2, 2)
    r = rng(15)
    g = _as_storage(crandn(r, shape), "c64")
    w0 = _as_storage(crandn(r, shape) * 0.02, "c64")
    a = oracle_mod.Oracle(shape, ranks, 0.05, 4)
    b = oracle_mod.Oracle(shape, ranks, 0.05, 4)
    wa, wb = w0.copy(), w0.copy()
    a.step(g, wa)
    sel = np.array([0, 7, 19], np.int64)
    b.step(g, wb, slabs=sel)
    wa2 = wa.reshape(20, 6, 3)
    wb2 = wb.reshape(20, 6, 3)
    w02 = w0.reshape(20, 6, 3)
    for s in range(20):
        if s in sel:
            assert np.array_equal(wa2[s], wb2[s])
        else:
            assert np.array_equal(wb2[s], w02[s])

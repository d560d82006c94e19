"""GPU parity: the CUDA library against the CPU oracle on the same seeded inputs.

Omega is compared bit for bit; factors by projector distance (eigenvector
phases are a convention, subspaces are unique when the eigengap is open);
weights and moments after teacher-forced steps (both sides start from the
same state) within the tolerance the method fixes: max relative error 1e-4
for fp32 gradients, 2e-3 for fp16 gradients.
"""

import math

import numpy as np
import pytest

from tests.helpers import TOL, as_complex, eigengap, projector_distance, random_moments, rel_err, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import rank_sparse_tensor_b200 as rst
    return rst


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


# (shape, ranks, gen_ranks, dtype, rho) -- sizes span several tiles with ragged tails
CASES = {
    "r32_16x16x8x8": ((16, 16, 8, 8), (4, 4, 2, 2), (4, 4, 2, 2), "r32", 0.05),
    "c64_64x64x32x17": ((64, 64, 32, 17), (16, 16, 8, 5), (16, 16, 8, 5), "c64", 0.05),
    "c32h_24x16x64x33": ((24, 16, 64, 33), (6, 4, 13, 7), (8, 4, 16, 9), "c32h", 0.05),
    "r16_12x10x9": ((12, 10, 9), (3, 3, 2), (3, 3, 2), "r16", 0.05),
    "c64_5way_8x6x8x4x17": ((8, 6, 8, 4, 17), (2, 3, 2, 2, 5), (2, 3, 2, 2, 5), "c64", 0.05),
    "c64_identity_modes": ((16, 8, 12, 5), (16, 3, 12, 2), (16, 3, 12, 2), "c64", 0.1),
    "c64_rho0": ((16, 12, 8, 9), (4, 3, 2, 3), (4, 3, 2, 3), "c64", 0.0),
    "c64_rho1": ((6, 5, 4, 3), (2, 2, 2, 2), (2, 2, 2, 2), "c64", 1.0),
    # Gram tiles: pairs of 64-row tiles with a ragged last tile (130, 70, 66),
    # and tile edges above I_n (9 -> 12, 5 -> 8)
    "c64_gram_pairs_130x20x9": ((130, 20, 9), (8, 5, 3), (8, 5, 3), "c64", 0.05),
    "c32h_gram_pairs_70x66x5": ((70, 66, 5), (6, 9, 2), (6, 9, 2), "c32h", 0.05),
    # tensor-core Grams of modes 64 < I_n <= 128: row boxes (B a multiple of
    # the chunk), whole slabs (B = 1), element copies (B = 48), for complex
    # and real, 32- and 16-bit values
    "c64_wide_96x32x8": ((96, 32, 8), (8, 4, 2), (8, 4, 2), "c64", 0.05),
    "c32h_wide_128x64": ((128, 64), (16, 8), (16, 8), "c32h", 0.05),
    "r32_wide_80x16x4": ((80, 16, 4), (8, 4, 2), (8, 4, 2), "r32", 0.05),
    "r16_wide_100x32": ((100, 32), (8, 4), (8, 4), "r16", 0.05),
    "r16_wide_72x48": ((72, 48), (6, 5), (6, 5), "r16", 0.05),
    "c64_wide_inner_5x100": ((5, 100), (2, 8), (2, 8), "c64", 0.05),
}


def _inputs(shape, gen_ranks, dtype, seed, steps=2):
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    gs = GradientStream(shape, gen_ranks, dtype, seed, outlier_frac=0.02, outlier_scale=10.0)
    grads = [to_np(gs.next()) for _ in range(steps)]
    return grads, to_np(weights(shape, dtype, seed))


def _gpu(lib, shape, ranks, rho, dtype, **kw):
    return lib.TensorGRaD(shape, ranks, rho, 0, lr=1e-3, wd=0.01, grad_dtype=dtype,
                          weight_dtype=dtype, auto_refresh=0, **kw)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("omega_mode", [0, 1])
def test_refresh_parity(lib, orc, name, omega_mode):
    shape, ranks, gen_ranks, dtype, rho = CASES[name]
    grads, _ = _inputs(shape, gen_ranks, dtype, seed=11)
    o = orc.Oracle(shape, ranks, rho, 0, grad_dtype=dtype, omega_mode=omega_mode, seed=5,
                   auto_refresh=0)
    o.refresh(grads[0])
    g = _gpu(lib, shape, ranks, rho, dtype, omega_mode=omega_mode, seed=5)
    g.refresh(torch.from_numpy(grads[0]).cuda())
    st = g.get_state()
    assert np.array_equal(st["omega"], o.omega)
    cplx = dtype in ("c64", "c32h")
    ov = o.omega_values()
    gv = st["omega_val"].reshape(-1, 2) if cplx else st["omega_val"]
    gv = gv[:, 0] + 1j * gv[:, 1] if cplx else gv.astype(np.complex128)
    assert np.array_equal(gv.astype(np.complex64), ov.astype(np.complex64))
    for n in range(len(shape)):
        if ranks[n] == shape[n]:
            assert np.array_equal(st["U"][n], np.eye(shape[n]))
            continue
        Uo = o.get_U(n)
        gap = eigengap(o.eigvals(n), ranks[n])
        d = projector_distance(st["U"][n], Uo)
        if gap > 1e-3:
            assert d <= 1e-3, (n, d, gap)
        assert np.allclose(st["U"][n].conj().T @ st["U"][n], np.eye(ranks[n]), atol=1e-5)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("complex_adam", [0, 1])
def test_teacher_forced_step(lib, orc, name, complex_adam):
    shape, ranks, gen_ranks, dtype, rho = CASES[name]
    cplx = dtype in ("c64", "c32h")
    if complex_adam and not cplx:
        pytest.skip("complex Adam mode applies to complex tensors")
    grads, w0 = _inputs(shape, gen_ranks, dtype, seed=3)
    o = orc.Oracle(shape, ranks, rho, 0, lr=1e-3, wd=0.01, grad_dtype=dtype,
                   complex_adam=complex_adam, auto_refresh=0)
    o.refresh(grads[0])
    g = _gpu(lib, shape, ranks, rho, dtype, complex_adam=complex_adam)
    rng = np.random.default_rng(7)
    mom = random_moments(rng, g.info, cplx)
    for key, v in mom.items():
        o.set_moment(key, v)
    o.set_counters(3, 1, True)
    state = dict(mom, omega=o.omega, U=[o.get_U(n) for n in range(len(shape))], t=3,
                 refreshes=1, has_subspace=True)
    g.set_state(state)
    w_ref = w0.copy()
    assert o.step(grads[1], w_ref) == 0
    w_dev = torch.from_numpy(w0.copy()).cuda()
    g.step(torch.from_numpy(grads[1]).cuda(), w_dev)
    g.sync()
    err = rel_err(to_np(w_dev), w_ref, dtype)
    assert err <= TOL[dtype], err
    st = g.get_state()
    for key in ("core_m", "core_v", "sparse_m", "sparse_v"):
        ref = o.get_moment(key)
        if ref.size:
            e = np.abs(st[key] - ref).max() / max(np.abs(ref).max(), 1e-30)
            assert e <= 10 * TOL[dtype], (key, e)
    assert st["t"] == 4


@pytest.mark.parametrize("dtype", ["r32", "c64", "c32h", "r16"])
@pytest.mark.parametrize("n,k,ties", [(1, 1, False), (1000, 0, False), (4097, 4097, False),
                                      (4097, 200, False), (100003, 5000, True),
                                      (300000, 15000, False)])
def test_topk_standalone_bit_exact(lib, orc, dtype, n, k, ties):
    rng = np.random.default_rng(n + k)
    if ties:
        re = rng.integers(-3, 4, n).astype(np.float32)
        im = rng.integers(-3, 4, n).astype(np.float32)
    else:
        re = rng.standard_normal(n).astype(np.float32)
        im = rng.standard_normal(n).astype(np.float32)
    g = {"r32": re, "r16": re.astype(np.float16), "c64": (re + 1j * im).astype(np.complex64),
         "c32h": np.stack([re, im], -1).astype(np.float16)}[dtype]
    om, vals = lib.topk_select(torch.from_numpy(g).cuda(), dtype, k)
    ref = orc.topk(g, dtype, k)
    assert np.array_equal(to_np(om), ref)
    if k:
        flat = (g.view(np.float32) if dtype == "c64" else g).reshape(n, -1).astype(np.float32)
        assert np.array_equal(to_np(vals).reshape(k, -1), flat[ref])


def test_free_running_trajectory_small(lib, orc):
    """Auto-refresh schedule on both sides from zero state (reported; gated
    loosely because refreshes may pick different near-degenerate subspaces)."""
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    shape, ranks, dtype = (16, 16, 8, 8), (4, 4, 2, 2), "r32"
    gs = GradientStream(shape, ranks, dtype, 1, outlier_frac=0.01)
    w = to_np(weights(shape, dtype, 1))
    o = orc.Oracle(shape, ranks, 0.05, 5, grad_dtype=dtype)
    g = lib.TensorGRaD(shape, ranks, 0.05, 5, grad_dtype=dtype)
    w_ref = w.copy()
    w_dev = torch.from_numpy(w.copy()).cuda()
    errs = []
    for t in range(10):
        gr = to_np(gs.next())
        o.step(gr, w_ref)
        g.step(torch.from_numpy(gr).cuda(), w_dev)
        errs.append(rel_err(to_np(w_dev), w_ref, dtype))
    assert g.info["refreshes"] == 2 and g.info["t"] == 10
    assert max(errs) < 1e-3, errs


def test_state_round_trip(lib, orc):
    shape, ranks, gen_ranks, dtype, rho = CASES["c64_64x64x32x17"]
    grads, w0 = _inputs(shape, gen_ranks, dtype, seed=9)
    g = _gpu(lib, shape, ranks, rho, dtype)
    g.refresh(torch.from_numpy(grads[0]).cuda())
    w = torch.from_numpy(w0.copy()).cuda()
    g.step(torch.from_numpy(grads[1]).cuda(), w)
    s1 = g.get_state()
    h = _gpu(lib, shape, ranks, rho, dtype)
    h.set_state(s1)
    s2 = h.get_state()
    for key in ("omega", "core_m", "core_v", "sparse_m", "sparse_v"):
        assert np.array_equal(s1[key], s2[key])
    for a, b in zip(s1["U"], s2["U"]):
        assert np.array_equal(a, b)
    # resumed and uninterrupted runs stay bit-identical
    w1, w2 = w.clone(), w.clone()
    g.step(torch.from_numpy(grads[0]).cuda(), w1)
    h.step(torch.from_numpy(grads[0]).cuda(), w2)
    assert torch.equal(w1, w2)


def test_step_before_refresh_is_a_state_error(lib):
    g = lib.TensorGRaD((8, 8, 8), (2, 2, 2), 0.05, 0, grad_dtype="c64")
    x = torch.zeros((8, 8, 8), dtype=torch.complex64, device="cuda")
    with pytest.raises(lib.TgdError) as e:
        g.step(x, x.clone())
    assert e.value.name == "STATE"


def test_bad_state_rejected(lib):
    g = lib.TensorGRaD((8, 8, 8), (2, 2, 2), 0.05, 0, grad_dtype="c64")
    k = g.info["k"]
    with pytest.raises(lib.TgdError) as e:
        g.set_state({"omega": np.arange(k)[::-1].copy()})
    assert e.value.name == "INVALID_ARG"


@pytest.mark.parametrize("dtype,shape,ranks,path", [
    ("r32", (16, 12, 8, 9), (4, 3, 2, 3), "generic"),     # CUDA-core path
    ("c32h", (4, 8, 64, 33), (2, 4, 16, 8), "tcgen05"),   # tensor-core path, fp16
    ("c64", (16, 12, 8, 9), (4, 3, 2, 3), "tcgen05"),     # tensor-core path, fp32
])
def test_step_host_equals_device_step(lib, dtype, shape, ranks, path):
    """tgd_step_host (host buffers, copies inside the call) leaves bit for bit
    the weights tgd_step leaves from the same state."""
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    g = GradientStream(shape, ranks, dtype, 4, outlier_frac=0.02, outlier_scale=10.0).next()
    w = weights(shape, dtype, 4)
    a = _gpu(lib, shape, ranks, 0.05, dtype, path=path)
    b = _gpu(lib, shape, ranks, 0.05, dtype, path=path)
    g_dev, w_dev = g.cuda(), w.cuda()
    a.refresh(g_dev)
    b.refresh(g_dev)
    a.step(g_dev, w_dev)
    a.sync()
    g_host, w_host = to_np(g).copy(), to_np(w).copy()
    b.step_host(g_host, w_host)
    assert np.array_equal(to_np(w_dev).view(np.uint8), w_host.view(np.uint8))
    assert not np.array_equal(w_host, to_np(w))
    assert a.get_state()["t"] == b.get_state()["t"] == 1


@pytest.mark.parametrize("name", ["c64_64x64x32x17", "c32h_24x16x64x33", "c64_gram_pairs_130x20x9"])
def test_second_refresh_starts_from_the_first(lib, orc, name):
    """A refresh after the first starts the eigensolver from the previous
    eigenvectors; its factors must still be those of the new gradient's
    Grams (projector distance to the oracle's cold solve where the gap is
    open), and orthonormal."""
    shape, ranks, gen_ranks, dtype, rho = CASES[name]
    grads, _ = _inputs(shape, gen_ranks, dtype, seed=21, steps=3)
    g = _gpu(lib, shape, ranks, rho, dtype)
    for gr in grads:
        g.refresh(torch.from_numpy(gr).cuda())
    st = g.get_state()
    o = orc.Oracle(shape, ranks, rho, 0, grad_dtype=dtype, auto_refresh=0)
    o.refresh(grads[-1])
    assert np.array_equal(st["omega"], o.omega)
    for n in range(len(shape)):
        if ranks[n] == shape[n]:
            continue
        U = st["U"][n].astype(np.complex128)
        assert np.allclose(U.conj().T @ U, np.eye(ranks[n]), atol=1e-5)
        if eigengap(o.eigvals(n), ranks[n]) > 1e-3:
            assert projector_distance(U, o.get_U(n)) <= 1e-3

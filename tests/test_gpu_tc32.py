"""GPU parity of the tensor-core (tcgen05) step path for fp32 gradients.

Teacher-forced: the oracle and the kernel path start from the same state
(Omega, factors, non-zero moments, step count); the weights, their change
over the step and the moments are compared after one step. Shapes cover one
and several K chunks per mode (32 complex or 64 real entries per chunk),
outputs wider than one tensor-core tile (more than 128 complex columns), a
trailing full-rank mode (the weight update then runs with a stride), real and
complex tensors, 3 to 5 modes, and rho = 0 and 1.
"""

import numpy as np
import pytest

from tests.helpers import TOL, random_moments, rel_err, to_np

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


# name: (shape, ranks, dtype, rho)
CASES = {
    "c64_fno_64x64x32x17": ((64, 64, 32, 17), (16, 16, 8, 5), "c64", 0.05),
    "c64_5way": ((8, 6, 8, 4, 17), (2, 3, 2, 2, 5), "c64", 0.05),
    "c64_trailing_full_rank": ((16, 12, 8, 9), (4, 3, 2, 9), "c64", 0.05),
    "c64_wide_mode_130": ((130, 20, 9), (8, 5, 3), "c64", 0.05),
    "c64_one_projected_mode": ((12, 40, 6), (12, 7, 6), "c64", 0.1),
    "c64_rho0": ((16, 12, 8, 9), (4, 3, 2, 3), "c64", 0.0),
    "c64_rho1": ((6, 5, 4, 3), (2, 2, 2, 2), "c64", 1.0),
    "r32_16x16x8x8": ((16, 16, 8, 8), (4, 4, 2, 2), "r32", 0.05),
    "r32_3way": ((7, 6, 9), (3, 2, 4), "r32", 0.05),
    "r32_two_chunks_70x66x5": ((70, 66, 5), (6, 9, 2), "r32", 0.05),
    # innermost-mode launches over whole 128-row tiles plus a ragged one (300 rows)
    "c64_ragged_tail_10x30x17": ((10, 30, 17), (3, 6, 5), "c64", 0.05),
    "r32_ragged_tail_5x52x33": ((5, 52, 33), (2, 6, 7), "r32", 0.05),
}


def _run(lib, orc, shape, ranks, dtype, rho, complex_adam=0, seed=3, wd=0.01):
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    gs = GradientStream(shape, ranks, dtype, seed, outlier_frac=0.02, outlier_scale=10.0)
    g0, g1 = to_np(gs.next()), to_np(gs.next())
    w0 = to_np(weights(shape, dtype, seed))
    o = orc.Oracle(shape, ranks, rho, 0, lr=1e-3, wd=wd, grad_dtype=dtype, complex_adam=complex_adam,
                   auto_refresh=0)
    o.refresh(g0)
    g = lib.TensorGRaD(shape, ranks, rho, 0, lr=1e-3, wd=wd, grad_dtype=dtype,
                       complex_adam=complex_adam, auto_refresh=0, path="tcgen05")
    assert g.info["path"] == "tcgen05"
    mom = random_moments(np.random.default_rng(5), g.info, dtype == "c64")
    for key, v in mom.items():
        o.set_moment(key, v)
    o.set_counters(2, 1, True)
    g.set_state(dict(mom, omega=o.omega, U=[o.get_U(n) for n in range(len(shape))], t=2,
                     refreshes=1, has_subspace=True))
    w_ref = w0.copy()
    assert o.step(g1, w_ref) == 0
    w_dev = torch.from_numpy(w0.copy()).cuda()
    g.step(torch.from_numpy(g1).cuda(), w_dev)
    g.sync()
    return o, g, to_np(w_dev), w_ref, w0


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("complex_adam", [0, 1])
def test_tc32_teacher_forced_step(lib, orc, name, complex_adam):
    shape, ranks, dtype, rho = CASES[name]
    if complex_adam and dtype != "c64":
        pytest.skip("complex Adam mode applies to complex tensors")
    o, g, w, w_ref, w0 = _run(lib, orc, shape, ranks, dtype, rho, complex_adam)
    assert rel_err(w, w_ref, dtype) <= TOL[dtype]
    dw = w.astype(np.complex128) - w0.astype(np.complex128)
    dw_ref = w_ref.astype(np.complex128) - w0.astype(np.complex128)
    upd = np.abs(dw - dw_ref).max() / np.abs(dw_ref).max()
    assert upd <= 1e-4, upd
    st = g.get_state()
    for key in ("core_m", "core_v", "sparse_m", "sparse_v"):
        ref = o.get_moment(key)
        if ref.size:
            e = np.abs(st[key] - ref).max() / max(np.abs(ref).max(), 1e-30)
            assert e <= 1e-4, (key, e)
    assert st["t"] == 3


def test_tc32_agrees_with_generic_over_steps(lib):
    """Both kernel paths follow the same trajectory with automatic refreshes."""
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    shape, ranks = (16, 12, 8, 17), (4, 3, 2, 5)
    gs = GradientStream(shape, ranks, "c64", 9, outlier_frac=0.02)
    w0 = weights(shape, "c64", 9).cuda()
    a = lib.TensorGRaD(shape, ranks, 0.05, 3, grad_dtype="c64", path="tcgen05")
    b = lib.TensorGRaD(shape, ranks, 0.05, 3, grad_dtype="c64", path="generic")
    wa, wb = w0.clone(), w0.clone()
    for _ in range(7):
        gr = gs.next().cuda()
        a.step(gr, wa)
        b.step(gr, wb)
    a.sync()
    b.sync()
    assert a.info["refreshes"] == 3
    assert rel_err(to_np(wa), to_np(wb), "c64") <= TOL["c64"]

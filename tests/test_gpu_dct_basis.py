"""GPU parity of the DCT factor basis (dynamic column selection as a refresh)
against the oracle's Oracle(basis=1): Omega bit-exact, each mode's factors by
projector distance wherever the alignment gap at r_n is open, the
alignments themselves to fp32-Gram accuracy."""

import numpy as np
import pytest

from tests.helpers import eigengap, projector_distance, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

CASES = {
    "c64_4way": ((16, 12, 8, 9), (4, 3, 2, 3), "c64", 0.05),
    "c32h_4way": ((4, 8, 64, 33), (2, 4, 16, 8), "c32h", 0.05),
    "r32_3way": ((20, 12, 9), (5, 3, 2), "r32", 0.1),
    "c64_pairs_130": ((130, 20, 9), (8, 5, 3), "c64", 0.05),
}


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


@pytest.mark.parametrize("name", list(CASES))
def test_dct_refresh(lib, orc, name):
    from rank_sparse_tensor_b200.synth import GradientStream
    shape, ranks, dtype, rho = CASES[name]
    g = to_np(GradientStream(shape, ranks, dtype, 11, outlier_frac=0.02, outlier_scale=10.0).next())
    o = orc.Oracle(shape, ranks, rho, 0, grad_dtype=dtype, auto_refresh=0, basis=1)
    o.refresh(g)
    h = lib.TensorGRaD(shape, ranks, rho, 0, grad_dtype=dtype, auto_refresh=0, basis=1)
    h.refresh(torch.from_numpy(g).cuda())
    st = h.get_state()
    assert np.array_equal(st["omega"], o.omega)
    for n in range(len(shape)):
        if ranks[n] == shape[n]:
            continue
        if eigengap(o.eigvals(n), ranks[n]) > 1e-3:
            assert projector_distance(st["U"][n], o.get_U(n)) <= 1e-3, n
        # the factors are DCT columns: real, orthonormal
        U = st["U"][n]
        assert np.abs(U.imag).max() == 0
        assert np.allclose(U.conj().T @ U, np.eye(ranks[n]), atol=1e-5)


def test_dct_and_hosvd_differ(lib):
    """The two bases are different factors for a generic gradient."""
    from rank_sparse_tensor_b200.synth import GradientStream
    shape, ranks = (16, 12, 8, 9), (4, 3, 2, 3)
    g = GradientStream(shape, ranks, "c64", 3, device="cuda").next()
    U = []
    for basis in (0, 1):
        h = lib.TensorGRaD(shape, ranks, 0.05, 0, grad_dtype="c64", auto_refresh=0, basis=basis)
        h.refresh(g)
        U.append(h.get_state()["U"][0])
    assert projector_distance(U[0], U[1]) > 1e-2

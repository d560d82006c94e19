"""Failure detection on the GPU without a fault: a bounded wait runs out.

Every wait inside the tensor-core kernels is bounded; when one runs out the
kernel sets an error bit, stops its work, waits (again bounded) for the copies
and tensor-core operations it has in flight, frees its tensor memory and
returns. The test hook `test_stall` makes the projection kernel's first CTA
skip the load of its first tile, so the wait for that tile is on a barrier
nothing will complete; with `wait_limit_ms` = 20 it gives up after 20 ms. The
host must then see TGD_ERR_TIMEOUT on the next synchronising call, the error
word must be cleared by that report, and the device must stay usable: a
normal step afterwards matches the oracle.
"""

import time

import numpy as np
import pytest

from tests.helpers import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

SHAPE, RANKS = (16, 8, 32, 17), (4, 2, 8, 5)


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


def _inputs():
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    gs = GradientStream(SHAPE, RANKS, "c32h", 5, outlier_frac=0.02)
    return to_np(gs.next()), to_np(gs.next()), to_np(weights(SHAPE, "c32h", 5))


def test_wait_that_runs_out_is_reported(lib, orc):
    g0, g1, w0 = _inputs()
    bad = lib.TensorGRaD(SHAPE, RANKS, 0.05, 0, grad_dtype="c32h", auto_refresh=0,
                         wait_limit_ms=20, test_stall=1)
    assert bad.info["path"] == "tcgen05"
    bad.refresh(torch.from_numpy(g0).cuda())
    bad.sync()
    w = torch.from_numpy(w0.copy()).cuda()
    t0 = time.perf_counter()
    bad.step(torch.from_numpy(g1).cuda(), w)
    with pytest.raises(lib.TgdError) as e:
        bad.sync()
    elapsed = time.perf_counter() - t0
    assert e.value.name == "TIMEOUT"
    assert elapsed < 5.0, elapsed          # 20 ms limit, not the default 2 s
    bad.sync()                             # the report cleared the error word
    bad.close()

    # the context is intact: a normal handle's teacher-forced step matches
    # the oracle
    o = orc.Oracle(SHAPE, RANKS, 0.05, 0, grad_dtype="c32h", auto_refresh=0)
    o.refresh(g0)
    good = lib.TensorGRaD(SHAPE, RANKS, 0.05, 0, grad_dtype="c32h", auto_refresh=0)
    good.set_state({"omega": o.omega, "U": [o.get_U(n) for n in range(4)], "t": 0,
                    "refreshes": 1, "has_subspace": True})
    w_ref = w0.copy()
    o.step(g1, w_ref)
    w = torch.from_numpy(w0.copy()).cuda()
    good.step(torch.from_numpy(g1).cuda(), w)
    good.sync()
    assert rel_err(to_np(w), w_ref, "c32h") <= TOL["c32h"]


def test_wait_limit_alone_changes_nothing(lib):
    """A short limit without the stall: waits that complete are unaffected
    and the weights are bit-identical to the default limit's."""
    g0, g1, w0 = _inputs()
    out = []
    for limit in (0, 50):
        opt = lib.TensorGRaD(SHAPE, RANKS, 0.05, 0, grad_dtype="c32h", auto_refresh=0,
                             wait_limit_ms=limit)
        opt.refresh(torch.from_numpy(g0).cuda())
        w = torch.from_numpy(w0.copy()).cuda()
        opt.step(torch.from_numpy(g1).cuda(), w)
        opt.sync()
        out.append(to_np(w))
    assert np.array_equal(out[0].view(np.uint8), out[1].view(np.uint8))

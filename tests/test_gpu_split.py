"""One tensor split across devices along mode 0, emulated on one GPU.

A tensor's mode-0 product of the projection sums over mode 0's rows, so a
block of rows projects to a partial core and the whole core is the sum of the
blocks' partial cores. Each block is a handle with `mode0_total` set, holding
its rows of U_0, its share of Omega (rebased to the block) and its sparse
moments; the core moments are replicated. The blocks' partial cores are
summed between tgd_step_begin and tgd_step_end (here with torch on the one
GPU, standing in for an all-reduce over GPUs), and the concatenated weights
are compared element by element with the oracle's step on the whole tensor.
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


# name: (shape, ranks, dtype, blocks, path)
CASES = {
    "c32h_tensor_core_2": ((8, 8, 64, 33), (4, 4, 16, 8), "c32h", 2, "tcgen05"),
    "c64_tensor_core_3": ((10, 12, 8, 17), (4, 3, 2, 5), "c64", 3, "tcgen05"),
    "r32_tensor_core_2": ((12, 6, 9), (5, 2, 4), "r32", 2, "tcgen05"),
    "c64_generic_3": ((10, 12, 8, 17), (4, 3, 2, 5), "c64", 3, "generic"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_split_step_equals_whole_step(lib, orc, name):
    from rank_sparse_tensor_b200.synth import GradientStream, weights
    shape, ranks, dtype, nb, path = CASES[name]
    cplx = dtype in ("c64", "c32h")
    gs = GradientStream(shape, ranks, dtype, 7, outlier_frac=0.02, outlier_scale=10.0)
    g0, g1 = to_np(gs.next()), to_np(gs.next())
    w0 = to_np(weights(shape, dtype, 7))
    rho = 0.05
    o = orc.Oracle(shape, ranks, rho, 0, lr=1e-3, wd=0.01, grad_dtype=dtype, auto_refresh=0)
    o.refresh(g0)
    omega = o.omega
    U = [o.get_U(n) for n in range(len(shape))]
    whole = lib.TensorGRaD(shape, ranks, rho, 0, lr=1e-3, wd=0.01, grad_dtype=dtype, auto_refresh=0)
    mom = random_moments(np.random.default_rng(8), whole.info, cplx)
    whole.close()
    for key, v in mom.items():
        o.set_moment(key, v)
    o.set_counters(2, 1, True)
    w_ref = w0.copy()
    assert o.step(g1, w_ref) == 0

    from rank_sparse_tensor_b200 import split
    state = dict(mom, omega=omega, U=U, t=2, refreshes=1, has_subspace=True)
    handles, grads, ws = [], [], []
    for blk in range(nb):
        b0, b1 = split.block_rows(shape[0], nb, blk)
        mine = split.block_state(state, shape, b0, b1, cplx)
        bshape = (b1 - b0,) + tuple(shape[1:])
        h = lib.TensorGRaD(bshape, ranks, rho, 0, lr=1e-3, wd=0.01, grad_dtype=dtype, auto_refresh=0,
                           path=path, sparse_k=mine["k"], mode0_total=shape[0])
        assert h.info["path"] == path
        assert h.info["k"] == mine["k"]
        h.set_state({key: v for key, v in mine.items() if key != "k"})
        handles.append(h)
        grads.append(torch.from_numpy(np.ascontiguousarray(g1[b0:b1])).cuda())
        ws.append(torch.from_numpy(np.ascontiguousarray(w0[b0:b1])).cuda())
    for h, g in zip(handles, grads):
        h.step_begin(g)
    cores = [h.core_tensor() for h in handles]
    total = torch.stack(cores).sum(0)
    for c in cores:
        c.copy_(total)
    for h, w in zip(handles, ws):
        h.step_end(w)
    torch.cuda.synchronize()
    w = np.concatenate([to_np(x) for x in ws], axis=0)
    assert rel_err(w, w_ref, dtype) <= TOL[dtype]
    # the replicated core moments agree with the whole tensor's
    ref_m = o.get_moment("core_m")
    for h in handles:
        st = h.get_state()
        assert st["t"] == 3
        e = np.abs(st["core_m"] - ref_m).max() / np.abs(ref_m).max()
        assert e <= (2.5e-2 if dtype == "c32h" else 1e-3), e


def test_split_calls_out_of_order_are_state_errors(lib):
    shape, ranks = (4, 8, 64, 33), (4, 4, 16, 8)
    h = lib.TensorGRaD(shape, ranks, 0.05, 0, grad_dtype="c32h", auto_refresh=0, mode0_total=8,
                       sparse_k=10)
    g = torch.zeros(shape + (2,), dtype=torch.float16, device="cuda")
    with pytest.raises(lib.TgdError) as e:
        h.step(g, g.clone())                 # a block steps only in two halves
    assert e.value.name == "STATE"
    with pytest.raises(lib.TgdError) as e:
        h.step_end(g.clone())                # end without begin
    assert e.value.name == "STATE"
    with pytest.raises(lib.TgdError) as e:
        h.refresh(g)                         # a block has no refresh of its own
    assert e.value.name == "UNSUPPORTED"

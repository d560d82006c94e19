"""The top-k entry point that allocates nothing, for callers that cannot
allocate device memory (it keeps its scratch in a fixed array inside the
library). Checked through the C ABI against tgd_topk_select, which uses a
caller workspace, on two calls in a row: the fixed array keeps the first
call's contents and the second call must not depend on them.

This file is collected last on purpose, so that a run stopping at the first
failure has run every other test first.
"""

import ctypes as C

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_sparse_tensor_b200 import native as nat
    nat.lib()
    return nat


def _select(nat, fn, g, dtype, n, k, static):
    cplx = dtype in ("c64", "c32h")
    om = torch.full((k,), -1, dtype=torch.int64, device="cuda")
    val = torch.full((k * (2 if cplx else 1),), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    L = nat.lib()
    if static:
        st = L.tgd_topk_select_static(g.data_ptr(), nat.DTYPES[dtype], n, k, om.data_ptr(),
                                      val.data_ptr(), stream)
    else:
        wsb = int(L.tgd_topk_workspace_bytes(n))
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        st = L.tgd_topk_select(g.data_ptr(), nat.DTYPES[dtype], n, k, om.data_ptr(), val.data_ptr(),
                               ws.data_ptr(), wsb, stream)
    assert st == 0, L.tgd_last_error(None)
    torch.cuda.synchronize()
    return om.cpu().numpy(), val.cpu().numpy()


def _grad(seed, n, dtype, ties):
    g = torch.Generator().manual_seed(seed)
    if ties:
        x = torch.randint(-3, 4, (n, 2), generator=g).float()
    else:
        x = torch.randn(n, 2, generator=g)
    if dtype == "c64":
        return torch.view_as_complex(x.contiguous()).cuda()
    return x.half().contiguous().cuda()


@pytest.mark.parametrize("dtype", ["c64", "c32h"])
def test_static_matches_workspace_version_twice(native, dtype):
    # two calls in a row with different inputs and sizes
    for seed, n, k, ties in [(1, 3_000_017, 150_000, False), (2, 1_000_003, 77_777, True)]:
        g = _grad(seed, n, dtype, ties)
        a_idx, a_val = _select(native, None, g, dtype, n, k, static=True)
        b_idx, b_val = _select(native, None, g, dtype, n, k, static=False)
        assert np.array_equal(a_idx, b_idx)
        assert np.array_equal(a_val, b_val)
        assert np.all(np.diff(a_idx) > 0)


def test_static_rejects_sizes_beyond_the_array(native):
    L = native.lib()
    n = native.TOPK_STATIC_MAX_N + 1
    st = L.tgd_topk_select_static(None, 1, n, 10, None, None, None)
    assert st == 1
    assert b"TGD_TOPK_STATIC_MAX_N" in L.tgd_last_error(None)

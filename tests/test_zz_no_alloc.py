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


def _select(nat, g, dtype, n, k, static, with_val=True):
    cplx = dtype in ("c64", "c32h")
    om = torch.full((max(k, 1),), -1, dtype=torch.int64, device="cuda")
    val = torch.full((max(k, 1) * (2 if cplx else 1),), float("nan"), dtype=torch.float32,
                     device="cuda")
    vp = val.data_ptr() if with_val else None
    stream = torch.cuda.current_stream().cuda_stream
    L = nat.lib()
    if static:
        st = L.tgd_topk_select_static(g.data_ptr(), nat.DTYPES[dtype], n, k, om.data_ptr(), vp,
                                      stream)
    else:
        wsb = int(L.tgd_topk_workspace_bytes(n))
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        st = L.tgd_topk_select(g.data_ptr(), nat.DTYPES[dtype], n, k, om.data_ptr(), vp,
                               ws.data_ptr(), wsb, stream)
    assert st == 0, L.tgd_last_error(None)
    torch.cuda.synchronize()
    return om.cpu().numpy()[:k], val.cpu().numpy()


def _grad(seed, n, dtype, ties):
    """n elements of `dtype` on the device (integer-valued when ties is set,
    so that magnitudes repeat)."""
    g = torch.Generator().manual_seed(seed)
    cplx = dtype in ("c64", "c32h")
    shape = (n, 2) if cplx else (n,)
    if ties:
        x = torch.randint(-3, 4, shape, generator=g).float()
    else:
        x = torch.randn(shape, generator=g)
    if dtype == "c64":
        return torch.view_as_complex(x.contiguous()).cuda()
    if dtype == "r32":
        return x.contiguous().cuda()
    return x.half().contiguous().cuda()


@pytest.mark.parametrize("dtype", ["r32", "c64", "c32h", "r16"])
def test_static_matches_workspace_version_twice(native, dtype):
    # two calls in a row with different inputs and sizes
    for seed, n, k, ties in [(1, 3_000_017, 150_000, False), (2, 1_000_003, 77_777, True)]:
        g = _grad(seed, n, dtype, ties)
        a_idx, a_val = _select(native, g, dtype, n, k, static=True)
        b_idx, b_val = _select(native, g, dtype, n, k, static=False)
        assert np.array_equal(a_idx, b_idx)
        assert np.array_equal(a_val, b_val)
        assert np.all(np.diff(a_idx) > 0)


def test_static_all_entries_and_no_values(native):
    # k == n (every index, no scratch used) and a NULL value output
    n = 100_003
    g = _grad(3, n, "c32h", False)
    a_idx, _ = _select(native, g, "c32h", n, n, static=True)
    b_idx, _ = _select(native, g, "c32h", n, n, static=False)
    assert np.array_equal(a_idx, np.arange(n))
    assert np.array_equal(a_idx, b_idx)
    k = 5_000
    a_idx, _ = _select(native, g, "c32h", n, k, static=True, with_val=False)
    b_idx, _ = _select(native, g, "c32h", n, k, static=False, with_val=False)
    assert np.array_equal(a_idx, b_idx)


def test_static_at_the_size_limit(native):
    # n = TGD_TOPK_STATIC_MAX_N exactly (fp16 reals, 512 MiB): the fixed array
    # is large enough for the biggest selection it accepts
    n = native.TOPK_STATIC_MAX_N
    gen = torch.Generator(device="cuda").manual_seed(4)
    g = torch.randint(-3, 4, (n,), generator=gen, device="cuda", dtype=torch.int16).half()
    k = n // 20
    a_idx, a_val = _select(native, g, "r16", n, k, static=True)
    b_idx, b_val = _select(native, g, "r16", n, k, static=False)
    assert np.array_equal(a_idx, b_idx)
    assert np.array_equal(a_val, b_val)
    del g
    torch.cuda.empty_cache()


def test_static_rejects_sizes_beyond_the_array(native):
    L = native.lib()
    n = native.TOPK_STATIC_MAX_N + 1
    st = L.tgd_topk_select_static(None, 1, n, 10, None, None, None)
    assert st == 1
    assert b"TGD_TOPK_STATIC_MAX_N" in L.tgd_last_error(None)

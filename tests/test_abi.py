"""The C ABI library builds, loads and exports every entry point that
include/tgd.h declares; argument checks run on the host (no GPU needed)."""

import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "tgd.h")).read()
    return sorted(set(re.findall(r"^TGD_API\s+[\w\s\*]+?\b(tgd_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def tgd():
    from rank_sparse_tensor_b200 import build, native
    build.build()
    return native


def test_header_declares_the_three_core_calls():
    names = declared_functions()
    for n in ("tgd_create", "tgd_step", "tgd_refresh", "tgd_destroy"):
        assert n in names


def test_every_declared_symbol_is_exported(tgd):
    out = subprocess.run(["nm", "-D", "--defined-only", tgd.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (tgd_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    L = tgd.lib()
    for n in declared_functions():
        assert hasattr(L, n)
    assert set(tgd.SIGNATURES) >= set(declared_functions())


def _create(tgd, shape, ranks, rho=0.05, T=5, gdt=1, wdt=1, opt=None):
    h = C.c_void_p()
    sh = (C.c_int64 * len(shape))(*shape)
    rk = (C.c_int64 * len(ranks))(*ranks)
    st = tgd.lib().tgd_create(C.byref(h), len(shape), sh, rk, rho, T, 1e-3, 0.9, 0.999, 1e-8, 0.0,
                              gdt, wdt, opt)
    return st, h


@pytest.mark.parametrize("shape,ranks,rho,T,gdt,wdt", [
    ((4, 4, 4), (5, 4, 4), 0.05, 5, 1, 1),     # rank above the mode size
    ((4, 4, 4), (0, 4, 4), 0.05, 5, 1, 1),     # zero rank
    ((4, 4, 4), (2, 2, 2), 1.5, 5, 1, 1),      # ratio above 1
    ((4, 4, 4), (2, 2, 2), -0.1, 5, 1, 1),     # negative ratio
    ((4, 4, 4), (2, 2, 2), 0.05, -1, 1, 1),    # negative period
    ((4, 4, 4), (2, 2, 2), 0.05, 5, 0, 1),     # real gradient, complex weight
    ((4, 4, 4), (2, 2, 2), 0.05, 5, 9, 9),     # unknown dtype
    ((4,), (2,), 0.05, 5, 1, 1),               # one mode
    ((4, 0, 4), (2, 0, 2), 0.05, 5, 1, 1),     # empty mode
    ((2,) * 9, (1,) * 9, 0.05, 5, 1, 1),       # more modes than supported
    ((1 << 21, 1 << 21), (1 << 21, 1 << 21), 0.05, 5, 1, 1),  # more elements than supported
])
def test_create_rejects_bad_arguments(tgd, shape, ranks, rho, T, gdt, wdt):
    st, h = _create(tgd, shape, ranks, rho, T, gdt, wdt)
    assert st == 1 and not h.value
    assert tgd.lib().tgd_last_error(None)


def test_unsupported_projected_mode(tgd):
    """A projected mode above 256 entries (the eigensolver's limit) is
    reported as unsupported; the same mode at full rank (identity) is not
    projected and passes the argument checks."""
    st, h = _create(tgd, (300, 4, 4), (10, 2, 2))
    assert st == 2 and not h.value  # TGD_ERR_UNSUPPORTED


def test_null_arguments(tgd):
    L = tgd.lib()
    assert L.tgd_step(None, None, None, None) == 1
    assert L.tgd_refresh(None, None, None) == 1
    assert L.tgd_destroy(None) == 0
    assert L.tgd_topk_select(None, 1, 10, 20, None, None, None, 0, None) == 1  # k > n
    assert L.tgd_topk_select(None, 1, 10, 0, None, None, None, 0, None) == 0   # k == 0: nothing
    assert L.tgd_topk_workspace_bytes(1 << 20) > 0


def test_default_options(tgd):
    o = tgd.Options()
    tgd.lib().tgd_default_options(C.byref(o))
    assert (o.omega_mode, o.sparse_scale, o.complex_adam, o.moments_on_refresh, o.auto_refresh,
            o.path, o.sm_budget, o.order, o.basis) == (0, 1.0, 0, 0, 1, 0, 0, 0, 0)


@pytest.mark.parametrize("order,path,status", [(2, 0, 1), (-1, 0, 1), (1, 2, 2)])
def test_bad_decomposition_order(tgd, order, path, status):
    """Orders other than 0 and 1 are invalid; the low-rank-first order on
    the forced tensor-core path is unsupported. Both fail before the device."""
    o = tgd.Options()
    tgd.lib().tgd_default_options(C.byref(o))
    o.order, o.path = order, path
    st, h = _create(tgd, (4, 8, 16), (2, 4, 8), opt=C.byref(o))
    assert st == status and not h.value


@pytest.mark.parametrize("basis", [-1, 2])
def test_bad_factor_basis(tgd, basis):
    o = tgd.Options()
    tgd.lib().tgd_default_options(C.byref(o))
    o.basis = basis
    st, h = _create(tgd, (4, 8, 16), (2, 4, 8), opt=C.byref(o))
    assert st == 1 and not h.value


def test_create_without_device_fails_cleanly(tgd):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    st, h = _create(tgd, (8, 8, 8), (2, 2, 2))
    assert st == 4 and not h.value  # TGD_ERR_CUDA


def test_product_path_has_no_cpu_fallback():
    """The product package never imports the oracle, and loading fails loudly
    when the CUDA library is absent."""
    pkg = os.path.join(ROOT, "rank_sparse_tensor_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn
    native_src = open(os.path.join(pkg, "native.py")).read()
    assert "raise RuntimeError" in native_src

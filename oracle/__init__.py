"""CPU oracle of the TensorGRaD optimizer step (test infrastructure only).

This package is the reference that the CUDA library is checked against. It is
plain C++ in fp64 (``tgd_oracle.cpp``) behind a thin ctypes wrapper. Only the
test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it; the product path never does, and this package
imports nothing from the product package.

What each function follows is cited in ``tgd_oracle.cpp``. Pins that tie the
oracle to facts the pages and mathematics fix live in ``tests/test_oracle_*``.
"""

from __future__ import annotations

import ctypes as C
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tgd_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle_tgd.so")
_lock = threading.Lock()
_lib = None

# dtype codes of the oracle (its own numbering; the same names as the library)
DTYPES = {"r32": 0, "c64": 1, "c32h": 2, "r16": 3}


def build(force: bool = False) -> str:
    """Compile the oracle shared library in-tree (g++, no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
               "-ffp-contract=off", "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            # TGD_ORACLE_LIB selects a prebuilt copy (the planted-mistake test
            # compiles mutated copies of the oracle and points here).
            path = os.environ.get("TGD_ORACLE_LIB") or build()
            L = C.CDLL(path)
            i64, u64, i32, dbl, vp = C.c_int64, C.c_uint64, C.c_int, C.c_double, C.c_void_p
            L.orc_create.restype = vp
            L.orc_create.argtypes = [i32, vp, vp, dbl, i64, dbl, dbl, dbl, dbl, dbl, i32, i32,
                                     i32, u64, dbl, i32, i32, i32]
            L.orc_destroy.argtypes = [vp]
            L.orc_set_order.argtypes = [vp, i32]
            L.orc_set_basis.argtypes = [vp, i32]
            L.orc_refresh.argtypes = [vp, vp]
            L.orc_step.argtypes = [vp, vp, vp, i64, vp]
            L.orc_info.argtypes = [vp, vp]
            L.orc_set_counters.argtypes = [vp, i64, i64, i32]
            L.orc_get_omega.argtypes = [vp, vp]
            L.orc_set_omega.argtypes = [vp, vp]
            L.orc_get_omega_val.argtypes = [vp, vp]
            L.orc_get_U.argtypes = [vp, i32, vp]
            L.orc_set_U.argtypes = [vp, i32, vp]
            L.orc_get_eigvals.argtypes = [vp, i32, vp]
            L.orc_get_eigvals.restype = i64
            L.orc_get_moment.argtypes = [vp, i32, vp]
            L.orc_set_moment.argtypes = [vp, i32, vp]
            L.orc_f64_to_f16.argtypes = [vp, vp, i64]
            L.orc_f16_to_f64.argtypes = [vp, vp, i64]
            L.orc_mag_keys.argtypes = [vp, i32, i64, vp]
            L.orc_topk.argtypes = [vp, i32, i64, i64, vp]
            L.orc_splitmix64_mix.argtypes = [u64]
            L.orc_splitmix64_mix.restype = u64
            L.orc_random_key.argtypes = [u64, u64, u64]
            L.orc_random_key.restype = u64
            L.orc_random_omega.argtypes = [u64, u64, i64, i64, vp]
            L.orc_mode_product.argtypes = [vp, i32, vp, i32, vp, i64, i64, i32, vp]
            L.orc_mode_gram.argtypes = [vp, i32, vp, i32, vp]
            L.orc_eigh.argtypes = [vp, i64, vp, vp]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ------------------------------------------------------------ pure functions
def f64_to_f16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f64_to_f16(_p(x), _p(out), x.size)
    return out


def f16_bits_to_f64(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    out = np.empty(b.shape, np.float64)
    lib().orc_f16_to_f64(_p(b), _p(out), b.size)
    return out


def _raw(g: np.ndarray, dtype: str) -> np.ndarray:
    """Raw storage array of a gradient buffer: float32 / uint16 views."""
    g = np.ascontiguousarray(g)
    if dtype == "r32":
        assert g.dtype == np.float32
    elif dtype == "c64":
        assert g.dtype in (np.complex64, np.float32)
    elif dtype in ("c32h", "r16"):
        assert g.dtype in (np.uint16, np.float16)
    return g


def mag_keys(g: np.ndarray, dtype: str) -> np.ndarray:
    g = _raw(g, dtype)
    n = g.size if dtype in ("r32", "r16") else g.size // (2 if g.dtype != np.complex64 else 1)
    out = np.empty(n, np.uint32)
    lib().orc_mag_keys(_p(g), DTYPES[dtype], n, _p(out))
    return out


def n_elems(g: np.ndarray, dtype: str) -> int:
    if dtype in ("r32", "r16"):
        return g.size
    return g.size if g.dtype == np.complex64 else g.size // 2


def topk(g: np.ndarray, dtype: str, k: int) -> np.ndarray:
    g = _raw(g, dtype)
    n = n_elems(g, dtype)
    out = np.empty(max(k, 0), np.int64)
    lib().orc_topk(_p(g), DTYPES[dtype], n, k, _p(out) if k > 0 else None)
    return out


def splitmix64_mix(z: int) -> int:
    return int(lib().orc_splitmix64_mix(z))


def random_key(seed: int, ordinal: int, i: int) -> int:
    return int(lib().orc_random_key(seed, ordinal, i))


def random_omega(seed: int, ordinal: int, n: int, k: int) -> np.ndarray:
    out = np.empty(max(k, 0), np.int64)
    lib().orc_random_omega(seed, ordinal, n, k, _p(out) if k > 0 else None)
    return out


def mode_product(x: np.ndarray, n: int, U: np.ndarray, proj: bool) -> np.ndarray:
    """proj: x x_n U^H (U is I_n x r_n); else x x_n U. Complex128 in and out."""
    x = np.ascontiguousarray(x, np.complex128)
    U = np.ascontiguousarray(U, np.complex128)
    In, rn = U.shape
    dims = np.array(x.shape, np.int64)
    out_shape = list(x.shape)
    out_shape[n] = rn if proj else In
    assert x.shape[n] == (In if proj else rn)
    y = np.empty(out_shape, np.complex128)
    lib().orc_mode_product(_p(x), x.ndim, _p(dims), n, _p(U), In, rn, 1 if proj else 0, _p(y))
    return y


def mode_gram(x: np.ndarray, n: int) -> np.ndarray:
    x = np.ascontiguousarray(x, np.complex128)
    dims = np.array(x.shape, np.int64)
    out = np.empty((x.shape[n], x.shape[n]), np.complex128)
    lib().orc_mode_gram(_p(x), x.ndim, _p(dims), n, _p(out))
    return out


def eigh(A: np.ndarray):
    """Descending eigenvalues and phase-canonical eigenvectors (columns)."""
    A = np.ascontiguousarray(A, np.complex128)
    n = A.shape[0]
    w = np.empty(n, np.float64)
    V = np.empty((n, n), np.complex128)
    lib().orc_eigh(_p(A), n, _p(w), _p(V))
    return w, V


# ----------------------------------------------------------------- optimizer
class Oracle:
    """The whole optimizer state machine (create / refresh / step)."""

    def __init__(self, shape, ranks, sparse_ratio, T, lr=1e-3, betas=(0.9, 0.999), eps=1e-8,
                 wd=0.0, grad_dtype="c64", weight_dtype=None, omega_mode=0, seed=0,
                 sparse_scale=1.0, complex_adam=0, moments_on_refresh=0, auto_refresh=1,
                 order=0, basis=0):
        """order: 0 extracts the sparse part first (the method), 1 the
        low-rank part first (the ablated order). basis: 0 HOSVD factors (the
        method), 1 DCT columns chosen by their alignment with the Gram."""
        weight_dtype = weight_dtype or grad_dtype
        self.shape = tuple(int(s) for s in shape)
        self.ranks = tuple(int(r) for r in ranks)
        self.grad_dtype, self.weight_dtype = grad_dtype, weight_dtype
        sh = np.array(self.shape, np.int64)
        rk = np.array(self.ranks, np.int64)
        self._h = lib().orc_create(len(shape), _p(sh), _p(rk), float(sparse_ratio), int(T),
                                   lr, betas[0], betas[1], eps, wd, DTYPES[grad_dtype],
                                   DTYPES[weight_dtype], omega_mode, seed, sparse_scale,
                                   complex_adam, moments_on_refresh, auto_refresh)
        if not self._h:
            raise ValueError("oracle rejected the configuration")
        if order and lib().orc_set_order(self._h, int(order)) != 0:
            raise ValueError("unknown decomposition order")
        if basis and lib().orc_set_basis(self._h, int(basis)) != 0:
            raise ValueError("unknown factor basis")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            lib().orc_destroy(h)
            self._h = None

    @property
    def info(self):
        a = np.zeros(9, np.int64)
        lib().orc_info(self._h, _p(a))
        keys = ["N", "k", "ncore", "nslabs", "t", "refreshes", "has_subspace", "mcomp", "vcomp"]
        return dict(zip(keys, (int(v) for v in a)))

    def refresh(self, grad: np.ndarray):
        lib().orc_refresh(self._h, _p(np.ascontiguousarray(grad)))

    def step(self, grad: np.ndarray, weight: np.ndarray, slabs=None) -> int:
        """Updates `weight` (storage dtype array) in place; returns status."""
        assert weight.flags["C_CONTIGUOUS"]
        if slabs is None:
            return lib().orc_step(self._h, _p(np.ascontiguousarray(grad)), _p(weight), 0, None)
        sl = np.ascontiguousarray(slabs, np.int64)
        return lib().orc_step(self._h, _p(np.ascontiguousarray(grad)), _p(weight), sl.size, _p(sl))

    # -- state
    def set_counters(self, t, refreshes, has_subspace=True):
        lib().orc_set_counters(self._h, t, refreshes, 1 if has_subspace else 0)

    @property
    def omega(self):
        out = np.empty(self.info["k"], np.int64)
        lib().orc_get_omega(self._h, _p(out))
        return out

    @omega.setter
    def omega(self, v):
        v = np.ascontiguousarray(v, np.int64)
        assert v.size == self.info["k"]
        lib().orc_set_omega(self._h, _p(v))

    def omega_values(self):
        out = np.empty((self.info["k"], 2), np.float64)
        lib().orc_get_omega_val(self._h, _p(out))
        return out[:, 0] + 1j * out[:, 1]

    def get_U(self, n) -> np.ndarray:
        """U_n as complex64 (I_n x r_n), as stored (fp32)."""
        I, r = self.shape[n], self.ranks[n]
        out = np.empty((I, r, 2), np.float32)
        lib().orc_get_U(self._h, n, _p(out))
        return out[..., 0] + 1j * out[..., 1]

    def set_U(self, n, U):
        U = np.asarray(U)
        a = np.ascontiguousarray(np.stack([U.real, U.imag], -1).astype(np.float32))
        lib().orc_set_U(self._h, n, _p(a))

    def eigvals(self, n):
        out = np.empty(self.shape[n], np.float64)
        c = lib().orc_get_eigvals(self._h, n, _p(out))
        return out[:c]

    _MOM = {"core_m": 0, "core_v": 1, "sparse_m": 2, "sparse_v": 3}

    def _msize(self, which):
        i = self.info
        n = i["ncore"] if which.startswith("core") else i["k"]
        return n * (i["mcomp"] if which.endswith("_m") else i["vcomp"])

    def get_moment(self, which) -> np.ndarray:
        out = np.empty(self._msize(which), np.float32)
        lib().orc_get_moment(self._h, self._MOM[which], _p(out))
        return out

    def set_moment(self, which, v):
        v = np.ascontiguousarray(v, np.float32).reshape(-1)
        assert v.size == self._msize(which)
        lib().orc_set_moment(self._h, self._MOM[which], _p(v))


def state_memory(shape, ranks, sparse_ratio, dtype="c64", complex_adam=0) -> dict:
    """Optimizer-state bytes of TensorGRaD for one tensor, and AdamW's.

    Low-rank branch: the review's appended paper text counts the tensor
    low-rank state as the Tucker core (prod r_n entries) plus one factor of
    I_n x r_n entries per mode (its equation (10), r_max^4 + 2 r_max N +
    2 r_max M for an N x N x M x M weight at rank r_max in every mode); a mode
    kept at full rank is the identity and stores nothing. Sparse branch (the
    nullthought summary, section 3): the COO index of each entry of Omega
    (int64) and the Adam moments of its value. Moments are FP32: m complex
    (8 bytes) or real (4); v real (4), or two reals (8) under the view-as-real
    complex Adam. AdamW keeps m and v for every element.
    """
    cplx = dtype in ("c64", "c32h")
    N = 1
    for I in shape:
        N *= int(I)
    core = 1
    for r in ranks:
        core *= int(r)
    factors = sum(int(I) * int(r) for I, r in zip(shape, ranks) if r < I)
    k = math.floor(sparse_ratio * N)
    m_b = 8 if cplx else 4
    v_b = 8 if (cplx and complex_adam) else 4
    u_b = 8 if cplx else 4
    out = {
        "N": N, "k": k, "core_elems": core, "factor_elems": factors,
        "adamw_bytes": N * (m_b + v_b),
        "core_bytes": core * (m_b + v_b),
        "factor_bytes": factors * u_b,
        "sparse_bytes": k * (8 + m_b + v_b),
    }
    out["total_bytes"] = out["core_bytes"] + out["factor_bytes"] + out["sparse_bytes"]
    return out

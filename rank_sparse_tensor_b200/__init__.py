"""TensorGRaD optimizer step on NVIDIA B200 (sm_100a), over a C ABI.

    opt = TensorGRaD(shape, ranks, sparse_ratio=0.05, T=100, lr=1e-3,
                     grad_dtype="c32h", weight_dtype="c32h")
    opt.step(grad, weight)          # torch CUDA tensors, weight updated in place

Gradients and weights are storage tensors: float32 ("r32"), complex64 ("c64"),
float16 with a trailing (re, im) axis ("c32h") or float16 ("r16"). The work
runs in libtgd.so on the current CUDA stream; this module only passes
pointers and sizes.
"""

from __future__ import annotations

import ctypes as C
import math
from typing import Optional, Sequence

import numpy as np

from . import native
from .native import TgdError, check, lib

__all__ = ["TensorGRaD", "TgdError", "state_memory", "topk_select", "topk_select_static"]


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


class _DeviceMemory:
    """A float32 device buffer described for torch.as_tensor (no copy)."""

    def __init__(self, ptr: int, count: int):
        self.__cuda_array_interface__ = {"shape": (count,), "typestr": "<f4",
                                         "data": (ptr, False), "version": 2}


def _device_view(ptr: int, count: int, dtype):
    import torch
    assert dtype == torch.float32
    return torch.as_tensor(_DeviceMemory(ptr, count), device="cuda")


def _check_tensor(t, dtype: str, n: int, what: str):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{what} must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if t.numel() * t.element_size() != n * native.ELEM_BYTES[dtype]:
        raise ValueError(f"{what} has {t.numel() * t.element_size()} bytes, expected "
                         f"{n * native.ELEM_BYTES[dtype]} for {n} elements of {dtype}")
    if t.data_ptr() % 16:
        raise ValueError(f"{what} must be 16-byte aligned")


class TensorGRaD:
    """One tensor's TensorGRaD optimizer state (a tgd_handle)."""

    def __init__(self, shape: Sequence[int], ranks: Sequence[int], sparse_ratio: float, T: int,
                 lr: float = 1e-3, betas=(0.9, 0.999), eps: float = 1e-8, wd: float = 0.0,
                 grad_dtype: str = "c64", weight_dtype: Optional[str] = None,
                 omega_mode: int = 0, seed: int = 0, sparse_scale: float = 1.0,
                 complex_adam: int = 0, moments_on_refresh: int = 0, auto_refresh: int = 1,
                 path: str = "auto", sm_budget: int = 0, order: int = 0, basis: int = 0,
                 wait_limit_ms: int = 0, test_stall: int = 0, sparse_k: int = -1,
                 mode0_total: int = 0):
        weight_dtype = weight_dtype or grad_dtype
        self.shape = tuple(int(s) for s in shape)
        self.ranks = tuple(int(r) for r in ranks)
        self.grad_dtype, self.weight_dtype = grad_dtype, weight_dtype
        self.N = math.prod(self.shape)
        opt = native.Options()
        lib().tgd_default_options(C.byref(opt))
        opt.omega_mode, opt.seed, opt.sparse_scale = omega_mode, seed, sparse_scale
        opt.complex_adam, opt.moments_on_refresh = complex_adam, moments_on_refresh
        opt.auto_refresh, opt.path = auto_refresh, native.PATHS[path]
        opt.sm_budget = sm_budget
        opt.order = order
        opt.basis = basis
        opt.wait_limit_ms = wait_limit_ms
        opt.test_stall = test_stall
        opt.sparse_k = sparse_k
        opt.mode0_total = mode0_total
        sh = (C.c_int64 * len(self.shape))(*self.shape)
        rk = (C.c_int64 * len(self.ranks))(*self.ranks)
        h = C.c_void_p()
        st = lib().tgd_create(C.byref(h), len(self.shape), sh, rk, float(sparse_ratio), int(T),
                              lr, betas[0], betas[1], eps, wd, native.DTYPES[grad_dtype],
                              native.DTYPES[weight_dtype], C.byref(opt))
        check(st)
        self._h = h

    # ------------------------------------------------------------ lifecycle
    def close(self):
        if getattr(self, "_h", None):
            lib().tgd_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------ the step
    def step(self, grad, weight, stream=None):
        _check_tensor(grad, self.grad_dtype, self.N, "grad")
        _check_tensor(weight, self.weight_dtype, self.N, "weight")
        check(lib().tgd_step(self._h, grad.data_ptr(), weight.data_ptr(), _stream_ptr(stream)), self._h)

    def refresh(self, grad, stream=None):
        _check_tensor(grad, self.grad_dtype, self.N, "grad")
        check(lib().tgd_refresh(self._h, grad.data_ptr(), _stream_ptr(stream)), self._h)

    # -------------------------------------------- the step in two halves
    def step_begin(self, grad, stream=None):
        """Sparse AdamW and the projection into the core buffer."""
        _check_tensor(grad, self.grad_dtype, self.N, "grad")
        check(lib().tgd_step_begin(self._h, grad.data_ptr(), _stream_ptr(stream)), self._h)

    def core_buffer(self):
        """(device address, float count) of the core between the halves."""
        ptr, cnt = C.c_void_p(), C.c_int64()
        check(lib().tgd_core_buffer(self._h, C.byref(ptr), C.byref(cnt)), self._h)
        return int(ptr.value or 0), int(cnt.value)

    def core_tensor(self):
        """The core buffer as a torch float32 tensor viewing the device
        memory (valid until step_end), for summing partial cores."""
        import torch
        ptr, cnt = self.core_buffer()
        return _device_view(ptr, cnt, torch.float32)

    def step_end(self, weight, stream=None):
        """Core AdamW on the (summed) core, expansion and weight update."""
        _check_tensor(weight, self.weight_dtype, self.N, "weight")
        check(lib().tgd_step_end(self._h, weight.data_ptr(), _stream_ptr(stream)), self._h)

    def step_host(self, grad_host: np.ndarray, weight_host: np.ndarray, stream=None):
        """Host buffers in, host weights out (copies inside the call)."""
        for a, dt, what in ((grad_host, self.grad_dtype, "grad"), (weight_host, self.weight_dtype, "weight")):
            if not a.flags["C_CONTIGUOUS"] or a.nbytes != self.N * native.ELEM_BYTES[dt]:
                raise ValueError(f"{what}: expected a contiguous host array of {self.N} {dt} elements")
        check(lib().tgd_step_host(self._h, grad_host.ctypes.data, weight_host.ctypes.data,
                                  _stream_ptr(stream)), self._h)

    def sync(self, stream=None):
        check(lib().tgd_sync(self._h, _stream_ptr(stream)), self._h)

    # ------------------------------------------------------------ timing
    def profile(self, enable: bool):
        """Start (and clear) or stop per-kernel CUDA-event timing."""
        check(lib().tgd_profile(self._h, 1 if enable else 0), self._h)

    def profile_read(self) -> dict:
        """{kernel name: (launches, total ms)} recorded since profile(True)."""
        cap = 64
        arr = (native.KernelTime * cap)()
        cnt = C.c_int()
        check(lib().tgd_profile_read(self._h, arr, cap, C.byref(cnt)), self._h)
        return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms))
                for i in range(min(cnt.value, cap))}

    # ------------------------------------------------------------ state
    @property
    def info(self) -> dict:
        inf = native.Info()
        check(lib().tgd_query(self._h, C.byref(inf)), self._h)
        d = inf.ndim
        return {"ndim": d, "shape": tuple(inf.shape[:d]), "ranks": tuple(inf.ranks[:d]),
                "N": inf.N, "k": inf.k, "ncore": inf.ncore, "core_m_len": inf.core_m_len,
                "core_v_len": inf.core_v_len, "sparse_m_len": inf.sparse_m_len,
                "sparse_v_len": inf.sparse_v_len,
                "path": {1: "generic", 2: "tcgen05"}.get(inf.path, str(inf.path)),
                "device_bytes": inf.device_bytes, "t": inf.t, "refreshes": inf.refreshes,
                "has_subspace": bool(inf.has_subspace)}

    def get_state(self, stream=None) -> dict:
        i = self.info
        cplx = self.grad_dtype in ("c64", "c32h")
        out = {
            "omega": np.zeros(i["k"], np.int64),
            "omega_val": np.zeros(i["k"] * (2 if cplx else 1), np.float32),
            "U": [np.zeros((I, r, 2), np.float32) for I, r in zip(self.shape, self.ranks)],
            "core_m": np.zeros(i["core_m_len"], np.float32),
            "core_v": np.zeros(i["core_v_len"], np.float32),
            "sparse_m": np.zeros(i["sparse_m_len"], np.float32),
            "sparse_v": np.zeros(i["sparse_v_len"], np.float32),
        }
        v = native.StateView()
        v.omega, v.omega_val = out["omega"].ctypes.data, out["omega_val"].ctypes.data
        for n, u in enumerate(out["U"]):
            v.U[n] = u.ctypes.data
        for key in ("core_m", "core_v", "sparse_m", "sparse_v"):
            setattr(v, key, out[key].ctypes.data)
        check(lib().tgd_get_state(self._h, C.byref(v), _stream_ptr(stream)), self._h)
        out["t"], out["refreshes"], out["has_subspace"] = v.t, v.refreshes, bool(v.has_subspace)
        out["U"] = [u[..., 0] + 1j * u[..., 1] for u in out["U"]]
        return out

    def set_state(self, state: dict, stream=None):
        """Replaces the parts present in `state` (same keys as get_state)."""
        i = self.info
        keep = []

        def arr(x, dtype, size=None):
            a = np.ascontiguousarray(x, dtype).reshape(-1)
            if size is not None and a.size != size:
                raise ValueError(f"expected {size} values, got {a.size}")
            keep.append(a)
            return a.ctypes.data

        v = native.StateView()
        v.t = int(state.get("t", i["t"]))
        v.refreshes = int(state.get("refreshes", i["refreshes"]))
        v.has_subspace = int(bool(state.get("has_subspace", True)))
        if "omega" in state:
            v.omega = arr(state["omega"], np.int64, i["k"])
        if "omega_val" in state:
            v.omega_val = arr(state["omega_val"], np.float32)
        if "U" in state:
            for n, u in enumerate(state["U"]):
                if u is None:
                    continue
                u = np.asarray(u)
                v.U[n] = arr(np.stack([u.real, u.imag], -1), np.float32,
                             self.shape[n] * self.ranks[n] * 2)
        for key in ("core_m", "core_v", "sparse_m", "sparse_v"):
            if key in state:
                setattr(v, key, arr(state[key], np.float32, i[key + "_len"]))
        check(lib().tgd_set_state(self._h, C.byref(v), _stream_ptr(stream)), self._h)


def state_memory(shape: Sequence[int], ranks: Sequence[int], sparse_ratio: float,
                 grad_dtype: str = "c64", complex_adam: int = 0) -> dict:
    """Optimizer-state bytes of the method for one tensor next to AdamW's
    (tgd_state_memory; host arithmetic, no device needed). Adds "ratio" =
    total_bytes / adamw_bytes."""
    d = len(shape)
    if len(ranks) != d:
        raise ValueError("shape and ranks differ in length")
    sh = (C.c_int64 * max(d, 1))(*shape)
    rk = (C.c_int64 * max(d, 1))(*ranks)
    m = native.Memory()
    check(lib().tgd_state_memory(d, C.cast(sh, C.c_void_p), C.cast(rk, C.c_void_p),
                                 float(sparse_ratio), native.DTYPES[grad_dtype], int(complex_adam),
                                 C.byref(m)))
    out = {name: int(getattr(m, name)) for name, _ in native.Memory._fields_}
    out["ratio"] = out["total_bytes"] / out["adamw_bytes"]
    return out


def topk_select(grad, dtype: str, k: int, stream=None):
    """Standalone top-k COO selection: (omega int64[k], values float32[k(,2)])."""
    import torch
    n = grad.numel() * grad.element_size() // native.ELEM_BYTES[dtype]
    _check_tensor(grad, dtype, n, "grad")
    cplx = dtype in ("c64", "c32h")
    omega = torch.empty(max(k, 1), dtype=torch.int64, device=grad.device)
    vals = torch.empty(max(k, 1) * (2 if cplx else 1), dtype=torch.float32, device=grad.device)
    wsb = int(lib().tgd_topk_workspace_bytes(n))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=grad.device)
    check(lib().tgd_topk_select(grad.data_ptr(), native.DTYPES[dtype], n, k, omega.data_ptr(),
                                vals.data_ptr(), ws.data_ptr(), wsb, _stream_ptr(stream)))
    vals = vals[: k * (2 if cplx else 1)]
    return omega[:k], (vals.view(k, 2) if cplx else vals)


def topk_select_static(grad, dtype: str, k: int, stream=None):
    """The same selection as topk_select, for callers that cannot allocate
    device scratch memory: the library uses a fixed array of its own (one per
    device, n <= 2**28). Only the outputs are allocated here, by the caller's
    framework. Calls that overlap on the GPU share that array and must not
    run concurrently."""
    import torch
    n = grad.numel() * grad.element_size() // native.ELEM_BYTES[dtype]
    _check_tensor(grad, dtype, n, "grad")
    cplx = dtype in ("c64", "c32h")
    omega = torch.empty(max(k, 1), dtype=torch.int64, device=grad.device)
    vals = torch.empty(max(k, 1) * (2 if cplx else 1), dtype=torch.float32, device=grad.device)
    check(lib().tgd_topk_select_static(grad.data_ptr(), native.DTYPES[dtype], n, k, omega.data_ptr(),
                                       vals.data_ptr(), _stream_ptr(stream)))
    vals = vals[: k * (2 if cplx else 1)]
    return omega[:k], (vals.view(k, 2) if cplx else vals)

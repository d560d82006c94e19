"""GPU parity at the benchmark workloads' full sizes, in the launch
configuration the benchmark times.

Both sides get the same state (Omega from the oracle's own selection, factors
from a seeded QR of a Gaussian, non-zero moments, step count), take one
teacher-forced step, and the weights are compared: element by element where
the oracle can afford the whole tensor, on sampled slabs (the oracle's slab
selection reconstructs only those) for the 545M-element spectral tensor.
Omega itself is compared bit for bit with the device refresh at full size.
"""

import math

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


def _factors(shape, ranks, cplx, seed):
    """Seeded orthonormal factors (QR of a Gaussian); identity for full rank."""
    rng = np.random.default_rng(seed)
    out = []
    for I, r in zip(shape, ranks):
        if r == I:
            out.append(np.eye(I))
            continue
        a = rng.standard_normal((I, r))
        if cplx:
            a = a + 1j * rng.standard_normal((I, r))
        q, _ = np.linalg.qr(a)
        out.append(q)
    return out


def _teacher_forced(lib, orc, wl_name, slabs=None, seed=5):
    from rank_sparse_tensor_b200.synth import WORKLOADS, GradientStream, weights
    wl = WORKLOADS[wl_name]
    shape, ranks, dt, wdt = wl.shape, wl.ranks, wl.dtype, wl.weight_dtype
    cplx = dt in ("c64", "c32h")
    gs = GradientStream(shape, wl.gen_ranks, dt, seed, outlier_frac=wl.outlier_frac,
                        outlier_scale=wl.outlier_scale, device="cuda")
    g_dev = gs.next()
    w_dev = weights(shape, wdt, seed, device="cuda")
    g = to_np(g_dev)
    w0 = to_np(w_dev)
    k = math.floor(wl.sparse_ratio * math.prod(shape))
    omega = orc.topk(g, dt, k)
    U = _factors(shape, ranks, cplx, seed + 1)
    o = orc.Oracle(shape, ranks, wl.sparse_ratio, 0, wl.lr, wl.betas, wl.eps, wl.wd, dt, wdt,
                   auto_refresh=0)
    gpu = lib.TensorGRaD(shape, ranks, wl.sparse_ratio, 0, wl.lr, wl.betas, wl.eps, wl.wd, dt,
                         wdt, auto_refresh=0)
    mom = random_moments(np.random.default_rng(seed + 2), gpu.info, cplx)
    o.omega = omega
    for n in range(len(shape)):
        o.set_U(n, U[n])
    for key, v in mom.items():
        o.set_moment(key, v)
    o.set_counters(4, 1, True)
    gpu.set_state(dict(mom, omega=omega, U=U, t=4, refreshes=1, has_subspace=True))
    gpu.step(g_dev, w_dev)
    gpu.sync()
    w_gpu = to_np(w_dev)
    w_ref = w0.copy()
    assert o.step(g, w_ref, slabs=slabs) == 0
    st = gpu.get_state()
    assert st["t"] == 5
    return wl, gpu, w_gpu, w_ref, w0


def test_spectral_545m_sampled_slabs(lib, orc):
    """The benchmark's headline tensor (256,256,128,65) complex fp16: weights
    on 24 sampled slabs (first, last, a spread between) within 2e-3."""
    n_slabs = 256 * 256
    rng = np.random.default_rng(11)
    sel = np.unique(np.concatenate([[0, 1, n_slabs - 1], rng.choice(n_slabs, 21, replace=False)]))
    wl, gpu, w_gpu, w_ref, w0 = _teacher_forced(lib, orc, "spectral_c32h_256x256x128x65",
                                                 slabs=sel)
    assert gpu.info["path"] == "tcgen05"
    flat_g = w_gpu.reshape(n_slabs, 128, 65, 2)
    flat_r = w_ref.reshape(n_slabs, 128, 65, 2)
    err = rel_err(flat_g[sel], flat_r[sel], "c32h")
    assert err <= TOL["c32h"], err
    # the slabs the oracle skipped are still its inputs; the GPU updated them
    assert not np.array_equal(flat_g[2], w0.reshape(n_slabs, 128, 65, 2)[2])


def test_fno4_tensor_full(lib, orc):
    """One (128,128,64,33) complex fp16 tensor of the 4-tensor workload, every
    element compared."""
    wl, gpu, w_gpu, w_ref, _ = _teacher_forced(lib, orc, "fno4_c32h_128x128x64x33")
    assert gpu.info["path"] == "tcgen05"
    err = rel_err(w_gpu, w_ref, "c32h")
    assert err <= TOL["c32h"], err


def test_refresh5_full_step(lib, orc):
    """The 5-way complex fp32 tensor (64,64,32,32,17), every element."""
    wl, gpu, w_gpu, w_ref, _ = _teacher_forced(lib, orc, "refresh_c64_64x64x32x32x17")
    err = rel_err(w_gpu, w_ref, "c64")
    assert err <= TOL["c64"], err


@pytest.mark.parametrize("wl_name,omega_mode", [
    ("spectral_c32h_256x256x128x65", 0),
    ("refresh_c64_64x64x32x32x17", 0),
    ("refresh_c64_64x64x32x32x17", 1),
])
def test_full_size_omega_bit_exact(lib, orc, wl_name, omega_mode):
    """Omega of the device refresh against the oracle's selection at full
    size: top-k by magnitude (ties to the lower index) and the seeded random
    variant."""
    from rank_sparse_tensor_b200.synth import WORKLOADS, GradientStream
    wl = WORKLOADS[wl_name]
    gs = GradientStream(wl.shape, wl.gen_ranks, wl.dtype, 3, outlier_frac=wl.outlier_frac,
                        outlier_scale=wl.outlier_scale, device="cuda")
    g_dev = gs.next()
    N = math.prod(wl.shape)
    k = math.floor(wl.sparse_ratio * N)
    gpu = lib.TensorGRaD(wl.shape, wl.ranks, wl.sparse_ratio, 0, grad_dtype=wl.dtype,
                         weight_dtype=wl.weight_dtype, omega_mode=omega_mode, seed=9,
                         auto_refresh=0)
    gpu.refresh(g_dev)
    om = gpu.get_state()["omega"]
    ref = orc.topk(to_np(g_dev), wl.dtype, k) if omega_mode == 0 else orc.random_omega(9, 0, N, k)
    assert np.array_equal(om, ref)


def test_fno4_four_tensors_side_by_side(lib, orc):
    """The 4-tensor workload as the benchmark runs it: four (128,128,64,33)
    complex fp16 tensors stepped at once, each on its own stream with a
    quarter of the SMs (sm_budget), every tensor's weights compared with the
    oracle's teacher-forced step element by element."""
    import math
    from rank_sparse_tensor_b200.synth import WORKLOADS, GradientStream, weights
    wl = WORKLOADS["fno4_c32h_128x128x64x33"]
    shape, ranks = wl.shape, wl.ranks
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    budget = max(1, n_sms // 4)
    streams = [torch.cuda.Stream() for _ in range(4)]
    runs = []
    for j in range(4):
        gs = GradientStream(shape, wl.gen_ranks, wl.dtype, 40 + j, outlier_frac=wl.outlier_frac,
                            outlier_scale=wl.outlier_scale, device="cuda")
        g_dev = gs.next()
        w_dev = weights(shape, wl.weight_dtype, 40 + j, device="cuda")
        g, w0 = to_np(g_dev), to_np(w_dev)
        k = math.floor(wl.sparse_ratio * math.prod(shape))
        omega = orc.topk(g, wl.dtype, k)
        U = _factors(shape, ranks, True, 50 + j)
        gpu = lib.TensorGRaD(shape, ranks, wl.sparse_ratio, 0, wl.lr, wl.betas, wl.eps, wl.wd,
                             wl.dtype, wl.weight_dtype, auto_refresh=0, sm_budget=budget)
        assert gpu.info["path"] == "tcgen05"
        mom = random_moments(np.random.default_rng(60 + j), gpu.info, True)
        gpu.set_state(dict(mom, omega=omega, U=U, t=4, refreshes=1, has_subspace=True))
        runs.append((gpu, g_dev, w_dev, g, w0, omega, U, mom))
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()
    fork = torch.cuda.Event()
    fork.record(main)
    for (gpu, g_dev, w_dev, *_), st in zip(runs, streams):
        st.wait_event(fork)
        with torch.cuda.stream(st):
            gpu.step(g_dev, w_dev)
    torch.cuda.synchronize()
    for gpu, g_dev, w_dev, g, w0, omega, U, mom in runs:
        gpu.sync()
        o = orc.Oracle(shape, ranks, wl.sparse_ratio, 0, wl.lr, wl.betas, wl.eps, wl.wd, wl.dtype,
                       wl.weight_dtype, auto_refresh=0)
        o.omega = omega
        for n in range(len(shape)):
            o.set_U(n, U[n])
        for key, v in mom.items():
            o.set_moment(key, v)
        o.set_counters(4, 1, True)
        w_ref = w0.copy()
        assert o.step(g, w_ref) == 0
        assert rel_err(to_np(w_dev), w_ref, wl.dtype) <= TOL[wl.dtype]

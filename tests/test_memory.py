"""Optimizer-state memory accounting (host arithmetic, no device).

The oracle's count is pinned to the review's tensor low-rank parameter count
(the appended paper text, equation (10)) and to the headline spectral tensor
worked out by hand from the definitions; the library's tgd_state_memory must
then equal the oracle on every seeded case, integer for integer.
"""

import math

import numpy as np
import pytest

import oracle


EQ10_CASES = [(64, 17, 4), (128, 33, 8), (128, 64, 32), (256, 65, 16)]


def pin_equation_10(fn):
    """Core plus factors of an N x N x M x M weight at rank r in every mode:
    r^4 + 2 r N + 2 r M entries."""
    for N, M, r in EQ10_CASES:
        m = fn((N, N, M, M), (r, r, r, r), 0.0, "c64")
        assert m["core_elems"] + m["factor_elems"] == r ** 4 + 2 * r * N + 2 * r * M


def pin_headline_by_hand(fn):
    """(256,256,128,65) complex fp16, ranks (64,64,32,16), rho 0.05:
    N = 545,259,520; k = floor(0.05 N) = 27,262,976;
    core 64*64*32*16 = 2,097,152 entries x (8 + 4) B = 25,165,824 B;
    factors 2*256*64 + 128*32 + 65*16 = 37,904 entries x 8 B = 303,232 B;
    sparse 27,262,976 x (8 + 8 + 4) B = 545,259,520 B;
    AdamW 545,259,520 x 12 B = 6,543,114,240 B."""
    m = fn((256, 256, 128, 65), (64, 64, 32, 16), 0.05, "c32h")
    assert m["N"] == 545_259_520 and m["k"] == 27_262_976
    assert m["core_bytes"] == 25_165_824
    assert m["factor_bytes"] == 303_232
    assert m["sparse_bytes"] == 545_259_520
    assert m["total_bytes"] == 570_728_576
    assert m["adamw_bytes"] == 6_543_114_240


def pin_special_cases(fn):
    # no sparse part at rho = 0
    m = fn((16, 12, 8), (4, 3, 2), 0.0, "r32")
    assert m["k"] == 0 and m["sparse_bytes"] == 0
    # k = floor(rho N): 0.1 * 21 = 2.1 -> 2
    assert fn((7, 3), (7, 3), 0.1, "r32")["k"] == 2
    # every mode at full rank: the core is the whole tensor and no factor is kept
    m = fn((16, 12, 8), (16, 12, 8), 0.0, "c64")
    assert m["factor_elems"] == 0 and m["core_bytes"] == m["adamw_bytes"]
    # real tensors: 4-byte m and v and factors
    m = fn((10, 6), (2, 3), 0.5, "r16")
    assert m["core_bytes"] == 6 * 8 and m["factor_bytes"] == (20 + 18) * 4
    assert m["sparse_bytes"] == 30 * (8 + 8) and m["adamw_bytes"] == 60 * 8
    # view-as-real complex Adam keeps two second moments
    a = fn((10, 6), (2, 3), 0.5, "c64", complex_adam=0)
    b = fn((10, 6), (2, 3), 0.5, "c64", complex_adam=1)
    assert b["adamw_bytes"] - a["adamw_bytes"] == 60 * 4
    assert b["sparse_bytes"] - a["sparse_bytes"] == 30 * 4


PINS = [pin_equation_10, pin_headline_by_hand, pin_special_cases]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pins(pin):
    pin(oracle.state_memory)


# (name, original text, mutated text): plausible slips in the oracle's count
MUTANTS = [
    ("factor_for_full_rank_mode", "if r < I)", "if r <= I)"),
    ("complex_m_as_real", "m_b = 8 if cplx else 4", "m_b = 4"),
    ("index_4_bytes", "k * (8 + m_b + v_b)", "k * (4 + m_b + v_b)"),
    ("v_doubled_by_default", "v_b = 8 if (cplx and complex_adam) else 4", "v_b = 8 if cplx else 4"),
    ("core_m_only", "core * (m_b + v_b)", "core * m_b"),
    ("k_rounded_up", "math.floor(sparse_ratio * N)", "math.ceil(sparse_ratio * N)"),
    ("real_factor_8_bytes", "u_b = 8 if cplx else 4", "u_b = 8"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    """A mutated copy of the oracle's count (the shipped one is untouched)
    fails at least one pin."""
    import inspect
    src = inspect.getsource(oracle.state_memory)
    assert src.count(old) == 1, name
    ns = {"math": math}
    exec(src.replace(old, new), ns)
    mutant = ns["state_memory"]
    failed = 0
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            failed += 1
    assert failed > 0, f"mutant {name} passed every pin"


def test_library_equals_oracle():
    import rank_sparse_tensor_b200 as rst
    rng = np.random.default_rng(7)
    for _ in range(300):
        d = int(rng.integers(1, 9))
        shape = [int(rng.integers(1, 300 if d <= 3 else 20)) for _ in range(d)]
        ranks = [int(rng.integers(1, I + 1)) for I in shape]
        rho = float(rng.choice([0.0, 1.0, rng.random()]))
        dt = str(rng.choice(["r32", "c64", "c32h", "r16"]))
        ca = int(rng.integers(0, 2))
        got = rst.state_memory(shape, ranks, rho, dt, ca)
        want = oracle.state_memory(shape, ranks, rho, dt, ca)
        assert {k: got[k] for k in want} == want, (shape, ranks, rho, dt, ca)
        assert got["ratio"] == pytest.approx(want["total_bytes"] / want["adamw_bytes"])


@pytest.mark.parametrize("shape,ranks,rho,dt,ca", [
    ((4, 4), (5, 4), 0.1, 1, 0),          # rank above the mode size
    ((4, 4), (0, 4), 0.1, 1, 0),          # rank 0
    ((4, 0), (4, 1), 0.1, 1, 0),          # empty mode
    ((4, 4), (2, 2), -0.1, 1, 0),         # rho below 0
    ((4, 4), (2, 2), 1.5, 1, 0),          # rho above 1
    ((4, 4), (2, 2), float("nan"), 1, 0),
    ((4, 4), (2, 2), 0.1, 7, 0),          # unknown dtype
    ((4, 4), (2, 2), 0.1, 1, 2),          # complex_adam out of range
    ((1 << 21, 1 << 21), (1 << 21, 1 << 21), 0.1, 1, 0),  # above 2^40 elements
    ((2,) * 9, (1,) * 9, 0.1, 1, 0),      # too many modes
    ((), (), 0.1, 1, 0),                  # no modes
])
def test_library_rejects_bad_arguments(shape, ranks, rho, dt, ca):
    import ctypes as C
    from rank_sparse_tensor_b200 import native
    d = len(shape)
    sh = (C.c_int64 * max(d, 1))(*shape)
    rk = (C.c_int64 * max(d, 1))(*ranks)
    out = native.Memory()
    out.total_bytes = -7
    st = native.lib().tgd_state_memory(d, C.cast(sh, C.c_void_p), C.cast(rk, C.c_void_p), rho, dt,
                                       ca, C.byref(out))
    assert st == 1  # TGD_ERR_INVALID_ARG
    assert out.total_bytes == -7  # untouched


def test_bench_reports_the_rank_total():
    """The benchmark line's optimizer_state sums the rank's tensors."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from rank_sparse_tensor_b200.synth import WORKLOADS
    wl = WORKLOADS["fno4_c32h_128x128x64x33"]
    one = oracle.state_memory(wl.shape, wl.ranks, wl.sparse_ratio, wl.dtype)
    got = bench.optimizer_state(wl, 4, 12345)
    assert got["bytes"] == 4 * one["total_bytes"] and got["adamw_bytes"] == 4 * one["adamw_bytes"]
    assert got["device_bytes"] == 12345
    assert math.isclose(got["ratio"], one["total_bytes"] / one["adamw_bytes"])

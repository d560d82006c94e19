"""The benchmark's roofline numerators, pinned to the step's byte count worked
out by hand from its definition: G read once, W read and written once,
Omega's int64 index with the sparse FP32 moments read and written, the core
moments read and written, the factors read once."""

import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from rank_sparse_tensor_b200.synth import WORKLOADS  # noqa: E402


def test_headline_step_bytes():
    """(256,256,128,65) complex fp16, ranks (64,64,32,16), rho 0.05:
    N = 545,259,520, k = 27,262,976;
    G 4N = 2,181,038,080; W 2 x 4N = 4,362,076,160;
    sparse k (8 + 2 (8 + 4)) = 872,415,232; core 2 x 2,097,152 x 12 = 50,331,648;
    factors (2*256*64 + 128*32 + 65*16) x 8 = 303,232; total 7,466,164,352
    (13.69 bytes per gradient element)."""
    a = bench.algorithmic_bytes(WORKLOADS["spectral_c32h_256x256x128x65"])
    assert a == {"grad": 2_181_038_080, "weight": 4_362_076_160, "sparse": 872_415_232,
                 "core": 50_331_648, "factors": 303_232, "total": 7_466_164_352}


def test_fno_tensor_step_bytes():
    """(128,128,64,33) complex fp16, ranks (26,26,13,7), rho 0.05:
    N = 34,603,008, k = floor(1,730,150.4) = 1,730,150;
    G 138,412,032; W 276,824,064; sparse 1,730,150 x 32 = 55,364,800;
    core 2 x 61,516 x 12 = 1,476,384; factors (2*128*26 + 64*13 + 33*7) x 8 = 61,752;
    total 472,139,032 per tensor, 1,888,556,128 for the four."""
    wl = WORKLOADS["fno4_c32h_128x128x64x33"]
    a = bench.algorithmic_bytes(wl)
    assert a["total"] == 472_139_032 and 4 * a["total"] == 1_888_556_128
    assert (a["sparse"], a["core"], a["factors"]) == (55_364_800, 1_476_384, 61_752)


def test_kernel_shares_of_the_headline():
    """The stream kernels' numerators: the projection moves G and Omega's index
    (2,181,038,080 + 8 k = 2,399,141,888), the sparse AdamW the moments
    (24 k = 654,311,424), the reconstruction W (4,362,076,160)."""
    wl = WORKLOADS["spectral_c32h_256x256x128x65"]
    assert bench.kernel_algorithmic_bytes("proj_stream", wl) == 2_399_141_888
    assert bench.kernel_algorithmic_bytes("sparse_adam", wl) == 654_311_424
    assert bench.kernel_algorithmic_bytes("recon_stream", wl) == 4_362_076_160


def test_headline_roofline_time():
    """At the measured 6,540.2 GB/s copy bandwidth the headline step cannot
    take less than 7.466 GB / 6540.2 GB/s = 1.1416 ms."""
    a = bench.algorithmic_bytes(WORKLOADS["spectral_c32h_256x256x128x65"])
    assert a["total"] / 6540.2e9 * 1e3 == pytest.approx(1.1416, abs=1e-4)

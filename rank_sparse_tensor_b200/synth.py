"""Seeded synthetic gradients and weights shaped like FNO spectral weights.

This module only draws random inputs. It holds none of the optimizer's
arithmetic (no selection, projection, Adam or update); tests feed the same
arrays to the CUDA library and to the CPU oracle.

Gradient model (a low-rank-plus-outlier tensor, as the method assumes):
    G = core x_1 Q_1 x_2 Q_2 ... x_d Q_d + outliers + noise
  * Q_n: I_n x c_n with orthonormal columns, from the QR factorisation of a
    Gaussian matrix (complex Gaussian for complex tensors). Fixed across steps
    unless ``drift`` > 0, in which case Q_n <- qr(Q_n + drift * N(0, 1)) before
    every step after the first.
  * core: c_1 x ... x c_d, N(0, 1) per element (complex: re, im ~ N(0, 1/2)),
    redrawn every step.
  * outliers: floor(p * N) positions drawn uniformly without replacement, each
    gets N(0, scale^2) added (complex: per component variance scale^2 / 2).
  * noise: dense N(0, noise^2) (complex: per component variance noise^2 / 2).
Weights: N(0, 0.02^2) per real component.

Gradients are returned as storage arrays: float32 (r32), complex64 (c64),
float16 with a trailing (re, im) axis of 2 (c32h), float16 (r16).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: tuple
    ranks: tuple            # ranks the optimizer uses
    gen_ranks: tuple        # Tucker ranks of the synthetic gradient
    dtype: str              # gradient storage dtype
    weight_dtype: str
    sparse_ratio: float
    T: int
    steps: int
    outlier_frac: float
    outlier_scale: float
    noise: float = 0.01
    drift: float = 0.0
    n_tensors: int = 1
    lr: float = 1e-3
    betas: tuple = (0.9, 0.999)
    eps: float = 1e-8
    wd: float = 0.0
    omega_modes: tuple = (0,)

    @property
    def N(self) -> int:
        return math.prod(self.shape)

    @property
    def k(self) -> int:
        return int(math.floor(self.sparse_ratio * self.N))


def ceil_ranks(shape, frac):
    return tuple(int(math.ceil(frac * s - 1e-12)) for s in shape)


# The five workloads: a tiny real tensor, one FNO spectral gradient in complex64,
# a four-layer mixed-precision FNO parameter set, one large complex fp16
# spectral tensor (the throughput workload), and a five-way refresh stress case.
WORKLOADS = {
    "tiny_r32_16x16x8x8": Workload(
        "tiny_r32_16x16x8x8", (16, 16, 8, 8), (4, 4, 2, 2), (4, 4, 2, 2), "r32", "r32",
        0.05, 5, 10, 0.01, 10.0),
    "fno_c64_64x64x32x17": Workload(
        "fno_c64_64x64x32x17", (64, 64, 32, 17), (16, 16, 8, 5), (16, 16, 8, 5), "c64", "c64",
        0.05, 50, 200, 0.02, 10.0),
    "fno4_c32h_128x128x64x33": Workload(
        "fno4_c32h_128x128x64x33", (128, 128, 64, 33), (26, 26, 13, 7), (32, 32, 16, 9),
        "c32h", "c32h", 0.05, 100, 300, 0.02, 10.0, drift=0.01, n_tensors=4),
    "spectral_c32h_256x256x128x65": Workload(
        "spectral_c32h_256x256x128x65", (256, 256, 128, 65), (64, 64, 32, 16),
        (64, 64, 32, 16), "c32h", "c32h", 0.05, 0, 50, 0.02, 10.0),
    "refresh_c64_64x64x32x32x17": Workload(
        "refresh_c64_64x64x32x32x17", (64, 64, 32, 32, 17), (16, 16, 8, 8, 5),
        (16, 16, 8, 8, 5), "c64", "c64", 0.05, 1, 20, 0.02, 10.0, omega_modes=(0, 1)),
}


def is_complex(dtype: str) -> bool:
    return dtype in ("c64", "c32h")


def _randn(shape, complex_, gen, device):
    if complex_:
        re = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        im = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        return torch.complex(re, im) * math.sqrt(0.5)
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _orthonormal(rows, cols, complex_, gen, device):
    a = _randn((rows, cols), complex_, gen, device)
    q, _ = torch.linalg.qr(a.cpu() if device != "cpu" else a)
    return q.to(device)


def to_storage(x: torch.Tensor, dtype: str) -> torch.Tensor:
    """float32/complex64 tensor -> storage layout of `dtype` (same device)."""
    if dtype == "r32":
        return x.real.float().contiguous() if x.is_complex() else x.float().contiguous()
    if dtype == "r16":
        return (x.real if x.is_complex() else x).half().contiguous()
    if dtype == "c64":
        return x.to(torch.complex64).contiguous()
    if dtype == "c32h":
        return torch.view_as_real(x.to(torch.complex64)).half().contiguous()
    raise ValueError(dtype)


class GradientStream:
    """Per-step synthetic gradients for one tensor (seeded, reproducible)."""

    def __init__(self, shape: Sequence[int], gen_ranks: Sequence[int], dtype: str, seed: int,
                 outlier_frac: float = 0.01, outlier_scale: float = 10.0, noise: float = 0.01,
                 drift: float = 0.0, device: str = "cpu"):
        self.shape = tuple(shape)
        self.gen_ranks = tuple(gen_ranks)
        self.dtype = dtype
        self.complex = is_complex(dtype)
        self.seed = seed
        self.p, self.scale, self.noise, self.drift = outlier_frac, outlier_scale, noise, drift
        self.device = device
        g = torch.Generator(device="cpu").manual_seed(seed)
        self.Q = [_orthonormal(I, c, self.complex, g, "cpu").to(device)
                  for I, c in zip(self.shape, self.gen_ranks)]
        self.t = 0

    def _gen(self, salt: int):
        g = torch.Generator(device=self.device)
        g.manual_seed((self.seed * 1_000_003 + salt * 7919 + 17) % (2 ** 63))
        return g

    def next(self) -> torch.Tensor:
        """Gradient for the next step, as a storage-dtype tensor."""
        t = self.t
        self.t += 1
        if self.drift > 0 and t > 0:
            gq = torch.Generator(device="cpu").manual_seed(self.seed * 31 + t)
            newQ = []
            for q in self.Q:
                pert = _randn(tuple(q.shape), self.complex, gq, "cpu").to(q.device)
                qq, _ = torch.linalg.qr((q + self.drift * pert).cpu())
                newQ.append(qq.to(q.device))
            self.Q = newQ
        gen = self._gen(t)
        x = _randn(self.gen_ranks, self.complex, gen, self.device)
        for n, q in enumerate(self.Q):
            q = q.to(x.dtype)
            x = torch.movedim(torch.tensordot(x, q, dims=([n], [1])), -1, n)
        x = x.reshape(-1)
        N = x.numel()
        n_out = int(math.floor(self.p * N))
        if n_out > 0:
            pos = torch.randperm(N, generator=gen, device=self.device)[:n_out]
            x[pos] += self.scale * _randn((n_out,), self.complex, gen, self.device)
        x += self.noise * _randn((N,), self.complex, gen, self.device)
        return to_storage(x.reshape(self.shape), self.dtype)


def weights(shape: Sequence[int], dtype: str, seed: int, device: str = "cpu") -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(seed + 4242)
    w = 0.02 * torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if is_complex(dtype):
        wi = 0.02 * torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
        w = torch.complex(w, wi)
    return to_storage(w, dtype)


def tucker_exact(shape, ranks, dtype: str, seed: int, device: str = "cpu"):
    """An exactly Tucker-rank tensor (no outliers, no noise) and its factors."""
    s = GradientStream(shape, ranks, dtype, seed, outlier_frac=0.0, noise=0.0, device=device)
    return s.next(), s.Q


def integer_ties(shape, dtype: str, seed: int, levels: int = 4, device: str = "cpu"):
    """Small-integer-valued gradient: magnitudes repeat, forcing ties in top-k."""
    g = torch.Generator(device=device).manual_seed(seed)
    re = torch.randint(-levels, levels + 1, tuple(shape), generator=g, device=device).float()
    if is_complex(dtype):
        im = torch.randint(-levels, levels + 1, tuple(shape), generator=g, device=device).float()
        return to_storage(torch.complex(re, im), dtype)
    return to_storage(re, dtype)

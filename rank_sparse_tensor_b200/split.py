"""One tensor split across GPUs along mode 0: the host-side plumbing.

Each rank holds a contiguous block of mode 0's rows of the gradient and the
weights. The projection's mode-0 product sums over those rows (the mode-n
product of the paper text appended to the Pith review, Appendix K), so a
block projects to a partial core and the whole core is the sum over blocks;
the core AdamW then runs replicated and the expansion, the sparse part and
the weight update stay local. This module computes the blocks, cuts the
whole tensor's state (Omega, U_0, sparse moments) into a block's share, and
runs a split step: tgd_step_begin, an all-reduce (sum) of the core buffer
over the process group, tgd_step_end. The arithmetic stays in the library.
"""

from __future__ import annotations

import math
from typing import Sequence

import numpy as np


def block_rows(I0: int, nblocks: int, block: int):
    """Rows [begin, end) of mode 0 held by `block` of `nblocks` (contiguous,
    sizes differing by at most one, the larger blocks first)."""
    if not (0 <= block < nblocks) or nblocks > I0:
        raise ValueError("need 0 <= block < nblocks <= I0")
    base, extra = divmod(I0, nblocks)
    begin = block * base + min(block, extra)
    return begin, begin + base + (1 if block < extra else 0)


def block_state(state: dict, shape: Sequence[int], begin: int, end: int, cplx: bool,
                complex_adam: int = 0) -> dict:
    """The share of a whole tensor's state view (as tgd_get_state returns it)
    that the block of mode-0 rows [begin, end) holds: its Omega entries
    rebased to the block, U_0's rows, the sparse moments of those entries,
    and the (replicated) core moments, counters and other factors."""
    S = math.prod(shape[1:])
    omega = np.asarray(state["omega"], np.int64)
    e0, e1 = (int(x) for x in np.searchsorted(omega, [begin * S, end * S]))
    mc = 2 if cplx else 1
    vc = 2 if (cplx and complex_adam == 1) else 1
    out = {k: state[k] for k in ("t", "refreshes", "has_subspace") if k in state}
    out["omega"] = omega[e0:e1] - begin * S
    out["k"] = e1 - e0
    if state.get("U") is not None:
        out["U"] = [np.ascontiguousarray(state["U"][0][begin:end])] + list(state["U"][1:])
    for key in ("core_m", "core_v"):
        if state.get(key) is not None:
            out[key] = state[key]
    if state.get("sparse_m") is not None:
        out["sparse_m"] = np.asarray(state["sparse_m"])[e0 * mc:e1 * mc]
    if state.get("sparse_v") is not None:
        out["sparse_v"] = np.asarray(state["sparse_v"])[e0 * vc:e1 * vc]
    return out


def allreduce_core(core, group=None):
    """Sums a block's partial core over the process group, in place."""
    import torch.distributed as dist
    dist.all_reduce(core, op=dist.ReduceOp.SUM, group=group)
    return core


class SplitStep:
    """The TensorGRaD step of one block of mode-0 rows of a tensor split
    across the ranks of a process group (one rank per GPU)."""

    def __init__(self, opt, group=None):
        self.opt = opt
        self.group = group

    def step(self, grad, weight, stream=None):
        import torch
        self.opt.step_begin(grad, stream)
        core = self.opt.core_tensor()
        if stream is not None:
            with torch.cuda.stream(stream):
                allreduce_core(core, self.group)
        else:
            allreduce_core(core, self.group)
        self.opt.step_end(weight, stream)

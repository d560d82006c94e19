"""The Python binding refuses tensors the C ABI cannot take, before any call
into the library: host tensors (there is no CPU path), wrong byte sizes,
non-contiguous views and host arrays of the wrong size."""

import numpy as np
import pytest
import torch

import rank_sparse_tensor_b200 as rst


def _handle(shape, grad_dtype="c64", weight_dtype="c64"):
    h = object.__new__(rst.TensorGRaD)
    h.shape = tuple(shape)
    h.N = int(np.prod(shape))
    h.grad_dtype, h.weight_dtype = grad_dtype, weight_dtype
    h._h = None
    return h


def test_host_tensors_are_refused():
    h = _handle((4, 5, 6))
    g = torch.zeros(4, 5, 6, dtype=torch.complex64)
    with pytest.raises(ValueError, match="CUDA device"):
        h.step(g, g.clone())
    with pytest.raises(ValueError, match="CUDA device"):
        h.refresh(g)


def test_non_tensors_are_refused():
    h = _handle((4, 5, 6))
    with pytest.raises(TypeError):
        h.step(np.zeros((4, 5, 6), np.complex64), np.zeros((4, 5, 6), np.complex64))


def test_host_arrays_of_the_wrong_size_are_refused():
    h = _handle((4, 5, 6), "c32h", "c32h")
    good = np.zeros((4, 5, 6, 2), np.float16)
    with pytest.raises(ValueError, match="c32h"):
        h.step_host(np.zeros((4, 5, 5, 2), np.float16), good)
    with pytest.raises(ValueError, match="c32h"):
        h.step_host(good, np.zeros((4, 5, 6, 2), np.float16)[:, :, ::2])


def test_state_memory_needs_matching_lengths():
    with pytest.raises(ValueError):
        rst.state_memory((4, 5), (2,), 0.1)

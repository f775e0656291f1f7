"""The Python binding rejects what the library cannot take, before any call
into it: CPU tensors (there is no CPU fallback), wrong dtypes and shapes.
Runs without a GPU."""
import numpy as np
import pytest
import torch

import block_sparse_attention_38_b200 as bsa


def _bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _i32(n):
    return torch.zeros(n, dtype=torch.int32)


def test_forward_refuses_cpu_tensors():
    q = _bf(1, 2, 256, 64)
    with pytest.raises(ValueError):
        bsa.forward(q, q, q, _i32(17), _i32(8), 32)


def test_forward_refuses_mismatched_shapes():
    with pytest.raises(ValueError):
        bsa.forward(_bf(1, 2, 256, 64), _bf(1, 2, 128, 64), _bf(1, 2, 256, 64), _i32(17),
                    _i32(8), 32)


def test_backward_refuses_cpu_tensors_and_bad_lse():
    q = _bf(1, 2, 256, 64)
    lse = torch.zeros(1, 2, 256)
    with pytest.raises(ValueError):
        bsa.backward(q, q, q, q, q, lse, _i32(17), _i32(8), _i32(17), _i32(8), 32, 0.125)
    with pytest.raises(ValueError):
        bsa.backward(_bf(1, 2, 256), q, q, q, q, lse, _i32(17), _i32(8), _i32(17), _i32(8), 32,
                     0.125)


def test_decode_refuses_cpu_tensors_and_bad_shapes():
    q = _bf(2, 4, 64)
    cache = _bf(2, 4, 512, 64)
    with pytest.raises(ValueError):
        bsa.decode(q, cache, cache, _i32(2), _i32(4 * 16 + 1), _i32(8), 32, 0.125)
    with pytest.raises(ValueError):
        bsa.decode(_bf(2, 4, 32), cache, cache, _i32(2), _i32(65), _i32(8), 32, 0.125)
    with pytest.raises(ValueError):  # only one of k_new / v_new
        bsa.decode(q, cache, cache, _i32(2), _i32(65), _i32(8), 32, 0.125, k_new=q)


def test_topk_refuses_cpu_tensors():
    q = _bf(1, 2, 256, 64)
    with pytest.raises(ValueError):
        bsa.topk_pattern(q, q, 32, 4)
    with pytest.raises(ValueError):
        bsa.topk_pattern_static(q, q, 32, 4, False, _i32(17), _i32(40))


def test_host_transpose_checks_row_ptr_length():
    with pytest.raises(ValueError):
        bsa.transpose_pattern(np.zeros(5, np.int32), np.zeros(0, np.int32), 2, 4)

"""Plain fp64 CPU oracle of the block-sparse attention forward.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg (and its ``--impl reference`` arm) may import,
call, link or run anything in this package.  The product path never does: the
CUDA extension fails loudly when it is missing instead of falling back here.

* ``oracle.c`` -- the forward in fp64 C with OpenMP (the plain definition of
  "Block Sparse Attention with Log-Linear Complexity", section 3.3: a softmax
  restricted to the connected key blocks, then the weighted sum of V).
* ``patterns.py`` -- the block patterns enumerated from the pages' rules.
* ``topk.py`` -- content-based top-k block selection.
* ``decode.py`` -- one decode step: a new token per (b, h) against the
  cached tokens of its block row.
* ``backward.py`` -- the gradients dQ, dK, dV of the forward, and the
  column-major copy of a block-CSR.

Every function here is pinned by the ``-m "not gpu"`` tests against brute
force, closed forms, library routines and a hand-enumerated block list; see
``tests/test_oracle.py`` and ``tests/test_patterns.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

from . import patterns  # noqa: F401  (re-exported)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """ctypes handle of a compiled oracle.c (the tests also load planted-mistake copies)."""
    lib = ctypes.CDLL(path)
    f = lib.oracle_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int,
                                                                ctypes.c_void_p, ctypes.c_int64,
                                                                ctypes.c_void_p, ctypes.c_void_p,
                                                                ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = load_library(_LIB)
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 bit patterns (no value change)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16, x.dtype
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16, a.dtype
    return a


def forward(q, k, v, row_ptr, col_idx, block_size: int, scale: float, causal: bool = False,
            rows: Optional[Sequence[int]] = None, nthreads: int = 0, lib=None):
    """fp64 O and LSE.

    q, k, v: bf16 torch tensors (or uint16 bit arrays) of shape [B, H, N, d].
    row_ptr int32 [H*M+1], col_idx int32 [nnz] (block-CSR, head-major rows).
    rows: optional flat row indices (b*H + h)*N + q; then O is [len(rows), d]
    and LSE is [len(rows)], else O is [B, H, N, d] and LSE is [B, H, N].
    Returns (O, LSE, threads_used) as numpy float64 arrays and an int.
    """
    lib = _load() if lib is None else lib
    B, H, N, d = (int(s) for s in q.shape)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    M = N // block_size
    if rp.shape[0] != H * M + 1:
        raise ValueError("row_ptr must have H*M+1 entries")
    if rows is None:
        O = np.empty((B, H, N, d), dtype=np.float64)
        L = np.empty((B, H, N), dtype=np.float64)
        rows_arr = None
        nrows = 0
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        if rows_arr.size and (rows_arr.min() < 0 or rows_arr.max() >= B * H * N):
            raise ValueError("row index out of range")
        nrows = int(rows_arr.shape[0])
        O = np.empty((nrows, d), dtype=np.float64)
        L = np.empty((nrows,), dtype=np.float64)
    rc = lib.oracle_forward(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, rp.ctypes.data,
                            ci.ctypes.data, B, H, N, d, block_size, float(scale), int(bool(causal)),
                            None if rows_arr is None else rows_arr.ctypes.data, nrows,
                            O.ctypes.data, L.ctypes.data, int(nthreads))
    if rc == -2:
        raise ValueError("bad sizes")
    if rc == -1:
        raise ValueError("column index out of range in col_idx")
    return O, L, rc

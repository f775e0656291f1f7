"""Host side of the top-k selection entry points (no GPU needed)."""
import ctypes

import numpy as np
import pytest

import block_sparse_attention_38_b200 as bsa
from oracle import topk


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("M,k", [(1, 0), (1, 3), (8, 0), (8, 2), (8, 7), (8, 50), (128, 25)])
def test_nnz_matches_the_oracle_row_lengths(M, k, causal):
    BH = 3
    expect = BH * sum(topk.row_length(i, M, k, causal) for i in range(M))
    assert bsa.topk_nnz(BH, M, k, causal) == expect


def test_workspace_size_and_argument_errors():
    lib = bsa.library()
    assert lib.bsa_topk_workspace_bytes(16, 4096, 64, 32) == 2 * 16 * 128 * 64 * 8
    assert lib.bsa_topk_workspace_bytes(16, 4001, 64, 32) == 0   # N % block_size
    assert lib.bsa_topk_nnz(0, 8, 2, 0) == -1
    assert lib.bsa_topk_nnz(1, 8, -1, 0) == -1
    ws = (ctypes.c_double * 64)()
    buf = (ctypes.c_int32 * 64)()
    args = dict(Q=ctypes.addressof(buf), K=ctypes.addressof(buf), BH=1, N=64, d=16, bs=16,
                k=2, causal=0, rp=ctypes.addressof(buf), ci=ctypes.addressof(buf),
                ws=ctypes.addressof(ws), wsb=ctypes.sizeof(ws))

    def call(**kw):
        a = dict(args, **kw)
        return lib.bsa_topk_pattern(a["Q"], a["K"], a["BH"], a["N"], a["d"], a["bs"], a["k"],
                                    a["causal"], a["rp"], a["ci"], a["ws"], a["wsb"], None)
    # every rejection happens before anything is launched
    assert call(Q=None) == bsa.ERR_INVALID_ARG
    assert call(ws=None) == bsa.ERR_INVALID_ARG
    assert call(N=60) == bsa.ERR_INVALID_ARG
    assert call(k=-1) == bsa.ERR_INVALID_ARG
    assert call(causal=2) == bsa.ERR_INVALID_ARG
    assert call(ws=ctypes.addressof(ws) + 4) == bsa.ERR_INVALID_ARG       # alignment
    assert call(d=300) == bsa.ERR_UNSUPPORTED
    assert call(N=16 * 5000) == bsa.ERR_UNSUPPORTED                      # M > 4096
    assert call(wsb=8) == bsa.ERR_BUFFER_TOO_SMALL

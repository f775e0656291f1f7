"""Host side of the backward: bsa_transpose_pattern bit-exact against the
oracle's column-major copy, and bsa_backward's argument checks (every call
below fails a check made before any CUDA call)."""
import ctypes

import numpy as np
import pytest

import block_sparse_attention_38_b200 as bsa
import workloads
from oracle import backward as obw
from oracle import patterns


@pytest.mark.parametrize("name", ["tiny_loglinear", "loglinear_4k", "local_global_8k",
                                  "bernoulli_4k", "causal_loglinear_32k", "sliding_window_8k",
                                  "bigbird_4k"])
def test_transpose_matches_the_oracle_on_workload_patterns(name):
    w = workloads.WORKLOADS[name]
    rp, ci = patterns.csr(w.pattern)
    cp, ri = bsa.transpose_pattern(rp, ci, w.pattern.H, w.pattern.M)
    ocp, ori = obw.transpose_pattern(rp, ci, w.pattern.H, w.pattern.M)
    assert np.array_equal(cp, ocp) and np.array_equal(ri, ori)


def test_transpose_counts_repeats_once_and_handles_empty_rows():
    rng = np.random.default_rng(3)
    H, M = 2, 37
    rows = [list(rng.integers(0, M, rng.integers(0, 9))) for _ in range(H * M)]
    rows[5] = []
    rows[6] = [4, 4, 4, 0, 36]
    rp = np.zeros(H * M + 1, np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([j for r in rows for j in r], np.int32)
    cp, ri = bsa.transpose_pattern(rp, ci, H, M)
    ocp, ori = obw.transpose_pattern(rp, ci, H, M)
    assert np.array_equal(cp, ocp) and np.array_equal(ri, ori)


def test_transpose_rejects_bad_patterns_and_short_buffers():
    lib = bsa.library()
    rp = np.array([0, 2, 3], np.int32)
    ci = np.array([0, 1, 1], np.int32)
    cp = np.zeros(3, np.int32)
    ri = np.zeros(3, np.int32)
    n = ctypes.c_int64(0)

    def call(rp_, ci_, cap=3):
        return lib.bsa_transpose_pattern(rp_.ctypes.data, ci_.ctypes.data, 1, 2, cp.ctypes.data,
                                         ri.ctypes.data, cap, ctypes.byref(n))
    assert call(rp, ci) == bsa.OK and n.value == 3
    assert call(rp, ci, cap=2) == bsa.ERR_BUFFER_TOO_SMALL and n.value == 3
    assert call(np.array([0, 2, 1], np.int32), ci) == bsa.ERR_BAD_PATTERN
    assert call(rp, np.array([0, 2, 1], np.int32)) == bsa.ERR_BAD_PATTERN
    assert call(np.array([1, 2, 3], np.int32), ci) == bsa.ERR_BAD_PATTERN
    assert lib.bsa_transpose_pattern(rp.ctypes.data, ci.ctypes.data, 0, 2, cp.ctypes.data,
                                     ri.ctypes.data, 3, ctypes.byref(n)) == bsa.ERR_INVALID_ARG


P = ctypes.c_void_p(4096)
P8 = ctypes.c_void_p(4104)


def _bwd(**kw):
    a = dict(Q=P, K=P, V=P, O=P, dO=P, LSE=P, rp=P, ci=P, cp=P, ri=P, B=1, H=2, N=512, d=64,
             bs=64, scale=0.125, causal=0, dQ=P, dK=P, dV=P, ws=P, wsb=1 << 20)
    a.update(kw)
    return bsa.library().bsa_backward(a["Q"], a["K"], a["V"], a["O"], a["dO"], a["LSE"], a["rp"],
                                      a["ci"], a["cp"], a["ri"], a["B"], a["H"], a["N"], a["d"],
                                      a["bs"], a["scale"], a["causal"], a["dQ"], a["dK"], a["dV"],
                                      a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw", [
    dict(Q=None), dict(O=None), dict(dO=None), dict(LSE=None), dict(cp=None), dict(ri=None),
    dict(dK=None), dict(ws=None), dict(B=0), dict(N=0), dict(causal=2), dict(N=500),
    dict(scale=float("nan")), dict(Q=P8), dict(dV=P8), dict(ws=ctypes.c_void_p(4100)),
    dict(LSE=ctypes.c_void_p(4098)),
])
def test_backward_invalid_arguments(kw):
    assert _bwd(**kw) == bsa.ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(d=96), dict(bs=16), dict(N=320, bs=64),
                                dict(N=4097 * 32, bs=32)])
def test_backward_unsupported(kw):
    assert _bwd(**kw) == bsa.ERR_UNSUPPORTED


def test_backward_short_workspace():
    # D per query row (fp32), then two costs and two orders per 128-row tile (int32)
    need = 4 * 2 * 512 + 4 * 4 * (2 * 512 // 128)
    assert bsa.library().bsa_backward_workspace_bytes(1, 2, 512) == need
    assert _bwd(wsb=need - 1) == bsa.ERR_BUFFER_TOO_SMALL

"""C-ABI checks that need no GPU.

* libbsa.so loads and exports every function include/bsa.h declares;
* bsa_build_pattern agrees bit for bit with the oracle's independent
  enumeration for every kind, over many M and parameter choices;
* bsa_validate_pattern rejects each kind of corrupted CSR (injected here, on
  the host) and accepts the builders' output;
* bsa_forward rejects bad arguments synchronously, before any CUDA call
  (only argument combinations that fail validation are passed, so nothing is
  ever launched from these tests).
"""
import ctypes
import itertools
import os
import re

import numpy as np
import pytest

import block_sparse_attention_38_b200 as bsa
from block_sparse_attention_38_b200 import build as bsa_build
from oracle import patterns
import workloads
from workloads import PatternDesc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    bsa_build.build()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "bsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert {"bsa_build_pattern", "bsa_validate_pattern", "bsa_forward",
            "bsa_device_status", "bsa_version", "bsa_topk_nnz", "bsa_topk_workspace_bytes",
            "bsa_topk_pattern", "bsa_topk_pattern_static", "bsa_transpose_pattern",
            "bsa_backward_workspace_bytes", "bsa_backward", "bsa_backward_status",
            "bsa_decode", "bsa_decode_status"} <= set(names)
    lib = ctypes.CDLL(bsa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert bsa.version() == 200


def _cases():
    out = []
    for M in (1, 2, 3, 8, 16, 128, 256):
        kmax = max(0, M.bit_length() - 2)
        anchors = (0, M // 2, M - 1)
        for causal in (False, True):
            out.append(PatternDesc(kind=0, M=M, H=2, local_radius=1, log_kmax=kmax,
                                   anchors=anchors, causal=causal))
            out.append(PatternDesc(kind=0, M=M, H=1, local_radius=2, log_kmax=min(3, kmax),
                                   anchors=(M - 1, 5, -3, 1000), causal=causal))
            out.append(PatternDesc(kind=1, M=M, H=2, local_radius=min(4, M), anchors=(0, M - 1),
                                   causal=causal))
            out.append(PatternDesc(kind=1, M=M, H=1, local_radius=0, anchors=(), causal=causal))
            out.append(PatternDesc(kind=2, M=M, H=3, p=0.3, seed=7, causal=causal))
            out.append(PatternDesc(kind=2, M=M, H=2, p=0.0, seed=1, causal=causal))
            out.append(PatternDesc(kind=2, M=M, H=2, p=1.0, seed=2 ** 64 - 1, causal=causal))
            out.append(PatternDesc(kind=3, M=M, H=2, local_radius=min(8, M), dilation=2,
                                   causal=causal))
            out.append(PatternDesc(kind=3, M=M, H=1, local_radius=5, dilation=3, causal=causal))
            out.append(PatternDesc(kind=4, M=M, H=3, local_radius=1, anchors=(0,), num_random=3,
                                   seed=11, causal=causal))
            out.append(PatternDesc(kind=4, M=M, H=2, local_radius=0, anchors=(M - 1, M // 2),
                                   num_random=0, seed=5, causal=causal))
    return out


@pytest.mark.parametrize("desc", _cases(), ids=lambda d: f"k{d.kind}M{d.M}H{d.H}c{int(d.causal)}r{d.local_radius}s{d.dilation}n{d.num_random}")
def test_builder_matches_oracle_enumeration(desc):
    rp, ci = bsa.build_pattern_from(desc)
    orp, oci = patterns.csr(desc)
    assert np.array_equal(rp, orp)
    assert np.array_equal(ci, oci)
    assert bsa.validate_pattern(rp, ci, desc.H, desc.M, desc.causal) == bsa.OK


@pytest.mark.parametrize("name", workloads.ORDER + workloads.EXTRA_ORDER)
def test_builder_matches_oracle_on_workloads(name):
    d = workloads.WORKLOADS[name].pattern
    rp, ci = bsa.build_pattern_from(d)
    orp, oci = patterns.csr(d)
    assert np.array_equal(rp, orp) and np.array_equal(ci, oci)


def test_builder_two_call_and_errors():
    lib = bsa.library()
    anc = (ctypes.c_int32 * 3)(0, 4, 7)
    d = bsa._Desc(0, 8, 2, 1, 2, 3, ctypes.cast(anc, ctypes.POINTER(ctypes.c_int32)), 0.0, 0, 0,
                  1, 0)
    nnz = ctypes.c_int64(-1)
    assert lib.bsa_build_pattern(ctypes.byref(d), None, None, 0, ctypes.byref(nnz)) == bsa.OK
    assert nnz.value == 104
    rp = np.zeros(17, np.int32)
    small = np.zeros(10, np.int32)
    assert lib.bsa_build_pattern(ctypes.byref(d), rp.ctypes.data, small.ctypes.data, 10,
                                 ctypes.byref(nnz)) == bsa.ERR_BUFFER_TOO_SMALL
    assert lib.bsa_build_pattern(ctypes.byref(d), rp.ctypes.data, None, 10,
                                 ctypes.byref(nnz)) == bsa.ERR_INVALID_ARG
    assert lib.bsa_build_pattern(None, None, None, 0, ctypes.byref(nnz)) == bsa.ERR_INVALID_ARG
    assert lib.bsa_build_pattern(ctypes.byref(d), None, None, 0, None) == bsa.ERR_INVALID_ARG
    for field, bad in (("kind", 9), ("M", 0), ("H", 0), ("local_radius", -1), ("log_kmax", 31),
                       ("n_anchors", -1), ("causal", 2)):
        dd = bsa._Desc.from_buffer_copy(d)
        setattr(dd, field, bad)
        assert lib.bsa_build_pattern(ctypes.byref(dd), None, None, 0,
                                     ctypes.byref(nnz)) == bsa.ERR_INVALID_ARG, field
    dd = bsa._Desc.from_buffer_copy(d)
    dd.kind, dd.p = 2, 1.5
    assert lib.bsa_build_pattern(ctypes.byref(dd), None, None, 0,
                                 ctypes.byref(nnz)) == bsa.ERR_INVALID_ARG
    dd = bsa._Desc.from_buffer_copy(d)
    dd.kind, dd.dilation = 3, 0
    assert lib.bsa_build_pattern(ctypes.byref(dd), None, None, 0,
                                 ctypes.byref(nnz)) == bsa.ERR_INVALID_ARG
    dd = bsa._Desc.from_buffer_copy(d)
    dd.kind, dd.num_random = 4, -1
    assert lib.bsa_build_pattern(ctypes.byref(dd), None, None, 0,
                                 ctypes.byref(nnz)) == bsa.ERR_INVALID_ARG
    dd = bsa._Desc.from_buffer_copy(d)
    dd.anchors = None
    assert lib.bsa_build_pattern(ctypes.byref(dd), None, None, 0,
                                 ctypes.byref(nnz)) == bsa.ERR_INVALID_ARG


def test_validator_catches_injected_corruption():
    d = workloads.WORKLOADS["tiny_loglinear"].pattern
    rp, ci = bsa.build_pattern_from(d)
    H, M = d.H, d.M
    assert bsa.validate_pattern(rp, ci, H, M) == bsa.OK

    def v(rp2, ci2, causal=False, cap=None):
        rp2 = np.ascontiguousarray(rp2, np.int32)
        ci2 = np.ascontiguousarray(ci2, np.int32)
        return bsa.library().bsa_validate_pattern(rp2.ctypes.data, ci2.ctypes.data,
                                                  ci2.size if cap is None else cap, H, M,
                                                  int(causal))

    bad = rp.copy(); bad[0] = 1
    assert v(bad, ci) == bsa.ERR_BAD_PATTERN                     # row_ptr[0] != 0
    bad = rp.copy(); bad[3], bad[4] = bad[4], bad[3]
    assert v(bad, ci) == bsa.ERR_BAD_PATTERN                     # not monotone
    bad = ci.copy(); bad[5] = M
    assert v(rp, bad) == bsa.ERR_BAD_PATTERN                     # column out of range
    bad = ci.copy(); bad[2] = -1
    assert v(rp, bad) == bsa.ERR_BAD_PATTERN
    bad = ci.copy(); bad[1], bad[2] = bad[2], bad[1]
    assert v(rp, bad) == bsa.ERR_BAD_PATTERN                     # not ascending
    bad = ci.copy(); bad[2] = bad[1]
    assert v(rp, bad) == bsa.ERR_BAD_PATTERN                     # repeated column
    assert v(rp, ci, causal=True) == bsa.ERR_BAD_PATTERN         # j > i with causal
    assert v(rp, ci, cap=len(ci) - 1) == bsa.ERR_BUFFER_TOO_SMALL
    lib = bsa.library()
    assert lib.bsa_validate_pattern(None, None, 0, H, M, 0) == bsa.ERR_INVALID_ARG
    assert lib.bsa_validate_pattern(rp.ctypes.data, ci.ctypes.data, len(ci), 0, M, 0) == bsa.ERR_INVALID_ARG


def test_forward_rejects_bad_arguments_without_launching():
    lib = bsa.library()
    P = 1 << 20  # fake, 16-byte aligned, never dereferenced: every case below fails validation
    base = dict(Q=P, K=P, V=P, rp=P, ci=P, B=1, H=2, N=256, d=64, bs=32, scale=0.125, causal=0,
                O=P, L=P)

    def call(**kw):
        a = dict(base, **kw)
        return lib.bsa_forward(a["Q"], a["K"], a["V"], a["rp"], a["ci"], a["B"], a["H"], a["N"],
                               a["d"], a["bs"], a["scale"], a["causal"], a["O"], a["L"], None)

    assert call(Q=None) == bsa.ERR_INVALID_ARG
    assert call(ci=None) == bsa.ERR_INVALID_ARG
    assert call(L=None) == bsa.ERR_INVALID_ARG
    assert call(B=0) == bsa.ERR_INVALID_ARG
    assert call(N=-32) == bsa.ERR_INVALID_ARG
    assert call(N=250) == bsa.ERR_INVALID_ARG                    # N % block_size != 0
    assert call(causal=3) == bsa.ERR_INVALID_ARG
    assert call(scale=float("nan")) == bsa.ERR_INVALID_ARG
    assert call(Q=P + 8) == bsa.ERR_INVALID_ARG                  # misaligned
    assert call(d=96) == bsa.ERR_UNSUPPORTED
    assert call(bs=16, N=256) == bsa.ERR_UNSUPPORTED
    assert call(N=32 * 4097) == bsa.ERR_UNSUPPORTED              # M above the supported maximum


def test_forward_ws_rejects_bad_arguments_and_sizes_its_workspace():
    """bsa_forward_ws checks its workspace pointer before any CUDA call, and
    bsa_forward_workspace_bytes is the closed form of its layout: 320 chunk
    slots, four 8-byte count words each, then per slot 128 (m, l) pairs of
    fp32 and a d x 128 fp32 block of O."""
    lib = bsa.library()
    P = 1 << 20
    base = dict(Q=P, K=P, V=P, rp=P, ci=P, B=1, H=2, N=256, d=64, bs=32, scale=0.125, causal=0,
                O=P, L=P, ws=P, nbytes=1 << 24)

    def call(**kw):
        a = dict(base, **kw)
        return lib.bsa_forward_ws(a["Q"], a["K"], a["V"], a["rp"], a["ci"], a["B"], a["H"],
                                  a["N"], a["d"], a["bs"], a["scale"], a["causal"], a["O"], a["L"],
                                  a["ws"], a["nbytes"], None)

    assert call(ws=P + 8) == bsa.ERR_INVALID_ARG                  # misaligned workspace
    assert call(Q=None) == bsa.ERR_INVALID_ARG
    assert call(N=250) == bsa.ERR_INVALID_ARG
    assert call(d=96) == bsa.ERR_UNSUPPORTED
    for d in (64, 128):
        assert bsa.forward_workspace_bytes(d) == 320 * 4 * 8 + 320 * (128 * 8 + 128 * d * 4)
    assert bsa.forward_workspace_bytes(32) == 0

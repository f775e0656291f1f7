"""Property tests of the host-side integer work against the oracle, bit for
bit: the pattern builder (bsa_build_pattern) on random descriptors of every
kind, the column-major copy (bsa_transpose_pattern) on random CSRs with
repeats and unsorted rows, and the closed-form top-k sizes (bsa_topk_nnz).
tests/test_abi.py and tests/test_backward_abi.py hold the hand-picked cases."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import block_sparse_attention_38_b200 as bsa
from oracle import patterns
from workloads import PatternDesc


@st.composite
def descs(draw):
    kind = draw(st.sampled_from([0, 1, 2, 3, 4]))
    M = draw(st.integers(1, 160))
    H = draw(st.integers(1, 3))
    # anchors may fall outside [0, M): both sides discard them
    anchors = tuple(draw(st.lists(st.integers(-3, M + 3), max_size=5)))
    return PatternDesc(kind=kind, M=M, H=H, local_radius=draw(st.integers(0, 12)),
                       log_kmax=draw(st.integers(0, 9)), anchors=anchors,
                       p=draw(st.floats(0.0, 1.0)), seed=draw(st.integers(0, 2 ** 64 - 1)),
                       causal=draw(st.booleans()), dilation=draw(st.integers(1, 7)),
                       num_random=draw(st.integers(0, 6)))


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(descs())
def test_builder_matches_oracle_on_random_descriptors(desc):
    rp, ci = bsa.build_pattern_from(desc)
    orp, oci = patterns.csr(desc)
    assert np.array_equal(rp, orp)
    assert np.array_equal(ci, oci)
    assert bsa.validate_pattern(rp, ci, desc.H, desc.M, desc.causal) == bsa.OK


@st.composite
def csrs(draw):
    H = draw(st.integers(1, 3))
    M = draw(st.integers(1, 40))
    rows = [draw(st.lists(st.integers(0, M - 1), max_size=8)) for _ in range(H * M)]
    rp = np.zeros(H * M + 1, np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([j for r in rows for j in r], np.int32)
    return H, M, rp, ci


@settings(max_examples=150, deadline=None)
@given(csrs())
def test_transpose_matches_oracle_on_random_csrs(case):
    from oracle import backward as obw

    H, M, rp, ci = case
    cp, ri = bsa.transpose_pattern(rp, ci, H, M)
    ocp, ori = obw.transpose_pattern(rp, ci, H, M)
    assert np.array_equal(cp, ocp) and np.array_equal(ri, ori)


@settings(max_examples=200, deadline=None)
@given(st.integers(1, 64), st.integers(1, 4096), st.integers(0, 5000), st.booleans())
def test_topk_nnz_closed_form_matches_the_row_lengths(BH, M, top_k, causal):
    from oracle import topk

    want = BH * sum(topk.row_length(i, M, top_k, causal) for i in range(M))
    assert bsa.topk_nnz(BH, M, top_k, causal) == want

"""Property test of the host pattern builder (bsa_build_pattern): for random
descriptors of every kind, the block-CSR equals the oracle's enumeration bit
for bit (tests/test_abi.py holds the hand-picked cases)."""
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

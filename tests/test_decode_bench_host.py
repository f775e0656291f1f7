"""Host logic of the decode benchmark: the attended-token counts behind its
flop and byte figures equal the sizes of the oracle's attended sets."""
import numpy as np

import bench
import workloads
from oracle import decode as odec
from oracle import patterns


def test_token_counts_match_the_oracle_sets():
    w = workloads.DECODE_WORKLOADS["decode_loglinear_4k"]
    rp, ci = patterns.csr(w.pattern)
    rng = np.random.default_rng(0)
    lens = np.concatenate([[1, w.block_size, w.block_size + 1, w.L][:w.B - 1],
                           rng.integers(1, w.L + 1, 1)])
    n = bench.decode_tokens(w, lens, rp, ci)
    for b in range(w.B):
        for h in range(w.H):
            assert n[b, h] == len(odec.attended_tokens(int(lens[b]) - 1, h, w.M, w.block_size,
                                                       rp, ci))
    assert bench.decode_flops(w, n) == 4.0 * w.d * n.sum()
    # bytes: K and V rows of every attended token, plus the per-(b, h) vectors
    vectors = w.B * w.H * w.d * 2 * 6 + 4 * w.B * w.H + 4 * w.B
    assert bench.decode_bytes(w, n) == 4.0 * w.d * n.sum() + vectors

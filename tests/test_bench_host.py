"""Host logic of the benchmark's flop and byte figures, against counts made
independently from the oracle: the decode leg's attended tokens, and the
causal-exact flops of a causal forward."""
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


def test_causal_exact_flops_count_the_masked_pairs():
    # the bench's closed form against a count over the token-level mask
    from oracle import backward as obw

    w = workloads.Workload("causal_small", 2, 3, 512, 64, 32,
                           workloads.PatternDesc(kind=workloads.LOGLINEAR, M=16, H=3,
                                                 local_radius=1, log_kmax=3,
                                                 anchors=(0, 8, 15), causal=True),
                           seed=0, causal=True)
    rp, ci = patterns.csr(w.pattern)
    pairs = sum(int(obw.allowed_mask(h, w.N, w.block_size, rp, ci, True).sum())
                for h in range(w.H))
    assert bench.causal_exact_flops(w, rp, ci) == 4.0 * w.d * pairs * w.B
    # and the full-block count the metric uses is larger by the masked halves
    assert bench.useful_flops(w, len(ci)) > bench.causal_exact_flops(w, rp, ci)

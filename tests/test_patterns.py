"""Pins of the oracle's pattern enumeration.

* the hand-enumerated log-linear block rows for M = 8 (tests/golden);
* the published SplitMix64 reference outputs that the Bernoulli mask draws from;
* the SparseFlashAttention article's own token-level Local+Global rule with its
  "more than half of the token pairs" block conversion, which must reproduce
  the block band w = 4 for a 256-token window and 64-token blocks;
* closed-form row lengths computed by arithmetic (power-of-two tests, interval
  lengths) instead of set enumeration;
* Bernoulli density within binomial bounds, and the CSR invariants.
"""
import math
import os
import pathlib

import numpy as np
import pytest

from oracle import patterns
import workloads
from workloads import LOGLINEAR, LOCAL_GLOBAL, BERNOULLI, PatternDesc


def _read_golden_rows(path):
    rows = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split(":")
        rows[int(k)] = [int(x) for x in v.split()]
    return rows


GOLDEN_DIR = pathlib.Path(__file__).parent / "golden"


def test_loglinear_matches_hand_enumeration(golden_dir):
    rows = _read_golden_rows(os.path.join(golden_dir, "loglinear_M8_rows.txt"))
    for i in range(8):
        assert patterns.loglinear_cols(i, 8, 2, (0, 4, 7)) == rows[i]
    desc = workloads.WORKLOADS["tiny_loglinear"].pattern
    rp, ci = patterns.csr(desc)
    assert rp[-1] == 2 * 52
    for h in range(2):
        for i in range(8):
            assert list(ci[rp[h * 8 + i]:rp[h * 8 + i + 1]]) == rows[i]


def test_splitmix64_reference_outputs(golden_dir):
    for line in open(os.path.join(golden_dir, "splitmix64_reference.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        state, outs = line.split(":")
        for n, want in enumerate(outs.split(), start=1):
            assert patterns.splitmix64_output(int(state), n) == int(want)


def test_page_token_rule_gives_block_band_of_four():
    # 256-token window, 64-token blocks; globals excluded here because the
    # article's >50 % conversion rule keeps no block for a single global token.
    n, bs, window = 2048, 64, 256
    tok = patterns.local_global_token_mask(n, window, [])
    blk = patterns.token_mask_to_block_mask(tok, bs)
    m = n // bs
    i, j = np.meshgrid(np.arange(m), np.arange(m), indexing="ij")
    assert np.array_equal(blk, np.abs(i - j) <= 4)


def _is_pow2(x):
    return x > 0 and (x & (x - 1)) == 0


def _loglinear_len(i, M, kmax, anchors):
    """Row length by arithmetic: offsets 0 and +/-2^k (k<=kmax) in range, plus the
    anchors that are not already one of those offsets."""
    n = 1
    n += sum(1 for k in range(kmax + 1) if i + (1 << k) < M)
    n += sum(1 for k in range(kmax + 1) if i - (1 << k) >= 0)
    for a in set(anchors):
        delta = abs(a - i)
        if not (delta == 0 or (_is_pow2(delta) and delta <= (1 << kmax))):
            n += 1
    return n


def _local_global_len(i, M, w, globals_):
    if i in globals_:
        return M
    n = min(i + w, M - 1) - max(i - w, 0) + 1
    return n + sum(1 for g in set(globals_) if abs(g - i) > w)


@pytest.mark.parametrize("name", ["tiny_loglinear", "loglinear_4k", "causal_loglinear_32k"])
def test_loglinear_row_lengths_closed_form(name):
    w = workloads.WORKLOADS[name]
    d = w.pattern
    for i in range(d.M):
        cols = patterns.loglinear_cols(i, d.M, d.log_kmax, d.anchors, 1, d.causal)
        if not d.causal:
            assert len(cols) == _loglinear_len(i, d.M, d.log_kmax, d.anchors)
        else:
            # causal: offsets 0 and -2^k in range, plus anchors a < i not already there
            n = 1 + sum(1 for k in range(d.log_kmax + 1) if i - (1 << k) >= 0)
            n += sum(1 for a in set(d.anchors)
                     if a < i and not (_is_pow2(i - a) and i - a <= (1 << d.log_kmax)))
            assert len(cols) == n


def test_local_global_row_lengths_closed_form():
    d = workloads.WORKLOADS["local_global_8k"].pattern
    for i in range(d.M):
        cols = patterns.local_global_cols(i, d.M, d.local_radius, d.anchors)
        assert len(cols) == _local_global_len(i, d.M, d.local_radius, d.anchors)
    assert len(patterns.local_global_cols(0, d.M, 4, d.anchors)) == d.M
    assert len(patterns.local_global_cols(d.M - 1, d.M, 4, d.anchors)) == d.M
    assert len(patterns.local_global_cols(64, d.M, 4, d.anchors)) == 11


def test_bernoulli_density_within_binomial_bounds():
    d = workloads.WORKLOADS["bernoulli_4k"].pattern
    rp, ci = patterns.csr(d)
    M, H, p = d.M, d.H, d.p
    off = H * M * (M - 1)                  # off-diagonal draws
    kept_off = int(rp[-1]) - H * M         # every row holds its diagonal exactly once
    mean, sd = p * off, math.sqrt(off * p * (1 - p))
    assert abs(kept_off - mean) < 6 * sd
    # heads differ (the draw is per (h, i, j))
    rows0 = [tuple(ci[rp[i]:rp[i + 1]]) for i in range(M)]
    rows1 = [tuple(ci[rp[M + i]:rp[M + i + 1]]) for i in range(M)]
    assert rows0 != rows1


def test_bernoulli_uniforms_look_uniform():
    u = np.array([patterns.bernoulli_uniform(7, 0, i, j, 200) for i in range(200) for j in range(200)])
    assert 0.0 <= u.min() and u.max() < 1.0
    hist, _ = np.histogram(u, bins=20, range=(0, 1))
    exp = len(u) / 20
    chi2 = ((hist - exp) ** 2 / exp).sum()
    assert chi2 < 60  # 19 degrees of freedom; p ~ 1e-6 at 50


@pytest.mark.parametrize("name", workloads.ORDER)
def test_csr_invariants(name):
    w = workloads.WORKLOADS[name]
    d = w.pattern
    rp, ci = patterns.csr(d)
    assert rp[0] == 0 and np.all(np.diff(rp) >= 0) and rp[-1] == len(ci)
    for r in range(d.H * d.M):
        row = ci[rp[r]:rp[r + 1]]
        i = r % d.M
        assert np.all(np.diff(row) > 0)
        assert row.min() >= 0 and row.max() < d.M
        assert i in row                      # diagonal present: no empty row
        if d.causal:
            assert row.max() <= i


def test_causal_loglinear_first_row_is_diagonal_only():
    d = workloads.WORKLOADS["causal_loglinear_32k"].pattern
    assert patterns.loglinear_cols(0, d.M, d.log_kmax, d.anchors, 1, True) == [0]


def test_sliding_window_matches_hand_enumeration():
    # M = 10, window 4 blocks each side, every second block: rows written out
    expect = {0: [0, 2, 4], 1: [1, 3, 5], 4: [0, 2, 4, 6, 8], 5: [1, 3, 5, 7, 9], 9: [5, 7, 9]}
    for i, cols in expect.items():
        assert patterns.sliding_window_cols(i, 10, 4, 2) == cols
    # dilation 1 is the plain band; causal keeps j <= i
    assert patterns.sliding_window_cols(3, 10, 2, 1) == [1, 2, 3, 4, 5]
    assert patterns.sliding_window_cols(5, 10, 4, 2, causal=True) == [1, 3, 5]


def test_bigbird_rows_are_window_globals_and_the_drawn_columns():
    M, H, w, seed, R = 64, 3, 1, 11, 3
    for h in range(H):
        for i in range(M):
            cols = patterns.bigbird_cols(h, i, M, w, (0,), R, seed)
            if i == 0:
                assert cols == list(range(M))              # a global row sees every block
                continue
            drawn = {patterns.bigbird_random_col(seed, h, i, r, M, R) for r in range(R)}
            # the draw is output key+1 of the stream, key = (h*M + i)*R + r
            key = (h * M + i) * R
            u = (patterns.splitmix64_output(seed, key + 1) >> 11) / float(1 << 53)
            assert patterns.bigbird_random_col(seed, h, i, 0, M, R) == int(u * M)
            band = {j for j in range(i - w, i + w + 1) if 0 <= j < M}
            assert set(cols) == band | {0} | drawn
    # random columns differ between heads; with no random draws the heads repeat
    rows = [tuple(patterns.bigbird_cols(h, 20, M, w, (0,), R, seed)) for h in range(H)]
    assert len(set(rows)) > 1
    assert patterns.bigbird_cols(1, 20, M, w, (0,), 0, seed) == patterns.bigbird_cols(0, 20, M, w, (0,), 0, seed)


def test_bigbird_row_worked_by_hand_from_published_outputs():
    """Row i = 0 of head 0 with seed 0, M = 16, window 1, global block 5 and
    three random draws.  Its keys are (0*16 + 0)*3 + r = 0, 1, 2, so the
    draws are outputs 1, 2, 3 of the SplitMix64 stream at state 0, which
    tests/golden/splitmix64_reference.txt gives from the published reference:
        16294208416658607535, 7960286522194355700, 487617019471545679.
    A column is floor(u * 16) with u = (output >> 11) / 2^53, i.e.
    floor(output / 2^60): 14.13 -> 14, 6.90 -> 6, 0.42 -> 0.
    The row is the window {0, 1}, the global column 5 and {14, 6, 0}."""
    golden = {}
    for line in open(GOLDEN_DIR / "splitmix64_reference.txt"):
        if line.strip() and not line.startswith("#"):
            state, outs = line.split(":")
            golden[int(state)] = [int(x) for x in outs.split()]
    outs = golden[0]
    assert [o >> 60 for o in outs] == [14, 6, 0]   # the hand division above
    assert [patterns.bigbird_random_col(0, 0, 0, r, 16, 3) for r in range(3)] == [14, 6, 0]
    assert patterns.bigbird_cols(0, 0, 16, 1, (5,), 3, 0) == [0, 1, 5, 6, 14]
    # the global row itself sees every block; another row gets column 5 too
    assert patterns.bigbird_cols(0, 5, 16, 1, (5,), 3, 0) == list(range(16))
    assert 5 in patterns.bigbird_cols(0, 9, 16, 1, (5,), 3, 0)


def test_bigbird_random_columns_spread_over_the_row():
    M, R, seed = 64, 3, 11
    hits = np.zeros(M)
    for h in range(16):
        for i in range(M):
            for r in range(R):
                hits[patterns.bigbird_random_col(seed, h, i, r, M, R)] += 1
    expect = 16 * M * R / M
    # chi-square over 64 cells, 63 degrees of freedom: far below the 0.1 % tail (~104)
    chi2 = float(((hits - expect) ** 2 / expect).sum())
    assert chi2 < 104.0


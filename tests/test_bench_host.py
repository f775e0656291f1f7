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


def test_reference_arm_prints_the_same_config():
    """`--impl reference` (the oracle on the host) and the CUDA arm describe
    the workload with one config dict; the stored-block count of the
    reference's own CSR equals the C builder's."""
    import json
    import os
    import subprocess
    import sys

    import block_sparse_attention_38_b200 as bsa

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_loglinear", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    w = workloads.WORKLOADS["tiny_loglinear"]
    _, ci = bsa.build_pattern_from(w.pattern)
    assert line["impl"] == "reference"
    assert line["config"] == bench.fwd_config(w, len(ci), 1)
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_clock_samples_are_taken_inside_the_region(tmp_path):
    """The sampler's statistics use the samples whose timestamps fall inside
    the timed region only."""
    import datetime

    s = bench.ClockSampler(0)
    path = tmp_path / "c.csv"
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    rows = []
    for i in range(10):
        ts = (t0 + datetime.timedelta(milliseconds=200 * i)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        mhz = 1965 if 3 <= i <= 6 else 900
        cap = "Active" if i == 5 else "Not Active"
        rows.append(f"{ts}, 0, {mhz}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, {cap}")
    path.write_text("\n".join(rows) + "\n")

    class _Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s.proc, s.path = _Done(), str(path)
    lo = (t0 + datetime.timedelta(milliseconds=550)).timestamp()
    hi = (t0 + datetime.timedelta(milliseconds=1250)).timestamp()
    info = s.stop((lo, hi))
    assert info["samples"] == 10 and info["samples_in_timed_region"] == 4
    assert info["sm_mhz"] == 1965 and info["sm_mhz_min"] == 1965
    assert info["reasons"] == ["sw_power_cap"]

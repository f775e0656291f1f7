"""Pins of the top-k block-selection oracle (oracle/topk.py)."""
import numpy as np
import pytest
import torch

from oracle import topk


def _bf16(rng, shape, scale=1.0):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return x.to(torch.bfloat16).float().numpy()


def test_block_means_are_exact_library_means():
    rng = np.random.default_rng(1)
    x = _bf16(rng, (3, 256, 64))
    got = topk.block_means(x, 32)
    ref = torch.from_numpy(x).double().reshape(3, 8, 32, 64).mean(dim=2).numpy()
    # sums of bf16 values of ordinary range are exact in fp64, in any order
    assert np.array_equal(got, ref)


def test_block_scores_match_einsum():
    rng = np.random.default_rng(2)
    qm = rng.standard_normal((2, 16, 64))
    km = rng.standard_normal((2, 16, 64))
    got = topk.block_scores(qm, km)
    ref = np.einsum("bic,bjc->bij", qm, km)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


def test_hand_example():
    # one head, M = 4; scores chosen by hand (row i, column j)
    s = np.array([[[9.0, 3.0, 5.0, 1.0],
                   [2.0, 9.0, 2.0, 7.0],
                   [4.0, 4.0, 9.0, 4.0],
                   [0.0, 6.0, 6.0, 9.0]]])
    rp, ci = topk.select(s, top_k=2, causal=False)
    rows = [list(ci[rp[i]:rp[i + 1]]) for i in range(4)]
    # row 0: 5 (j=2), 3 (j=1);  row 1: 7 (j=3), tie 2/2 -> smaller j = 0;
    # row 2: three-way tie at 4 -> j = 0, 1;  row 3: tie 6/6 -> j = 1, 2
    assert rows == [[0, 1, 2], [0, 1, 3], [0, 1, 2], [1, 2, 3]]
    rp, ci = topk.select(s, top_k=2, causal=True)
    rows = [list(ci[rp[i]:rp[i + 1]]) for i in range(4)]
    assert rows == [[0], [0, 1], [0, 1, 2], [1, 2, 3]]


@pytest.mark.parametrize("causal", [False, True])
def test_selection_keeps_the_highest_scoring_allowed_blocks(causal):
    rng = np.random.default_rng(3)
    BH, M, k = 3, 24, 5
    s = rng.standard_normal((BH, M, M))
    rp, ci = topk.select(s, k, causal)
    for bh in range(BH):
        for i in range(M):
            row = list(ci[rp[bh * M + i]:rp[bh * M + i + 1]])
            assert row == sorted(set(row)) and i in row
            assert len(row) == topk.row_length(i, M, k, causal)
            allowed = [j for j in range(M) if j != i and (not causal or j <= i)]
            chosen = [j for j in row if j != i]
            rest = [j for j in allowed if j not in chosen]
            assert all(j in allowed for j in chosen)
            if chosen and rest:
                assert min(s[bh, i, chosen]) >= max(s[bh, i, rest])


def test_degenerate_k():
    rng = np.random.default_rng(4)
    s = rng.standard_normal((1, 6, 6))
    rp, ci = topk.select(s, 0, False)
    assert list(ci) == list(range(6)) and list(np.diff(rp)) == [1] * 6     # diagonal only
    rp, ci = topk.select(s, 100, False)
    assert list(np.diff(rp)) == [6] * 6                                  # every block
    rp, ci = topk.select(s, 100, True)
    assert list(np.diff(rp)) == [1, 2, 3, 4, 5, 6]                       # causal lower triangle


def test_pattern_prefers_blocks_whose_keys_match_the_queries():
    # Q block 3 equals K block 7 up to noise, so block row 3 must pick column 7
    rng = np.random.default_rng(5)
    B, H, N, d, bs = 1, 1, 512, 64, 32
    q = _bf16(rng, (B, H, N, d), 0.1)
    k = _bf16(rng, (B, H, N, d), 0.1)
    direction = _bf16(rng, (d,), 3.0)
    q[0, 0, 3 * bs:4 * bs] += direction
    k[0, 0, 7 * bs:8 * bs] += direction
    rp, ci = topk.topk_pattern(q, k, bs, 1, False)
    assert list(ci[rp[3]:rp[4]]) == [3, 7]

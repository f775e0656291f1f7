"""Pins of the fp64 oracle's forward against things other than itself.

* brute force: dense fp64 attention over the token-expanded mask with an
  additive -inf mask and a library log-sum-exp (tiny sizes);
* library routines: torch scaled_dot_product_attention in fp64 on the CPU,
  for the all-blocks mask (= dense attention), the causal all-blocks mask,
  and arbitrary block masks given as a boolean attention mask;
* closed forms: diagonal-only mask = independent attention inside each block;
  constant V rows return that row; one-hot V exposes the weights, which sum to
  1 and vanish on unconnected keys ("Block Sparse Attention with Log-Linear
  Complexity", section 3.3); a causal first token sees only itself;
* invariants: the order of a row's column list and repeated entries do not
  change the result (the column set is a union).
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from _refs import _brute, _rand_case, _sdpa64, _token_mask


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 32, 8, 8), (2, 3, 64, 16, 16), (1, 2, 96, 8, 32)])
def test_bruteforce_dense_masked(shape, causal):
    rng = np.random.default_rng(hash((shape, causal)) & 0xFFFF)
    B, H, N, d, bs = shape
    q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.4)
    scale = 1.0 / math.sqrt(d)
    O, L, _ = oracle.forward(q, k, v, rp, ci, bs, scale, causal)
    Ob, Lb = _brute(q, k, v, mask, bs, scale, causal)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    assert np.array_equal(np.isinf(L), np.isinf(Lb))
    fin = np.isfinite(Lb)
    np.testing.assert_allclose(L[fin], Lb[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_all_blocks_equals_library_dense_attention(causal):
    B, H, N, d, bs = 2, 2, 128, 32, 32
    M = N // bs
    g = torch.Generator().manual_seed(11)
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    rp = np.arange(0, H * M * M + 1, M, dtype=np.int32)
    ci = np.tile(np.arange(M, dtype=np.int32), H * M)
    scale = 0.37
    O, L, _ = oracle.forward(q, k, v, rp, ci, bs, scale, causal)
    ref = _sdpa64(q, k, v, scale, is_causal=causal)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    # LSE of dense attention, from the library log-sum-exp of the full score matrix
    s = scale * torch.einsum("bhqc,bhkc->bhqk", q.double(), k.double()).numpy()
    if causal:
        s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    np.testing.assert_allclose(L, logsumexp(s, axis=-1), rtol=0, atol=1e-12)


def test_block_mask_equals_library_masked_attention():
    rng = np.random.default_rng(5)
    B, H, N, d, bs = 1, 3, 128, 16, 16
    q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.3)
    scale = 0.25
    O, L, _ = oracle.forward(q, k, v, rp, ci, bs, scale, False)
    tok = torch.from_numpy(_token_mask(mask, bs, False))[None]  # [1, H, N, N]
    ref = _sdpa64(q, k, v, scale, attn_mask=tok)
    nonempty = tok.any(-1).numpy()  # [1, H, N]
    np.testing.assert_allclose(O[nonempty], ref[nonempty], rtol=0, atol=1e-12)
    # empty rows: O = 0 and LSE = -inf
    assert (~nonempty).sum() > 0
    assert np.all(O[~nonempty] == 0.0)
    assert np.all(np.isneginf(L[~nonempty]))


def test_diagonal_only_is_per_block_attention():
    B, H, N, d, bs = 1, 2, 128, 16, 32
    M = N // bs
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    rp = np.arange(H * M + 1, dtype=np.int32)
    ci = np.tile(np.arange(M, dtype=np.int32), H)
    O, _, _ = oracle.forward(q, k, v, rp, ci, bs, 0.5, False)
    for r in range(M):
        sl = slice(r * bs, (r + 1) * bs)
        ref = _sdpa64(q[:, :, sl], k[:, :, sl], v[:, :, sl], 0.5)
        np.testing.assert_allclose(O[:, :, sl], ref, rtol=0, atol=1e-12)


def test_constant_v_rows_return_the_row():
    rng = np.random.default_rng(9)
    B, H, N, d, bs = 2, 2, 96, 8, 16
    q, k, _, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.5)
    row = torch.randn(d).to(torch.bfloat16)
    v = row.expand(B, H, N, d).contiguous()
    O, L, _ = oracle.forward(q, k, v, rp, ci, bs, 0.3, False)
    ok = np.isfinite(L)
    np.testing.assert_allclose(O[ok], np.broadcast_to(row.double().numpy(), O[ok].shape),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_weights_sum_to_one_and_vanish_off_pattern(causal):
    # V = identity over the N keys exposes w_k as O[q, k].
    rng = np.random.default_rng(21)
    B, H, N, bs = 1, 2, 64, 16
    _, _, _, mask, rp, ci = _rand_case(rng, B, H, N, 8, bs, 0.5)
    v = torch.eye(N).to(torch.bfloat16).expand(B, H, N, N).contiguous()
    # the oracle takes one head dim for Q, K and V, so d = N here
    g = torch.Generator().manual_seed(4)
    q = torch.randn(B, H, N, N, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, N, generator=g).to(torch.bfloat16)
    scale = 1.0 / 8
    W, L, _ = oracle.forward(q, k, v, rp, ci, bs, scale, causal)
    tok = _token_mask(mask, bs, causal)
    ok = np.isfinite(L)
    sums = W.sum(-1)
    np.testing.assert_allclose(sums[ok], 1.0, rtol=0, atol=1e-12)
    assert np.all(W[0][~tok] == 0.0)
    # every connected weight equals exp(s - LSE) with s from fp64 dot products
    s = scale * torch.einsum("bhqc,bhkc->bhqk", q.double(), k.double()).numpy()
    expect = np.where(tok[None], np.exp(s - L[..., None]), 0.0)
    np.testing.assert_allclose(W, expect, rtol=0, atol=1e-12)


def test_causal_first_token_sees_only_itself():
    B, H, N, d, bs = 1, 2, 256, 128, 128
    M = N // bs
    g = torch.Generator().manual_seed(4)
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    rp = np.array([0, 1, 3, 4, 6], np.int32)
    ci = np.array([0, 0, 1, 0, 0, 1], np.int32)
    scale = 1 / math.sqrt(d)
    O, L, _ = oracle.forward(q, k, v, rp, ci, bs, scale, True, rows=[0, N])
    for i, hh in enumerate([0, 1]):
        assert np.array_equal(O[i], v[0, hh, 0].double().numpy())
        dot = float((q[0, hh, 0].double() * k[0, hh, 0].double()).sum())
        assert L[i] == pytest.approx(scale * dot, abs=1e-12)


def test_column_order_and_repeats_do_not_matter():
    rng = np.random.default_rng(33)
    B, H, N, d, bs = 1, 2, 128, 16, 16
    q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.5)
    O1, L1, _ = oracle.forward(q, k, v, rp, ci, bs, 0.3, False)
    # shuffle each row and repeat its first entry
    rows = [list(ci[rp[i]:rp[i + 1]]) for i in range(len(rp) - 1)]
    new = []
    for r in rows:
        r = list(r)
        rng.shuffle(r)
        new.append(r + r[:1])
    rp2 = np.zeros(len(rows) + 1, np.int32)
    rp2[1:] = np.cumsum([len(r) for r in new])
    ci2 = np.array([j for r in new for j in r], np.int32)
    O2, L2, _ = oracle.forward(q, k, v, rp2, ci2, bs, 0.3, False)
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L2, L1, rtol=0, atol=1e-13)


def test_row_subset_matches_full_and_thread_count_is_irrelevant():
    rng = np.random.default_rng(2)
    B, H, N, d, bs = 2, 2, 64, 16, 16
    q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.5)
    O, L, _ = oracle.forward(q, k, v, rp, ci, bs, 0.3, True, nthreads=1)
    O4, L4, _ = oracle.forward(q, k, v, rp, ci, bs, 0.3, True, nthreads=4)
    assert np.array_equal(O, O4) and np.array_equal(L, L4)
    rows = [0, 5, 63, 64 + 17, 3 * 64 + 63]
    Os, Ls, _ = oracle.forward(q, k, v, rp, ci, bs, 0.3, True, rows=rows)
    flatO = O.reshape(-1, d)
    flatL = L.reshape(-1)
    assert np.array_equal(Os, flatO[rows]) and np.array_equal(Ls, flatL[rows])


def test_bad_column_is_reported():
    q = torch.zeros(1, 1, 32, 8, dtype=torch.bfloat16)
    rp = np.array([0, 1, 2], np.int32)
    ci = np.array([0, 5], np.int32)
    with pytest.raises(ValueError):
        oracle.forward(q, q, q, rp, ci, 16, 1.0, False)

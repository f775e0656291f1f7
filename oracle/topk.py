"""Oracle of content-based top-k block selection.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests, the smoke
check and the benchmark's CPU-baseline leg may use it.

What it computes.  The SparseFlashAttention article ("pattern generation",
third kind) describes patterns chosen from the content: the Top-K positions
by the similarity of Q and K.  The RTX 4090 article's tuning notes use
"dynamic sparsity, topk = 20%" for translation.  At block level this build
takes:

* block means  Qm[i, c] = (sum over the bs tokens t of block i of Q[t, c]) / bs,
  and Km likewise, per (b, h);
* block scores s[i, j] = sum over c of Qm[i, c] * Km[j, c];
* row i keeps its diagonal block and the top_k highest-scoring other allowed
  blocks (j != i; j <= i when causal), ties going to the smaller j; if fewer
  are allowed, it keeps all of them.

The integer decision (which blocks) must come out the same on the GPU, so the
arithmetic is fixed down to the rounding: every value is fp64; the means add
the tokens in ascending order (sums of bf16 values that stay exact in fp64
for inputs of ordinary range) and divide by bs (a power of two, exact); the
score adds the products in ascending c, each product rounded on its own (no
fused multiply-add).  numpy's elementwise float64 operations round each
operation exactly once, so the loops below are that definition.

Rows: one CSR row per (b, h, i), i.e. the pattern of a forward run with the
batch folded into the heads ([1, B*H, N, d]).
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def block_means(x: np.ndarray, bs: int) -> np.ndarray:
    """[BH, N, d] bf16-valued array -> [BH, M, d] fp64 block means (tokens added in order)."""
    BH, N, d = x.shape
    M = N // bs
    xb = np.asarray(x, dtype=np.float64).reshape(BH, M, bs, d)
    acc = np.zeros((BH, M, d), dtype=np.float64)
    for t in range(bs):
        acc = acc + xb[:, :, t, :]
    return acc / float(bs)


def block_scores(qm: np.ndarray, km: np.ndarray) -> np.ndarray:
    """[BH, M, d] x [BH, M, d] -> [BH, M, M]: s[i, j] = sum_c qm[i, c] * km[j, c],
    products rounded one by one and added in ascending c."""
    BH, M, d = qm.shape
    s = np.zeros((BH, M, M), dtype=np.float64)
    for c in range(d):
        s = s + qm[:, :, c][:, :, None] * km[:, :, c][:, None, :]
    return s


def row_length(i: int, M: int, top_k: int, causal: bool) -> int:
    """Blocks kept in row i: the diagonal plus min(top_k, other allowed blocks)."""
    others = i if causal else M - 1
    return 1 + min(top_k, others)


def select(scores: np.ndarray, top_k: int, causal: bool) -> Tuple[np.ndarray, np.ndarray]:
    """Top-k block CSR from [BH, M, M] scores: row_ptr int32 [BH*M+1], col_idx int32."""
    BH, M, _ = scores.shape
    rows = []
    for bh in range(BH):
        for i in range(M):
            cand = [j for j in range(M) if j != i and (not causal or j <= i)]
            # descending score, then ascending column
            cand.sort(key=lambda j: (-scores[bh, i, j], j))
            keep = sorted(cand[:top_k] + [i])
            rows.append(keep)
    row_ptr = np.zeros(BH * M + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    col_idx = np.fromiter((j for r in rows for j in r), dtype=np.int32, count=int(row_ptr[-1]))
    return row_ptr.astype(np.int32), col_idx


def topk_pattern(q: np.ndarray, k: np.ndarray, bs: int, top_k: int,
                 causal: bool) -> Tuple[np.ndarray, np.ndarray]:
    """The whole selection for q, k of shape [B, H, N, d] (any float dtype holding
    bf16 values): CSR over B*H*M rows."""
    B, H, N, d = q.shape
    qm = block_means(np.asarray(q, dtype=np.float64).reshape(B * H, N, d), bs)
    km = block_means(np.asarray(k, dtype=np.float64).reshape(B * H, N, d), bs)
    return select(block_scores(qm, km), top_k, causal)

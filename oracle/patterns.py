"""Oracle-side enumeration of the block patterns, written from the pages' rules.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the C++
pattern builder of the CUDA path; the two are compared bit for bit.

Each function returns the set of block columns of one block row, as a sorted
Python list of distinct ints (the CSR order; the forward does not depend on it).

Readings taken where the pages are loose (each is listed in the design notes):

* Log-linear, "Block Sparse Attention with Log-Linear Complexity" sections
  2.3 and 3.1: local blocks |i - j| <= 1, log-stride blocks i +/- 2^k counted
  in block units for k = 0..kmax, and global anchor blocks (start, middle,
  end = 0, M//2, M-1) that act as *columns* every row connects to.  Columns
  outside [0, M) are discarded (the section 4.2 prototype keeps only
  0 <= j < M), not clamped.
* Local+Global, SparseFlashAttention article, "Local + Global" and
  "Block-Sparse": a band |i - j| <= w at block level plus global blocks that
  see every block (full row) and are seen by every block (full column).
* Bernoulli, RTX 4090 article, "core implementation logic" step 1: every
  block kept independently with probability p (the argument the page calls
  "sparsity" is the keep probability of torch.bernoulli), per (h, i, j), with
  the diagonal forced on so that no row is empty.  The page fixes no
  generator; the draws use the counter-based SplitMix64 mix of Steele, Lea and
  Flood ("Fast splittable pseudorandom number generators", OOPSLA 2014): the
  key (h*M + i)*M + j selects output number key+1 of the SplitMix64 stream
  started at `seed`, and its top 53 bits give u in [0, 1).
* causal: only columns j <= i are kept.
"""
from __future__ import annotations

from typing import Iterable, List, Sequence, Tuple

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15


def splitmix64_output(seed: int, n: int) -> int:
    """Output number n (1-based) of the SplitMix64 stream whose state starts at seed.

    The state advances by the golden-ratio increment before each output and
    the output is the state passed through the variant-13 64-bit finaliser
    (xor-shift 30, multiply, xor-shift 27, multiply, xor-shift 31).
    """
    z = (seed + n * GOLDEN_GAMMA) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def bernoulli_uniform(seed: int, h: int, i: int, j: int, M: int) -> float:
    """u(seed, h, i, j) in [0, 1): top 53 bits of output key+1, key = (h*M + i)*M + j."""
    key = (h * M + i) * M + j
    return (splitmix64_output(seed, key + 1) >> 11) * (1.0 / (1 << 53))


def loglinear_cols(i: int, M: int, kmax: int, anchors: Sequence[int],
                   radius: int = 1, causal: bool = False) -> List[int]:
    cols = set()
    for j in range(i - radius, i + radius + 1):          # local blocks
        cols.add(j)
    for k in range(0, kmax + 1):                          # log-stride blocks
        cols.add(i - (1 << k))
        cols.add(i + (1 << k))
    for a in anchors:                                     # global anchor columns
        cols.add(a)
    keep = [j for j in cols if 0 <= j < M and (not causal or j <= i)]
    return sorted(keep)


def local_global_cols(i: int, M: int, w: int, globals_: Sequence[int],
                      causal: bool = False) -> List[int]:
    if i in set(globals_):                                # a global block sees every block
        cols = set(range(M))
    else:
        cols = {j for j in range(M) if abs(i - j) <= w}
        cols.update(g for g in globals_ if 0 <= g < M)    # every block sees the globals
    keep = [j for j in cols if 0 <= j < M and (not causal or j <= i)]
    return sorted(keep)


def bernoulli_cols(h: int, i: int, M: int, p: float, seed: int,
                   causal: bool = False) -> List[int]:
    keep = []
    for j in range(M):
        if causal and j > i:
            continue
        if j == i or bernoulli_uniform(seed, h, i, j, M) < p:
            keep.append(j)
    return keep


def sliding_window_cols(i: int, M: int, w: int, dilation: int,
                        causal: bool = False) -> List[int]:
    """Dilated sliding window at block level (the SparseFlashAttention article's
    sliding_window example): |i - j| <= w and (i - j) a multiple of the dilation."""
    keep = [j for j in range(max(0, i - w), min(M - 1, i + w) + 1)
            if (i - j) % dilation == 0 and (not causal or j <= i)]
    return keep


def bigbird_random_col(seed: int, h: int, i: int, r: int, M: int, num_random: int) -> int:
    """Random column r of block row i, head h: output key+1 of the SplitMix64
    stream at `seed`, key = (h*M + i)*num_random + r, scaled to [0, M)."""
    key = (h * M + i) * num_random + r
    u = (splitmix64_output(seed, key + 1) >> 11) * (1.0 / (1 << 53))
    return min(int(u * M), M - 1)


def bigbird_cols(h: int, i: int, M: int, w: int, globals_: Sequence[int], num_random: int,
                 seed: int, causal: bool = False) -> List[int]:
    """BigBird's three kinds of connections ("Block Sparse Attention with
    Log-Linear Complexity", section 2.2; parameters of the SparseFlashAttention
    article's bigbird example): window |i - j| <= w, global blocks (full row and
    full column) and num_random random columns drawn with replacement."""
    if i in set(globals_):
        cols = set(range(M))
    else:
        cols = {j for j in range(M) if abs(i - j) <= w}
        cols.update(g for g in globals_ if 0 <= g < M)
        cols.update(bigbird_random_col(seed, h, i, r, M, num_random) for r in range(num_random))
    return sorted(j for j in cols if 0 <= j < M and (not causal or j <= i))


def row_cols(desc, h: int, i: int) -> List[int]:
    """Columns of block row i of head h for a workloads.PatternDesc."""
    kind = desc.kind
    if kind == 0:
        return loglinear_cols(i, desc.M, desc.log_kmax, desc.anchors, desc.local_radius,
                              desc.causal)
    if kind == 1:
        return local_global_cols(i, desc.M, desc.local_radius, desc.anchors, desc.causal)
    if kind == 2:
        return bernoulli_cols(h, i, desc.M, desc.p, desc.seed, desc.causal)
    if kind == 3:
        return sliding_window_cols(i, desc.M, desc.local_radius, desc.dilation, desc.causal)
    if kind == 4:
        return bigbird_cols(h, i, desc.M, desc.local_radius, desc.anchors, desc.num_random,
                            desc.seed, desc.causal)
    raise ValueError(f"unknown pattern kind {kind}")


def csr(desc) -> Tuple[np.ndarray, np.ndarray]:
    """Block-CSR over H*M rows (head-major): row_ptr int32 [H*M+1], col_idx int32 [nnz]."""
    M, H = desc.M, desc.H
    rows: List[List[int]] = []
    if desc.kind == 2 or (desc.kind == 4 and desc.num_random > 0):  # drawn per head
        for h in range(H):
            for i in range(M):
                rows.append(row_cols(desc, h, i))
    else:
        one_head = [row_cols(desc, 0, i) for i in range(M)]
        for _ in range(H):
            rows.extend(one_head)
    row_ptr = np.zeros(H * M + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum([len(r) for r in rows], dtype=np.int64).astype(np.int32)
    col_idx = np.fromiter((j for r in rows for j in r), dtype=np.int32, count=int(row_ptr[-1]))
    return row_ptr, col_idx


def dense_block_mask(row_ptr: np.ndarray, col_idx: np.ndarray, H: int, M: int) -> np.ndarray:
    """Boolean [H, M, M] block mask from a CSR (used by brute-force checks)."""
    mask = np.zeros((H, M, M), dtype=bool)
    for h in range(H):
        for i in range(M):
            for p in range(int(row_ptr[h * M + i]), int(row_ptr[h * M + i + 1])):
                mask[h, i, int(col_idx[p])] = True
    return mask


def token_mask_to_block_mask(token_mask: np.ndarray, bs: int) -> np.ndarray:
    """The SparseFlashAttention article's conversion: keep a block when more than
    half of its token pairs are kept (section "Block-Sparse")."""
    n = token_mask.shape[0]
    m = n // bs
    t = token_mask[: m * bs, : m * bs].reshape(m, bs, m, bs)
    return t.mean(axis=(1, 3)) > 0.5


def local_global_token_mask(n: int, window: int, globals_: Iterable[int]) -> np.ndarray:
    """Token-level Local+Global mask of the SparseFlashAttention article: each token
    sees |i - j| <= window; a global token sees every token and is seen by all."""
    idx = np.arange(n)
    mask = np.abs(idx[:, None] - idx[None, :]) <= window
    for g in globals_:
        mask[g, :] = True
        mask[:, g] = True
    return mask

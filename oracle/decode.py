"""Oracle of the decode step: one new query token per (b, h) against its block list.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests, the smoke
check and the benchmark's CPU-baseline leg may use it.

What it computes.  "Block Sparse Attention with Log-Linear Complexity" claims
the pattern cuts the KV cache and the latency of inference (section 1). Its
troubleshooting table (section 5.1) keeps the cache in the (B, H, N, D) layout
of ``past_key_values`` and aligned to blocks.  At decode time each (b, h) adds
one token to its cache and attends once.  This build reads that as follows:

* the new token of batch entry b sits at position t = seq_len[b] - 1 (seq_len
  counts the cached tokens including the new one); its block row is
  i = t // block_size;
* it attends to the tokens of the blocks j listed in CSR row i of head h that
  hold only past or present tokens: blocks j <= i, and in block i the tokens
  up to t (the future is not in the cache, so blocks j > i are skipped);
* with k_new / v_new given, those are the key and value of token t (the
  step appends them to the cache at row t); otherwise row t of the cache is;
* o = sum_k softmax(scale * q . k) v over those tokens, LSE = the natural
  log-sum-exp of the scaled scores; no tokens gives o = 0 and LSE = -inf.

Everything is fp64 from bf16 inputs widened exactly.  Only the gathered rows
are widened, so full-size caches stay cheap.
"""
from __future__ import annotations

from typing import Iterable, Optional, Tuple

import numpy as np


def _rows(x, b: int, h: int, idx) -> np.ndarray:
    """Rows idx of x[b, h] (torch tensor or numpy array) as fp64 [len(idx), d]."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            sel = x[b, h, torch.as_tensor(np.asarray(idx, dtype=np.int64), device=x.device)]
            return sel.double().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x[b, h][np.asarray(idx, dtype=np.int64)], dtype=np.float64)


def _vec(x, b: int, h: int) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x[b, h].double().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x[b, h], dtype=np.float64)


def attended_tokens(t: int, h: int, M: int, bs: int, row_ptr, col_idx) -> list:
    """Token positions the query at position t of head h attends to, ascending."""
    i = t // bs
    cols = sorted(set(int(j) for j in col_idx[row_ptr[h * M + i]:row_ptr[h * M + i + 1]]))
    tokens = []
    for j in cols:
        if j < 0 or j >= M:
            raise ValueError("column index out of range in col_idx")
        if j > i:
            continue
        tokens.extend(range(j * bs, min(j * bs + bs, t + 1)))
    return tokens


def decode(q, k_cache, v_cache, seq_len, row_ptr, col_idx, block_size: int, scale: float,
           k_new=None, v_new=None,
           pairs: Optional[Iterable[Tuple[int, int]]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 O [B, H, d] and LSE [B, H] of one decode step.

    q: [B, H, d]; k_cache, v_cache: [B, H, L, d]; seq_len: [B] ints in [1, L];
    k_new, v_new: optional [B, H, d]; all bf16-valued (torch bf16 tensors or
    float arrays).  row_ptr [H*M+1], col_idx: block-CSR over M = L // block_size
    block rows per head.  pairs: optional (b, h) to compute; the others are NaN.
    """
    B, H, L, d = (int(s) for s in k_cache.shape)
    bs = int(block_size)
    M = L // bs
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx, dtype=np.int64)
    if rp.shape[0] != H * M + 1:
        raise ValueError("row_ptr must have H*M+1 entries")
    lens = [int(x) for x in np.asarray(seq_len).reshape(-1)]
    if len(lens) != B or min(lens) < 1 or max(lens) > M * bs:
        raise ValueError("seq_len must hold B values in [1, L]")
    O = np.full((B, H, d), np.nan)
    LSE = np.full((B, H), np.nan)
    todo = [(b, h) for b in range(B) for h in range(H)] if pairs is None else list(pairs)
    for b, h in todo:
        t = lens[b] - 1
        tokens = attended_tokens(t, h, M, bs, rp, ci)
        if not tokens:
            O[b, h] = 0.0
            LSE[b, h] = -np.inf
            continue
        keys = _rows(k_cache, b, h, tokens)
        vals = _rows(v_cache, b, h, tokens)
        if k_new is not None and tokens[-1] == t:
            keys[-1] = _vec(k_new, b, h)
            vals[-1] = _vec(v_new, b, h)
        s = scale * (keys @ _vec(q, b, h))
        m = s.max()
        w = np.exp(s - m)
        l = w.sum()
        O[b, h] = (w @ vals) / l
        LSE[b, h] = m + np.log(l)
    return O, LSE

"""Oracle of the block-sparse attention backward pass (dQ, dK, dV).

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests, the smoke
check and the benchmark's CPU-baseline leg may use it.

What it computes.  "Block Sparse Attention with Log-Linear Complexity"
(section 4.2) notes that the sparse product falls back to dense work in the
backward pass and (section 5.3) trains with the pattern, so the gradients of
the forward are needed; the pages write no formula for them.  They follow
from the forward's definition by the chain rule.  Per (b, h) and query row q,
with A(q) the keys its block row allows (token-level causal mask when asked):

    s_qk  = scale * q . k                        for k in A(q)
    P_qk  = exp(s_qk) / sum_{k' in A(q)} exp(s_qk')
    dV_k  = sum_q P_qk dO_q
    dP_qk = dO_q . v_k
    dS_qk = P_qk (dP_qk - sum_{k' in A(q)} P_qk' dP_qk')
    dQ_q  = scale * sum_k dS_qk k_k
    dK_k  = scale * sum_q dS_qk q_q

with P = 0 outside A(q) (a row with A(q) empty contributes nothing).  Every
value is fp64 from bf16 inputs widened exactly.  The dense [N, N] arrays per
(b, h) keep the code a plain transcription; inputs are test-sized.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def _f64(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().double().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def allowed_mask(h: int, N: int, bs: int, row_ptr, col_idx, causal: bool) -> np.ndarray:
    """[N, N] bool: key k allowed for query q in head h."""
    M = N // bs
    blocks = np.zeros((M, M), dtype=bool)
    for i in range(M):
        for j in col_idx[row_ptr[h * M + i]:row_ptr[h * M + i + 1]]:
            if j < 0 or j >= M:
                raise ValueError("column index out of range in col_idx")
            blocks[i, j] = True
    tok = np.repeat(np.repeat(blocks, bs, axis=0), bs, axis=1)
    if causal:
        tok &= np.tril(np.ones((N, N), dtype=bool))
    return tok


def backward(q, k, v, dout, row_ptr, col_idx, block_size: int, scale: float,
             causal: bool = False) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """fp64 (dQ, dK, dV), each [B, H, N, d], for bf16-valued q, k, v, dout [B, H, N, d]."""
    Q, Kt, Vt, dO = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = Q.shape
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx, dtype=np.int64)
    if rp.shape[0] != H * (N // block_size) + 1:
        raise ValueError("row_ptr must have H*M+1 entries")
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(Kt)
    dV = np.zeros_like(Vt)
    for h in range(H):
        allow = allowed_mask(h, N, block_size, rp, ci, causal)
        has = allow.any(axis=1)
        for b in range(B):
            s = scale * (Q[b, h] @ Kt[b, h].T)
            s = np.where(allow, s, -np.inf)
            m = np.where(has, s.max(axis=1), 0.0)
            e = np.where(allow, np.exp(s - m[:, None]), 0.0)
            den = e.sum(axis=1)
            P = np.where(has[:, None], e / np.where(has, den, 1.0)[:, None], 0.0)
            dV[b, h] = P.T @ dO[b, h]
            dP = dO[b, h] @ Vt[b, h].T
            rowdot = (P * dP).sum(axis=1)
            dS = P * (dP - rowdot[:, None])
            dQ[b, h] = scale * (dS @ Kt[b, h])
            dK[b, h] = scale * (dS.T @ Q[b, h])
    return dQ, dK, dV


def transpose_pattern(row_ptr, col_idx, H: int, M: int) -> Tuple[np.ndarray, np.ndarray]:
    """Column-major copy of a block-CSR: col_ptr [H*M+1] and row_idx, the rows
    of each (h, column j) ascending, repeats within a row counted once."""
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx, dtype=np.int64)
    cols = []
    for h in range(H):
        lists = [[] for _ in range(M)]
        for i in range(M):
            for j in sorted(set(int(x) for x in ci[rp[h * M + i]:rp[h * M + i + 1]])):
                if j < 0 or j >= M:
                    raise ValueError("column index out of range in col_idx")
                lists[j].append(i)
        cols.extend(lists)
    col_ptr = np.zeros(H * M + 1, dtype=np.int32)
    col_ptr[1:] = np.cumsum([len(c) for c in cols])
    row_idx = np.array([i for c in cols for i in c], dtype=np.int32)
    return col_ptr, row_idx

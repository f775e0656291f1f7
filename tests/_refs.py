"""Independent reference computations used by the oracle's pin tests.

Dense fp64 attention over a token-expanded mask with an additive -inf mask and
scipy's log-sum-exp, and torch's scaled_dot_product_attention in fp64 on the
CPU.  None of this code is shared with the oracle or with the CUDA path.
"""
import numpy as np
import torch
from scipy.special import logsumexp


def _rand_case(rng, B, H, N, d, bs, density, empty_rows=True):
    M = N // bs
    g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, H, N, d, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    mask = rng.random((H, M, M)) < density
    if empty_rows and M > 1:
        mask[0, M - 1, :] = False  # one empty row
    rows = []
    for h in range(H):
        for i in range(M):
            rows.append(sorted(np.nonzero(mask[h, i])[0].tolist()))
    row_ptr = np.zeros(H * M + 1, np.int32)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    col_idx = np.array([j for r in rows for j in r], np.int32)
    return q, k, v, mask, row_ptr, col_idx


def _token_mask(mask, bs, causal):
    """[H, N, N] token-level boolean mask from an [H, M, M] block mask."""
    tok = np.repeat(np.repeat(mask, bs, axis=1), bs, axis=2)
    if causal:
        n = tok.shape[-1]
        tok = tok & np.tril(np.ones((n, n), bool))[None]
    return tok


def _brute(q, k, v, mask, bs, scale, causal):
    """Dense fp64 masked attention: -inf additive mask, library logsumexp."""
    qd = q.double().numpy()
    kd = k.double().numpy()
    vd = v.double().numpy()
    B, H, N, d = qd.shape
    tok = _token_mask(mask, bs, causal)
    O = np.zeros((B, H, N, d))
    L = np.full((B, H, N), -np.inf)
    for b in range(B):
        for h in range(H):
            s = scale * (qd[b, h] @ kd[b, h].T)
            s = np.where(tok[h], s, -np.inf)
            lse = logsumexp(s, axis=1)
            ok = np.isfinite(lse)
            w = np.zeros_like(s)
            w[ok] = np.exp(s[ok] - lse[ok, None])
            O[b, h] = w @ vd[b, h]
            L[b, h] = lse
    return O, L


def _sdpa64(q, k, v, scale, attn_mask=None, is_causal=False):
    return torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), attn_mask=attn_mask, is_causal=is_causal,
        scale=scale).numpy()

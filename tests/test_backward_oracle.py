"""Pins of the backward oracle (oracle/backward.py).

(a) torch autograd in fp64 through a masked softmax attention (empty rows
    give zero output) on random block masks, causal and not;
(b) central finite differences of a dense brute-force forward (tests/_refs.py)
    for a few entries of Q, K and V;
(c) the transposed pattern equals scipy's CSR -> CSC conversion;
and planted mistakes in a copy of the source are each caught.
"""
import os
import types

import numpy as np
import pytest
import scipy.sparse
import torch

import oracle
from _refs import _brute, _rand_case
from oracle import backward as obw

SRC = os.path.join(os.path.dirname(oracle.__file__), "backward.py")


def _autograd(q, k, v, dout, allow, scale):
    """Gradients of sum(O * dO), O the masked-softmax attention (fp64 torch)."""
    Q, K, V = (t.double().clone().requires_grad_(True) for t in (q, k, v))
    s = scale * torch.einsum("bhqd,bhkd->bhqk", Q, K)
    a = torch.from_numpy(allow)[None]                      # [1, H, N, N]
    has = a.any(dim=-1, keepdim=True)
    s = torch.where(a, s, torch.full_like(s, -torch.inf))
    s = torch.where(has, s, torch.zeros_like(s))           # empty rows: any finite row
    p = torch.softmax(s, dim=-1) * has
    O = torch.einsum("bhqk,bhkd->bhqd", p, V)
    (O * dout.double()).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def _allow(H, N, bs, rp, ci, causal):
    return np.stack([obw.allowed_mask(h, N, bs, rp, ci, causal) for h in range(H)])


def _pin_autograd(mod, causal):
    rng = np.random.default_rng(21 + causal)
    B, H, N, d, bs = 2, 2, 128, 16, 16
    q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.4)   # with an empty row
    g = torch.Generator().manual_seed(3)
    dout = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    scale = 0.37
    got = mod.backward(q, k, v, dout, rp, ci, bs, scale, causal)
    want = _autograd(q, k, v, dout, _allow(H, N, bs, rp, ci, causal), scale)
    return all(np.allclose(a, b, rtol=0, atol=1e-10) for a, b in zip(got, want))


def _pin_finite_differences(mod):
    rng = np.random.default_rng(5)
    B, H, N, d, bs = 1, 1, 32, 8, 8
    q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.6, empty_rows=False)
    g = torch.Generator().manual_seed(4)
    dout = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    scale, causal, eps = 0.5, True, 1e-6
    dq, dk, dv = mod.backward(q, k, v, dout, rp, ci, bs, scale, causal)
    base = [t.double() for t in (q, k, v)]

    def loss(ts):
        O, _ = _brute(ts[0], ts[1], ts[2], mask, bs, scale, causal)
        return float((O * dout.numpy()).sum())

    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for (n, c) in ((3, 1), (17, 5), (31, 7)):
            plus = [t.clone() for t in base]
            minus = [t.clone() for t in base]
            plus[which][0, 0, n, c] += eps
            minus[which][0, 0, n, c] -= eps
            fd = (loss(plus) - loss(minus)) / (2 * eps)
            if abs(fd - grad[0, 0, n, c]) > 1e-6 * max(1.0, abs(fd)):
                return False
    return True


def _pin_transpose(mod):
    rng = np.random.default_rng(8)
    H, M = 3, 11
    rows = [sorted(set(rng.integers(0, M, rng.integers(0, 6)).tolist())) + [0]
            for _ in range(H * M)]           # repeats of column 0 in some rows
    rp = np.zeros(H * M + 1, np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([j for r in rows for j in r], np.int32)
    cp, ri = mod.transpose_pattern(rp, ci, H, M)
    for h in range(H):
        sub = scipy.sparse.csr_matrix(
            (np.ones(rp[(h + 1) * M] - rp[h * M]), ci[rp[h * M]:rp[(h + 1) * M]],
             rp[h * M:(h + 1) * M + 1] - rp[h * M]), shape=(M, M))
        sub.sum_duplicates()
        csc = sub.tocsc()
        csc.sort_indices()
        if not np.array_equal(cp[h * M:(h + 1) * M + 1] - cp[h * M], csc.indptr):
            return False
        if not np.array_equal(ri[cp[h * M]:cp[(h + 1) * M]], csc.indices):
            return False
    return True


PINS = [lambda m: _pin_autograd(m, False), lambda m: _pin_autograd(m, True),
        _pin_finite_differences, _pin_transpose]


@pytest.mark.parametrize("i", range(len(PINS)), ids=["autograd", "autograd_causal", "fd",
                                                      "transpose"])
def test_oracle_holds_its_pins(i):
    assert PINS[i](obw)


def test_empty_rows_give_zero_query_gradient():
    rng = np.random.default_rng(2)
    q, k, v, mask, rp, ci = _rand_case(rng, 1, 1, 64, 8, 16, 0.5)
    M = 4
    rows = [list(ci[rp[i]:rp[i + 1]]) for i in range(M)]
    rows[2] = []
    rp2 = np.zeros(M + 1, np.int32)
    rp2[1:] = np.cumsum([len(r) for r in rows])
    ci2 = np.array([j for r in rows for j in r], np.int32)
    dq, dk, dv = obw.backward(q, k, v, v, rp2, ci2, 16, 0.5)
    assert np.all(dq[0, 0, 32:48] == 0)


MUTANTS = {
    "rowdot_without_p": ("rowdot = (P * dP).sum(axis=1)", "rowdot = dP.sum(axis=1)"),
    "dk_without_scale": ("dK[b, h] = scale * (dS.T @ Q[b, h])", "dK[b, h] = dS.T @ Q[b, h]"),
    "dq_uses_transposed_ds": ("dQ[b, h] = scale * (dS @ Kt[b, h])", "dQ[b, h] = scale * (dS.T @ Kt[b, h])"),
    "dv_untransposed_p": ("dV[b, h] = P.T @ dO[b, h]", "dV[b, h] = P @ dO[b, h]"),
    "dp_against_k": ("dP = dO[b, h] @ Vt[b, h].T", "dP = dO[b, h] @ Kt[b, h].T"),
    "causal_ignored": ("if causal:\n        tok &=", "if False:\n        tok &="),
    "head_offset": ("row_ptr[h * M + i]:row_ptr[h * M + i + 1]", "row_ptr[i]:row_ptr[i + 1]"),
    "rows_as_columns": ("lists[j].append(i)", "lists[i].append(j)"),
}


def _mutant(name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, (name, old)
    mod = types.ModuleType(f"backward_mutant_{name}")
    exec(compile(text.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    mod = _mutant(name, *MUTANTS[name])
    caught = False
    for pin in PINS:
        try:
            if not pin(mod):
                caught = True
                break
        except (ValueError, IndexError):
            caught = True
            break
    assert caught, name

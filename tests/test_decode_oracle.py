"""Pins of the decode oracle (oracle/decode.py).

(a) the causal forward oracle (oracle.c, a separate implementation pinned in
    test_oracle.py) at query row t gives the same O and LSE as a decode step
    with seq_len = t + 1, on random block masks that also hold future blocks;
(b) with every block kept, a decode step is torch's scaled_dot_product_attention
    in fp64 over the cache prefix;
(c) closed form at seq_len = 1: o = v_0, LSE = scale * q . k_0;
(d) appending k_new / v_new equals writing them into cache row t first.
Planted mistakes in a copy of the source must each fail one of them.
"""
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle
from _refs import _rand_case
from oracle import decode as dec

SRC = os.path.join(os.path.dirname(oracle.__file__), "decode.py")


def _case(seed, B=2, H=3, N=256, d=32, bs=32, density=0.4):
    rng = np.random.default_rng(seed)
    q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, density)
    return rng, q, k, v, mask, rp, ci


def _pin_forward_row(mod):
    """(a): decode at t equals the causal forward oracle's query row t."""
    rng, Q, K, V, mask, rp, ci = _case(11)
    B, H, N, d = Q.shape
    bs, scale = 32, 1 / math.sqrt(d)
    # positions: a block start, a block end, the last row (empty for h = 0),
    # and random ones; one position per batch entry per trial
    trials = [(32, 255), (31, 0), (100, 200), (int(rng.integers(N)), int(rng.integers(N)))]
    for tb in trials:
        q = torch.stack([Q[b, :, tb[b]] for b in range(B)])
        O, L = mod.decode(q, K, V, np.array(tb) + 1, rp, ci, bs, scale)
        rows = [(b * H + h) * N + tb[b] for b in range(B) for h in range(H)]
        Of, Lf, _ = oracle.forward(Q, K, V, rp, ci, bs, scale, causal=True, rows=rows)
        if not np.allclose(O.reshape(-1, d), Of, rtol=0, atol=1e-12):
            return False
        if not np.array_equal(np.isinf(L.reshape(-1)), np.isinf(Lf)):
            return False
        fin = np.isfinite(Lf)
        if not np.allclose(L.reshape(-1)[fin], Lf[fin], rtol=0, atol=1e-12):
            return False
    return True


def _pin_sdpa(mod):
    """(b): every block kept -> library attention over the prefix."""
    g = torch.Generator().manual_seed(5)
    B, H, N, d, bs = 2, 2, 128, 16, 16
    K = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    V = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    M = N // bs
    rp = np.arange(H * M + 1, dtype=np.int32) * M
    ci = np.tile(np.arange(M, dtype=np.int32), H * M)
    lens = np.array([77, 128])
    scale = 0.3
    O, L = mod.decode(q, K, V, lens, rp, ci, bs, scale)
    for b in range(B):
        n = int(lens[b])
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[b].double()[:, None, :], K[b, :, :n].double(), V[b, :, :n].double(), scale=scale)
        s = scale * torch.einsum("hd,hnd->hn", q[b].double(), K[b, :, :n].double())
        if not np.allclose(O[b], ref[:, 0].numpy(), rtol=0, atol=1e-12):
            return False
        if not np.allclose(L[b], torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12):
            return False
    return True


def _pin_first_token(mod):
    """(c): seq_len = 1 sees only token 0."""
    _, Q, K, V, mask, rp, ci = _case(3, density=1.0)
    B, H, N, d = Q.shape
    q = Q[:, :, 5]
    O, L = mod.decode(q, K, V, np.ones(B, dtype=int), rp, ci, 32, 0.7)
    if not np.array_equal(O, V[:, :, 0].double().numpy()):
        return False
    want = 0.7 * (q.double() * K[:, :, 0].double()).sum(-1).numpy()
    # h = 0's last row is empty in _rand_case; row 0 is full here
    return np.allclose(L, want, rtol=0, atol=1e-12)


def _pin_append(mod):
    """(d): k_new / v_new act as cache row t."""
    _, Q, K, V, mask, rp, ci = _case(4, density=0.7)
    B, H, N, d = Q.shape
    g = torch.Generator().manual_seed(9)
    kn = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, H, d, generator=g).to(torch.bfloat16)
    lens = np.array([65, 190])
    q = Q[:, :, 0]
    O1, L1 = mod.decode(q, K, V, lens, rp, ci, 32, 0.5, k_new=kn, v_new=vn)
    K2, V2 = K.clone(), V.clone()
    for b in range(B):
        K2[b, :, lens[b] - 1] = kn[b]
        V2[b, :, lens[b] - 1] = vn[b]
    O2, L2 = mod.decode(q, K2, V2, lens, rp, ci, 32, 0.5)
    same = np.array_equal(O1, O2) and np.array_equal(L1, L2)
    # and the new token really is attended: the result differs from the old cache
    O3, _ = mod.decode(q, K, V, lens, rp, ci, 32, 0.5)
    return same and not np.array_equal(O1, O3)


PINS = (_pin_forward_row, _pin_sdpa, _pin_first_token, _pin_append)


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_holds_its_pins(pin):
    assert pin(dec)


def test_empty_row_and_argument_errors():
    _, Q, K, V, mask, rp, ci = _case(2)
    B, H, N, d = Q.shape
    # h = 0's block row M-1 is empty in _rand_case
    O, L = dec.decode(Q[:, :, 0], K, V, np.array([N, N]), rp, ci, 32, 1.0)
    assert np.all(O[:, 0] == 0) and np.all(np.isneginf(L[:, 0]))
    with pytest.raises(ValueError):
        dec.decode(Q[:, :, 0], K, V, np.array([0, 5]), rp, ci, 32, 1.0)
    with pytest.raises(ValueError):
        dec.decode(Q[:, :, 0], K, V, np.array([N + 1, 5]), rp, ci, 32, 1.0)


MUTANTS = {
    "last_token_excluded": ("min(j * bs + bs, t + 1)", "min(j * bs + bs, t)"),
    "block_row_rounds_up": ("i = t // bs", "i = (t + bs - 1) // bs"),
    "dropped_scale": ("s = scale * (keys @ _vec(q, b, h))", "s = keys @ _vec(q, b, h)"),
    "head_offset": ("row_ptr[h * M + i]:row_ptr[h * M + i + 1]", "row_ptr[i]:row_ptr[i + 1]"),
    "append_ignored": ("keys[-1] = _vec(k_new, b, h)", "keys[-1] = keys[-1]"),
    "lse_without_max": ("LSE[b, h] = m + np.log(l)", "LSE[b, h] = np.log(l)"),
    "no_normalisation": ("O[b, h] = (w @ vals) / l", "O[b, h] = w @ vals"),
    "values_are_keys": ("vals = _rows(v_cache, b, h, tokens)", "vals = _rows(k_cache, b, h, tokens)"),
    "first_entry_length": ("t = lens[b] - 1", "t = lens[0] - 1"),
    "max_sign": ("w = np.exp(s - m)", "w = np.exp(s + m)"),
}


def _mutant_module(name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, (name, old)
    mod = types.ModuleType(f"decode_mutant_{name}")
    exec(compile(text.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    return mod


def _caught(mod):
    for pin in PINS:
        try:
            if not pin(mod):
                return True
        except (ValueError, IndexError, FloatingPointError):
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    assert _caught(_mutant_module(name, old, new)), name

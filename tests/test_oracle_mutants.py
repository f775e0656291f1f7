"""Planted mistakes in a copy of the oracle must fail the pins.

Each mutant is a one-token edit of oracle.c of the kind a reader could miss
(a dropped term, a wrong sign or index, a transposed operand, an off-by-one in
the causal test).  The copy is compiled on the CPU into a temporary directory
and run through the same brute-force, library and closed-form checks as the
real oracle; every mutant must be caught by at least one of them, and the
unmodified source must pass all of them.
"""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from _refs import _brute, _rand_case, _sdpa64

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "causal_off_by_one": ("if (causal && k > q) continue;", "if (causal && k >= q) continue;"),
    "dropped_scale": ("score[i] = scale * dot;", "score[i] = dot;"),
    "max_sign": ("score[i] = exp(score[i] - m);", "score[i] = exp(score[i] + m);"),
    "k_operand_is_q": ("dot += widen_bf16(qrow[c]) * widen_bf16(krow[c]);",
                       "dot += widen_bf16(qrow[c]) * widen_bf16(qrow[c]);"),
    "v_row_index": ("const uint16_t *vrow = V + (head * N + keys[i]) * (int64_t)d;",
                    "const uint16_t *vrow = V + (head * N + q) * (int64_t)d;"),
    "block_to_token_index": ("int64_t k = (int64_t)j * bs + t;", "int64_t k = (int64_t)j + t;"),
    # an off-by-one that stays inside [0, M): (q - 1) / bs truncates to 0 at q = 0
    "block_row_of_query": ("const int64_t r = q / bs;", "const int64_t r = (q - 1) / bs;"),
    "no_normalisation": ("const double w = score[i] / l;", "const double w = score[i];"),
    "duplicates_counted": ("if (seen[j]) continue;", ";"),
    "lse_without_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "head_offset": ("const int64_t head = b * H + h;", "const int64_t head = h;"),
}


def _compile(tmp_path, name, text):
    src = tmp_path / f"{name}.c"
    lib = tmp_path / f"lib{name}.so"
    src.write_text(text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(src), "-o",
                    str(lib), "-lm"], check=True)
    return oracle.load_library(str(lib))


def _pins_pass(lib):
    """True when every pin holds for this library (a mutant that reports an
    error instead of a result fails them too)."""
    try:
        return _pins_hold(lib)
    except ValueError:
        return False


def _pins_hold(lib):
    rng = np.random.default_rng(1234)
    # brute force, plain and causal, with duplicated column entries
    for causal in (False, True):
        B, H, N, d, bs = 2, 2, 64, 16, 16
        q, k, v, mask, rp, ci = _rand_case(rng, B, H, N, d, bs, 0.5)
        rows = [list(ci[rp[i]:rp[i + 1]]) for i in range(len(rp) - 1)]
        rows = [r + r[:1] for r in rows]
        rp2 = np.zeros(len(rows) + 1, np.int32)
        rp2[1:] = np.cumsum([len(r) for r in rows])
        ci2 = np.array([j for r in rows for j in r], np.int32)
        scale = 1.0 / math.sqrt(d)
        O, L, _ = oracle.forward(q, k, v, rp2, ci2, bs, scale, causal, lib=lib)
        Ob, Lb = _brute(q, k, v, mask, bs, scale, causal)
        if not np.allclose(O, Ob, rtol=0, atol=1e-10):
            return False
        fin = np.isfinite(Lb)
        if not np.array_equal(fin, np.isfinite(L)) or not np.allclose(L[fin], Lb[fin], atol=1e-10):
            return False
    # library dense attention with all blocks present
    B, H, N, d, bs = 1, 2, 64, 16, 16
    M = N // bs
    g = torch.Generator().manual_seed(7)
    q, k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    rp = np.arange(0, H * M * M + 1, M, dtype=np.int32)
    ci = np.tile(np.arange(M, dtype=np.int32), H * M)
    O, _, _ = oracle.forward(q, k, v, rp, ci, bs, 0.3, True, lib=lib)
    return np.allclose(O, _sdpa64(q, k, v, 0.3, is_causal=True), rtol=0, atol=1e-10)


def test_unmodified_oracle_passes(tmp_path):
    assert _pins_pass(_compile(tmp_path, "orig", open(SRC).read()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    text = open(SRC).read()
    old, new = MUTANTS[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    assert not _pins_pass(_compile(tmp_path, name, text.replace(old, new)))

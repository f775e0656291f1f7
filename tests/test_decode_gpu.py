"""GPU parity of the decode step (bsa_decode) against the decode oracle.

Cache rows after each query's position are filled with NaN before the call
(row t too when the step appends), so any read of them would show in O.  The
append must write exactly row t of each (b, h) and leave every other row.
Tolerances are those of the forward: O max-abs 2e-2 and mean-abs 2e-3, LSE
1e-3 (bf16 inputs, fp32 accumulation, exp2 approximation).
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_38_b200 as bsa
import workloads
from _refs import _rand_case
from oracle import decode as odec

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _loglinear_csr(M, H, kmax):
    rp, ci = bsa.build_pattern(bsa.LOGLINEAR, M, H, local_radius=1, log_kmax=kmax,
                               anchors=(0, M // 2, M - 1), causal=True)
    return rp, ci


def _inputs(B, H, L, d, seed):
    g = torch.Generator().manual_seed(seed)

    def r(*shape):
        return torch.randn(*shape, generator=g).to(torch.bfloat16)

    return r(B, H, d), r(B, H, d), r(B, H, d), r(B, H, L, d), r(B, H, L, d)


def _poison_after(cache, lens, from_t):
    """NaN in rows > t (>= t when from_t) of each batch entry."""
    c = cache.clone()
    for b, n in enumerate(lens):
        start = n - 1 if from_t else n
        c[b, :, start:] = float("nan")
    return c


def _run_case(B, H, L, d, bs, lens, rp, ci, append, seed):
    q, kn, vn, K, V = _inputs(B, H, L, d, seed)
    Kp, Vp = _poison_after(K, lens, append), _poison_after(V, lens, append)
    if not append:
        kn = vn = None
    scale = 1.0 / math.sqrt(d)
    Kd, Vd = Kp.to(DEV), Vp.to(DEV)
    O, LSE = bsa.decode(q.to(DEV), Kd, Vd, torch.tensor(lens, dtype=torch.int32, device=DEV),
                        torch.from_numpy(np.asarray(rp, np.int32)).to(DEV),
                        torch.from_numpy(np.asarray(ci, np.int32)).to(DEV), bs, scale,
                        k_new=None if kn is None else kn.to(DEV),
                        v_new=None if vn is None else vn.to(DEV))
    torch.cuda.synchronize()
    assert bsa.decode_status(clear=True) == 0
    Or, Lr = odec.decode(q, K, V, np.asarray(lens), rp, ci, bs, scale, k_new=kn, v_new=vn)
    Og, Lg = O.float().cpu().numpy(), LSE.cpu().numpy()
    err = np.abs(Og - Or)
    assert np.isfinite(Og).all()
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    assert np.array_equal(np.isneginf(Lg), np.isneginf(Lr))
    fin = np.isfinite(Lr)
    assert np.abs(Lg[fin] - Lr[fin]).max(initial=0.0) <= 1e-3
    if append:
        Kc, Vc = Kd.cpu(), Vd.cpu()
        for b, n in enumerate(lens):
            assert torch.equal(Kc[b, :, n - 1], kn[b]) and torch.equal(Vc[b, :, n - 1], vn[b])
        # every other row is untouched (NaN rows compared by bits)
        mask = torch.ones(B, L, dtype=torch.bool)
        for b, n in enumerate(lens):
            mask[b, n - 1] = False
        for got, ref in ((Kc, Kp), (Vc, Vp)):
            g16 = got.view(torch.int16).permute(0, 2, 1, 3)[mask]
            r16 = ref.view(torch.int16).permute(0, 2, 1, 3)[mask]
            assert torch.equal(g16, r16)


# (B, H, L, d, bs, lens): lengths at 1, block starts and ends, and L
SHAPES = [
    (3, 2, 512, 64, 32, [1, 32, 512]),
    (2, 3, 1024, 128, 64, [64, 65]),
    (2, 2, 1024, 128, 128, [128, 1000]),
    (4, 2, 2048, 64, 64, [1, 127, 129, 2048]),
    (2, 4, 1024, 128, 32, [33, 1024]),
    (2, 2, 512, 64, 128, [255, 256]),
]


@pytest.mark.parametrize("append", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}L{}d{}bs{}".format(*s[:5]))
def test_random_masks(shape, append):
    B, H, L, d, bs, lens = shape
    rng = np.random.default_rng(L + d + bs)
    # random block masks with future blocks and one empty row (h = 0, last row)
    _, _, _, _, rp, ci = _rand_case(rng, 1, H, L, 8, bs, 0.35)
    _run_case(B, H, L, d, bs, lens, rp, ci, append, seed=B * L + d)


@pytest.mark.parametrize("append", [False, True])
def test_causal_loglinear(append):
    B, H, L, d, bs = 4, 4, 4096, 128, 64
    rp, ci = _loglinear_csr(L // bs, H, 6)
    rng = np.random.default_rng(2)
    lens = [int(x) for x in rng.integers(1, L + 1, B)]
    _run_case(B, H, L, d, bs, lens, rp, ci, append, seed=5)


def test_repeated_and_unsorted_columns_count_once():
    B, H, L, d, bs = 2, 2, 512, 64, 64
    M = L // bs
    rows = [[3, 0, 3, 1, 7, 0]] * (H * M)   # repeats, unsorted, one future block
    rp = np.zeros(H * M + 1, np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([j for r in rows for j in r], np.int32)
    _run_case(B, H, L, d, bs, [200, 512], rp, ci, True, seed=3)


def test_workload_full_size_sampled():
    w = workloads.DECODE_WORKLOADS["decode_loglinear_32k"]
    q, kn, vn, K, V, lens = workloads.make_decode_inputs(w, device=DEV)
    rp, ci = bsa.build_pattern_from(w.pattern)
    K0 = K.clone()
    O, LSE = bsa.decode(q, K, V, lens, torch.from_numpy(rp).to(DEV), torch.from_numpy(ci).to(DEV),
                        w.block_size, w.scale, k_new=kn, v_new=vn)
    torch.cuda.synchronize()
    assert bsa.decode_status(clear=True) == 0
    rng = np.random.default_rng(0)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, w.B, 48), rng.integers(0, w.H, 48))]
    pairs += [(b, w.H - 1) for b in range(w.B)]
    Or, Lr = odec.decode(q, K0, V, lens.cpu().numpy(), rp, ci, w.block_size, w.scale,
                         k_new=kn, v_new=vn, pairs=pairs)
    Og, Lg = O.float().cpu().numpy(), LSE.cpu().numpy()
    for b, h in pairs:
        assert np.abs(Og[b, h] - Or[b, h]).max() <= 2e-2
        assert abs(Lg[b, h] - Lr[b, h]) <= 1e-3
    assert np.isfinite(Og).all()
    # the append wrote row t of every (b, h)
    t = (lens.long() - 1).cpu()
    for b in range(w.B):
        assert torch.equal(K[b, :, t[b]].cpu(), kn[b].cpu())
        assert torch.equal(V[b, :, t[b]].cpu(), vn[b].cpu())


def test_bad_seq_len_and_bad_column_set_status():
    B, H, L, d, bs = 3, 2, 512, 64, 64
    M = L // bs
    rp, ci = _loglinear_csr(M, H, 2)
    q, _, _, K, V = _inputs(B, H, L, d, 9)
    dev = lambda x: torch.from_numpy(np.asarray(x, np.int32)).to(DEV)  # noqa: E731
    lens = [0, 300, L + 1]
    O, LSE = bsa.decode(q.to(DEV), K.to(DEV), V.to(DEV), dev(lens), dev(rp), dev(ci), bs, 0.125)
    torch.cuda.synchronize()
    assert bsa.decode_status(clear=True) == bsa.STATUS_BAD_SEQ_LEN
    Og, Lg = O.float().cpu().numpy(), LSE.cpu().numpy()
    for b in (0, 2):
        assert (Og[b] == 0).all() and np.isneginf(Lg[b]).all()
    Or, Lr = odec.decode(q[1:2], K[1:2], V[1:2], np.array([300]), rp, ci, bs, 0.125)
    assert np.abs(Og[1] - Or[0]).max() <= 2e-2
    # a column outside [0, M) is skipped and reported
    ci_bad = np.asarray(ci, np.int32).copy()
    ci_bad[rp[4]] = M + 5   # head 0, block row 4 (the row of token 300)
    O2, _ = bsa.decode(q.to(DEV), K.to(DEV), V.to(DEV), dev([300, 300, 300]), dev(rp),
                       dev(ci_bad), bs, 0.125)
    torch.cuda.synchronize()
    assert bsa.decode_status(clear=True) & bsa.STATUS_BAD_COLUMN
    keep = [j for j in ci[rp[4]:rp[5]]][1:]
    ci_ref = np.concatenate([ci[:rp[4]], keep, ci[rp[5]:]]).astype(np.int32)
    rp_ref = np.asarray(rp, np.int64).copy()
    rp_ref[5:] -= 1
    Or2, _ = odec.decode(q, K, V, np.array([300, 300, 300]), rp_ref, ci_ref, bs, 0.125)
    assert np.abs(O2.float().cpu().numpy() - Or2).max() <= 2e-2

"""GPU parity of the chunked tiles: long key walks cut into chunks whose
partial results are merged with log-sum-exp weights ("split long rows into
kv-chunks"; the merged softmax is the restricted softmax of "Block Sparse
Attention with Log-Linear Complexity", section 3.3).

Patterns with a few rows far longer than the rest (full global rows on a
single head) make the schedule cut those tiles; the workspace's count words
show that chunks ran and were merged.  Every output row is compared with the
fp64 oracle at the forward's tolerances.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_38_b200 as bsa
import oracle
from oracle import patterns
import workloads
from workloads import LOCAL_GLOBAL, LOGLINEAR, PatternDesc, Workload

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_ABS = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bsa.library()
    bsa.device_status(clear=True)
    yield
    torch.cuda.synchronize()


def _lg(N, d, bs, H=1, B=1, seed=21):
    M = N // bs
    return Workload(f"lg_{N}_{d}_{bs}", B, H, N, d, bs,
                    PatternDesc(kind=LOCAL_GLOBAL, M=M, H=H, local_radius=4, anchors=(0, M - 1)),
                    seed=seed, key_scale_max=3.0)


def _ll(N, d, bs, causal, H=1, seed=22):
    M = N // bs
    kmax = max(0, int(np.log2(M)) - 1)
    return Workload(f"ll_{N}_{d}_{bs}_{int(causal)}", 1, H, N, d, bs,
                    PatternDesc(kind=LOGLINEAR, M=M, H=H, local_radius=1, log_kmax=kmax,
                                anchors=(0, M // 2, M - 1), causal=causal),
                    seed=seed, causal=causal)


CASES = [
    _lg(8192, 128, 64),            # the long-row case: rows 0 and M-1 hold all 128 blocks
    _lg(8192, 64, 64),
    _lg(4096, 64, 32),             # four block rows per tile
    _lg(8192, 128, 128),
    _ll(16384, 128, 128, True),    # causal, rows of rising length
    _ll(4096, 64, 32, False),
]


def _slots(d, nbytes):
    per = 32 + 128 * 8 + 128 * d * 4      # count words + (m, l) + O of one chunk slot
    full = bsa.forward_workspace_bytes(d)
    return full // per, per


def _counts(ws, d):
    n, _ = _slots(d, ws.numel())
    words = ws[: n * 32].view(torch.int64).cpu().numpy().astype(np.uint64)
    return (words & np.uint64(0xFF)).astype(np.int64)


def _check(w, O, L, what):
    q, k, v = workloads.make_qkv(w)
    rp, ci = patterns.csr(w.pattern)
    Or, Lr, _ = oracle.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal)
    Og = O.float().cpu().numpy().astype(np.float64)
    Lg = L.cpu().numpy().astype(np.float64)
    err = np.abs(Og - Or)
    assert np.isfinite(Og).all(), what
    assert err.max() <= O_MAX, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: O mean-abs {err.mean():.3e}"
    ninf = np.isneginf(Lr)
    assert np.array_equal(np.isneginf(Lg), ninf), what
    if (~ninf).any():
        assert np.abs(Lg[~ninf] - Lr[~ninf]).max() <= LSE_ABS, what


def _inputs(w):
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    rp, ci = bsa.build_pattern_from(w.pattern)
    return q, k, v, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_split_matches_oracle(w):
    q, k, v, rp, ci = _inputs(w)
    nbytes = bsa.forward_workspace_bytes(w.d)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    O, L = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal, workspace=ws)
    torch.cuda.synchronize()
    assert bsa.device_status(clear=True) == 0
    cnt = _counts(ws, w.d)
    assert cnt.max() >= 2, "no tile was cut into chunks"
    _check(w, O, L, w.name)


def test_split_equals_unsplit_within_rounding():
    w = CASES[0]
    q, k, v, rp, ci = _inputs(w)
    O1, L1 = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal, split=False)
    O2, L2 = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal, split=True)
    torch.cuda.synchronize()
    assert bsa.device_status(clear=True) == 0
    assert (O1.float() - O2.float()).abs().max().item() <= 2e-2
    fin = torch.isfinite(L1)
    assert torch.equal(fin, torch.isfinite(L2))
    assert (L1[fin] - L2[fin]).abs().max().item() <= 1e-3
    _check(w, O1, L1, "unsplit")


@pytest.mark.parametrize("slots,cut", [(1, False), (70, True)])
def test_small_workspace(slots, cut):
    """A workspace of a few chunk slots: no cut when the heavy tiles alone do
    not fit; fewer, longer chunks when a few more fit (64 heavy tiles here)."""
    w = CASES[0]
    q, k, v, rp, ci = _inputs(w)
    n_max, per = _slots(w.d, 0)
    ws = torch.zeros(n_max * 32 + slots * (per - 32), dtype=torch.uint8, device="cuda")
    O, L = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal, workspace=ws)
    torch.cuda.synchronize()
    assert bsa.device_status(clear=True) == 0
    cnt = _counts(ws, w.d)
    assert (cnt.max() >= 2) == cut
    _check(w, O, L, f"{slots} slots")


def test_garbage_workspace_and_reuse():
    """Count words left by earlier launches or holding garbage are ignored."""
    w = CASES[1]
    q, k, v, rp, ci = _inputs(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    ws = torch.randint(0, 256, (bsa.forward_workspace_bytes(w.d),), generator=g,
                       dtype=torch.uint8, device="cuda")
    for rep in range(3):
        O, L = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal, workspace=ws)
        torch.cuda.synchronize()
        assert bsa.device_status(clear=True) == 0
        _check(w, O, L, f"launch {rep}")


def test_workspace_bytes():
    assert bsa.forward_workspace_bytes(64) > 0 and bsa.forward_workspace_bytes(128) > 0
    assert bsa.forward_workspace_bytes(96) == 0
    n64, _ = _slots(64, 0)
    n128, _ = _slots(128, 0)
    assert n64 == n128 >= 2 * 148

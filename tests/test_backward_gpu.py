"""GPU parity of the backward pass (bsa_backward) against the fp64 oracle.

The GPU side runs bsa_forward first and feeds its O (bf16) and LSE (fp32) to
the backward, as training does; the oracle computes the exact gradients of
the definition from Q, K, V and dO.

Tolerance, from the arithmetic: P and dS enter the tensor-core products
rounded to bf16 (relative error up to 2^-9), and D = dO . O uses the bf16 O
of the forward; with fp32 accumulation the error of an output element is a
few bf16 units of the magnitudes it sums.  Measured against each gradient's
scale: max-abs error <= 2e-2 * max|ref| and mean-abs error <= 1e-2 * mean|ref|
(about 10 and 5 bf16 units).
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_38_b200 as bsa
import workloads
from _refs import _rand_case
from oracle import backward as obw

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _run(B, H, N, d, bs, rp, ci, causal, seed):
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    do = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    M = N // bs
    cp, ri = bsa.transpose_pattern(rp, ci, H, M)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(DEV)  # noqa: E731
    rpd, cid, cpd, rid = dev(rp), dev(ci), dev(cp), dev(ri)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    O, L = bsa.forward(qd, kd, vd, rpd, cid, bs, scale, causal)
    dq, dk, dv = bsa.backward(qd, kd, vd, O, dod, L, rpd, cid, cpd, rid, bs, scale, causal)
    torch.cuda.synchronize()
    assert bsa.device_status(clear=True) == 0
    assert bsa.backward_status(clear=True) == 0
    ref = obw.backward(q, k, v, do, rp, ci, bs, scale, causal)
    for name, got, want in (("dQ", dq, ref[0]), ("dK", dk, ref[1]), ("dV", dv, ref[2])):
        g_ = got.float().cpu().numpy()
        assert np.isfinite(g_).all(), name
        err = np.abs(g_ - want)
        scale_max = max(np.abs(want).max(), 1e-6)
        scale_mean = max(np.abs(want).mean(), 1e-6)
        assert err.max() <= 2e-2 * scale_max, (name, err.max(), scale_max)
        assert err.mean() <= 1e-2 * scale_mean, (name, err.mean(), scale_mean)


# (B, H, N, d, bs, density, causal)
CASES = [
    (1, 2, 256, 64, 32, 0.4, False),
    (1, 2, 256, 128, 64, 0.5, True),
    (2, 1, 512, 128, 128, 0.5, False),
    (1, 2, 512, 64, 64, 0.3, False),
    (1, 1, 384, 64, 32, 1.0, True),
    (2, 2, 256, 128, 32, 0.5, False),
    (1, 1, 256, 64, 128, 1.0, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}N{}d{}bs{}p{}c{}".format(*c))
def test_random_masks(case):
    B, H, N, d, bs, density, causal = case
    rng = np.random.default_rng(N + d + bs)
    # random block masks, future blocks included, one empty row (h = 0, last row)
    _, _, _, _, rp, ci = _rand_case(rng, 1, H, N, 8, bs, density)
    _run(B, H, N, d, bs, rp, ci, causal, seed=B * N + d)


def test_causal_loglinear_pattern():
    B, H, N, d, bs = 1, 4, 1024, 128, 64
    M = N // bs
    rp, ci = bsa.build_pattern(bsa.LOGLINEAR, M, H, local_radius=1, log_kmax=3,
                               anchors=(0, M // 2, M - 1), causal=True)
    _run(B, H, N, d, bs, rp, ci, True, seed=7)


def test_tiny_loglinear_workload():
    w = workloads.WORKLOADS["tiny_loglinear"]
    rp, ci = bsa.build_pattern_from(w.pattern)
    _run(w.B, w.H, w.N, w.d, w.block_size, rp, ci, w.causal, seed=w.seed)


def _check_grads(got_list, ref_list, what):
    for name, got, want in zip(("dQ", "dK", "dV"), got_list, ref_list):
        g_ = np.asarray(got, dtype=np.float64)
        assert np.isfinite(g_).all(), (what, name)
        err = np.abs(g_ - want)
        scale_max = max(np.abs(want).max(), 1e-6)
        scale_mean = max(np.abs(want).mean(), 1e-6)
        assert err.max() <= 2e-2 * scale_max, (what, name, err.max(), scale_max)
        assert err.mean() <= 1e-2 * scale_mean, (what, name, err.mean(), scale_mean)


@pytest.mark.parametrize("name,branch", [("bernoulli_4k", "index"), ("local_global_8k", "sorted")])
def test_full_size_backward(name, branch):
    """The full workload in one backward launch (the bench's), compared on
    sampled (b, h) with the oracle.  bernoulli_4k (4096 tiles of even cost)
    runs its tiles in index order; local_global_8k (tiles of the global rows
    and columns far above the mean) in heavy-first order: the tile orders in
    the workspace show which branch ran."""
    w = workloads.WORKLOADS[name]
    B, H, N, d, bs = w.B, w.H, w.N, w.d, w.block_size
    q, k, v = workloads.make_qkv(w)
    g = torch.Generator().manual_seed(w.seed + 77)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    rp, ci = bsa.build_pattern_from(w.pattern)
    cp, ri = bsa.transpose_pattern(rp, ci, H, w.M)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(DEV)  # noqa: E731
    rpd, cid, cpd, rid = dev(rp), dev(ci), dev(cp), dev(ri)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    O, L = bsa.forward(qd, kd, vd, rpd, cid, bs, w.scale, w.causal)
    nbytes = bsa.library().bsa_backward_workspace_bytes(B, H, N)
    ws = torch.empty(nbytes // 4, dtype=torch.float32, device=DEV)
    dq, dk, dv = bsa.backward(qd, kd, vd, O, dod, L, rpd, cid, cpd, rid, bs, w.scale, w.causal,
                              workspace=ws)
    torch.cuda.synchronize()
    assert bsa.device_status(clear=True) == 0
    assert bsa.backward_status(clear=True) == 0

    rows, T = B * H * N, B * H * (N // 128)
    words = ws.view(torch.int32).cpu().numpy()
    cost = words[rows:rows + 2 * T]
    order = words[rows + 2 * T:rows + 4 * T]
    for half in range(2):
        o = order[half * T:(half + 1) * T]
        c = cost[half * T:(half + 1) * T]
        assert np.array_equal(np.sort(o), np.arange(T))
        if branch == "index":
            assert np.array_equal(o, np.arange(T))
        else:
            assert np.all(np.diff(c[o]) <= 0) and not np.array_equal(o, np.arange(T))

    rng = np.random.default_rng(0)
    pairs = {(0, 0), (B - 1, H - 1), (int(rng.integers(B)), int(rng.integers(H)))}
    got = [t.float().cpu().numpy() for t in (dq, dk, dv)]
    M = w.M
    for b, h in sorted(pairs):
        rph = (rp[h * M:(h + 1) * M + 1] - rp[h * M]).astype(np.int32)
        cih = ci[rp[h * M]:rp[(h + 1) * M]]
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = obw.backward(q[sl], k[sl], v[sl], do[sl], rph, cih, bs, w.scale, w.causal)
        _check_grads([x[b, h] for x in got], [r[0, 0] for r in ref], f"{name} b{b} h{h}")

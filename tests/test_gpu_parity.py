"""GPU parity: bsa_forward (through the C ABI) against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation): O max-abs <= 2e-2 and mean-abs
<= 2e-3, LSE abs <= 1e-3, and -inf exactly where the oracle has no key.
The block-CSR itself is compared bit for bit with the oracle's enumeration.

Small cases compare every output; the full-size workloads (the same single
launch the benchmark times) compare every row the oracle computes in seconds:
a whole head plus random rows of every head, and the global-anchor rows.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_38_b200 as bsa
import oracle
from oracle import patterns
import workloads

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


def _dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def _compare(O_gpu, L_gpu, O_ref, L_ref, what=""):
    O_gpu = np.asarray(O_gpu, dtype=np.float64)
    L_gpu = np.asarray(L_gpu, dtype=np.float64)
    assert O_gpu.shape == O_ref.shape and L_gpu.shape == L_ref.shape
    err = np.abs(O_gpu - O_ref)
    assert np.isfinite(O_gpu).all(), f"{what}: non-finite O"
    assert err.max() <= O_MAX, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: O mean-abs {err.mean():.3e}"
    ninf_ref = np.isneginf(L_ref)
    assert np.array_equal(np.isneginf(L_gpu), ninf_ref), f"{what}: -inf LSE pattern differs"
    fin = ~ninf_ref
    if fin.any():
        lerr = np.abs(L_gpu[fin] - L_ref[fin]).max()
        assert lerr <= LSE_ABS, f"{what}: LSE abs {lerr:.3e}"
    assert np.all(O_gpu[ninf_ref] == 0.0)
    return float(err.max()), float(err.mean())


def _run_gpu(q, k, v, rp, ci, bs, scale, causal):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    rpd, cid = _dev(rp, ci if ci.size else np.zeros(1, np.int32))
    O, L = bsa.forward(qd, kd, vd, rpd, cid, bs, scale, causal)
    torch.cuda.synchronize()
    return O.float().cpu().numpy(), L.cpu().numpy()


def _sample_rows(w, rng, n_random):
    B, H, N = w.B, w.H, w.N
    rows = set(range(N))                                   # all of (b=0, h=0)
    last = ((B - 1) * H + (H - 1)) * N
    rows.update(range(last, last + N))                     # all of the last head
    rows.update(int(x) for x in rng.integers(0, B * H * N, n_random))
    for bh in range(B * H):                                # first and last row of every head
        rows.add(bh * N)
        rows.add(bh * N + N - 1)
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name", workloads.ORDER + workloads.EXTRA_ORDER)
def test_workload_parity(name):
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.make_qkv(w)
    rp, ci = bsa.build_pattern_from(w.pattern)
    orp, oci = patterns.csr(w.pattern)
    assert np.array_equal(rp, orp) and np.array_equal(ci, oci)  # CSR bit-exact
    O, L = _run_gpu(q, k, v, rp, ci, w.block_size, w.scale, w.causal)
    assert bsa.device_status(clear=True) == 0
    flops_full = 4.0 * w.block_size * w.d * len(ci) * w.block_size * w.B
    if flops_full < 2e10:
        Or, Lr, _ = oracle.forward(q, k, v, orp, oci, w.block_size, w.scale, w.causal)
        _compare(O, L, Or, Lr, name)
    else:
        rows = _sample_rows(w, np.random.default_rng(0), 4096)
        Or, Lr, _ = oracle.forward(q, k, v, orp, oci, w.block_size, w.scale, w.causal, rows=rows)
        _compare(O.reshape(-1, w.d)[rows], L.reshape(-1)[rows], Or, Lr, name)


def _random_csr(rng, H, M, density, causal, shuffle=False, dup=False, empty_rows=0):
    rows = []
    for h in range(H):
        for i in range(M):
            cols = [j for j in range(M) if rng.random() < density]
            if causal:
                cols = [j for j in cols if j <= i]
            rows.append(cols)
    for r in rng.choice(H * M, size=min(empty_rows, H * M), replace=False):
        rows[int(r)] = []
    if shuffle:
        for r in rows:
            rng.shuffle(r)
    if dup:
        rows = [r + r[:1] for r in rows]
    rp = np.zeros(H * M + 1, np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([j for r in rows for j in r], np.int32)
    return rp, ci


SHAPES = [
    # B, H, N, d, bs   (N not a multiple of 128 gives a ragged last tile for bs < 128)
    (1, 1, 32, 64, 32),
    (1, 2, 96, 64, 32),
    (2, 3, 224, 128, 32),
    (1, 2, 192, 64, 64),
    (2, 1, 320, 128, 64),
    (1, 2, 128, 64, 128),
    (2, 2, 384, 128, 128),
    (1, 1, 1024, 64, 32),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}N{}d{}bs{}".format(*s))
def test_random_patterns(shape, causal):
    B, H, N, d, bs = shape
    M = N // bs
    rng = np.random.default_rng(abs(hash((shape, causal))) % (1 << 31))
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=int(rng.integers(1 << 30)),
                                       key_scale_max=3.0)
    rp, ci = _random_csr(rng, H, M, 0.35, causal, shuffle=True, dup=True, empty_rows=2)
    scale = 1.0 / math.sqrt(d)
    O, L = _run_gpu(q, k, v, rp, ci, bs, scale, causal)
    assert bsa.device_status(clear=True) == 0
    Or, Lr, _ = oracle.forward(q, k, v, rp, ci, bs, scale, causal)
    _compare(O, L, Or, Lr, str(shape))


@pytest.mark.parametrize("scale", [-0.2, 0.0, 0.7])
@pytest.mark.parametrize("shape", [(1, 2, 256, 64, 32), (1, 2, 384, 128, 64), (1, 2, 512, 128, 128)],
                         ids=lambda s: "B{}H{}N{}d{}bs{}".format(*s))
def test_negative_zero_and_large_scale(shape, scale):
    # the kernel is specialised on the sign of the scale (maximum or minimum
    # of the raw scores); scale 0 gives uniform weights over the allowed keys
    B, H, N, d, bs = shape
    M = N // bs
    rng = np.random.default_rng(int(abs(scale) * 1000) + N)
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=int(rng.integers(1 << 30)))
    for causal in (False, True):
        rp, ci = _random_csr(rng, H, M, 0.5, causal, shuffle=False, dup=False, empty_rows=1)
        O, L = _run_gpu(q, k, v, rp, ci, bs, scale, causal)
        assert bsa.device_status(clear=True) == 0
        Or, Lr, _ = oracle.forward(q, k, v, rp, ci, bs, scale, causal)
        _compare(O, L, Or, Lr, f"{shape} scale={scale} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [32, 64, 128])
def test_many_tiles_per_cta_varying_row_lengths(bs, d):
    # more tiles than SMs, so every CTA walks several tiles and reuses its
    # rings and buffers; band edges and random rows give many partial chunks
    B, H, N = 1, 16, 4096 if bs == 32 else 8192
    M = N // bs
    rng = np.random.default_rng(bs * 1000 + d)
    rows = []
    for h in range(H):
        for i in range(M):
            w = int(rng.integers(0, 4))
            cols = [j for j in range(i - w, i + w + 1) if 0 <= j < M]
            cols += [int(x) for x in rng.integers(0, M, int(rng.integers(0, 6)))]
            rows.append(sorted(set(cols)))
    rp = np.zeros(H * M + 1, np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([j for r in rows for j in r], np.int32)
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=bs + d)
    O, L = _run_gpu(q, k, v, rp, ci, bs, 1.0 / math.sqrt(d), False)
    assert bsa.device_status(clear=True) == 0
    rows_s = np.unique(np.concatenate([np.arange(0, 2 * N), rng.integers(0, B * H * N, 4096)]))
    Or, Lr, _ = oracle.forward(q, k, v, rp, ci, bs, 1.0 / math.sqrt(d), False, rows=rows_s)
    _compare(O.reshape(-1, d)[rows_s], L.reshape(-1)[rows_s], Or, Lr, f"bs={bs} d={d}")


@pytest.mark.parametrize("bs,d", [(64, 128), (32, 64)])
def test_many_global_rows_exercise_the_heavy_tile_schedule(bs, d):
    # local+global with six full rows per head: tiles holding a global row
    # cost many times the others, so they are dealt out one per CTA first and
    # those CTAs sit out the first rounds of the other tiles; every output row
    # is compared
    B, H, N = 2, 4, 4096
    M = N // bs
    desc = workloads.PatternDesc(kind=workloads.LOCAL_GLOBAL, M=M, H=H, local_radius=2,
                                 anchors=(0, 5, M // 3, M // 2, M - 7, M - 1))
    rp, ci = patterns.csr(desc)
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=bs + 7 * d, key_scale_max=3.0)
    O, L = _run_gpu(q, k, v, rp, ci, bs, 1.0 / math.sqrt(d), False)
    assert bsa.device_status(clear=True) == 0
    Or, Lr, _ = oracle.forward(q, k, v, rp, ci, bs, 1.0 / math.sqrt(d), False)
    _compare(O, L, Or, Lr, f"local_global bs={bs} d={d}")


def test_all_rows_empty():
    B, H, N, d, bs = 1, 2, 256, 64, 32
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=5)
    rp = np.zeros(H * (N // bs) + 1, np.int32)
    O, L = _run_gpu(q, k, v, rp, np.zeros(0, np.int32), bs, 0.125, False)
    assert np.all(O == 0.0) and np.all(np.isneginf(L))


@pytest.mark.parametrize("bs,d,N", [(32, 64, 1024), (32, 128, 2048), (64, 128, 512), (128, 64, 1024)])
def test_dense_pattern_large_logits_and_causal(bs, d, N):
    # every block present, K scaled up: the running max moves often and far.
    # At block_size 32 a row of 32+ blocks spans several TMEM-resident groups
    # of chunks, so the rescaling between groups is exercised too.
    B, H = 1, 2
    M = N // bs
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=8 + bs)
    k = (k.float() * 6).to(torch.bfloat16)
    rp = np.arange(0, H * M * M + 1, M, dtype=np.int32)
    ci = np.tile(np.arange(M, dtype=np.int32), H * M)
    for causal in (False, True):
        O, L = _run_gpu(q, k, v, rp, ci, bs, 1.0 / math.sqrt(d), causal)
        assert bsa.device_status(clear=True) == 0
        Or, Lr, _ = oracle.forward(q, k, v, rp, ci, bs, 1.0 / math.sqrt(d), causal)
        _compare(O, L, Or, Lr, f"dense bs={bs} causal={causal}")
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.float(), k.float(), v.float(), is_causal=causal, scale=1.0 / math.sqrt(d))
        assert float((torch.from_numpy(O) - ref).abs().max()) <= O_MAX


def test_out_of_range_columns_are_skipped_and_flagged():
    B, H, N, d, bs = 1, 1, 256, 64, 64
    M = N // bs
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=9)
    rp = np.array([0, 3, 5, 7, 9], np.int32)
    ci = np.array([0, 9, 1, -4, 1, 2, 100, 3, 2], np.int32)
    bsa.device_status(clear=True)
    O, L = _run_gpu(q, k, v, rp, ci, bs, 0.125, False)
    assert bsa.device_status(clear=True) & bsa.STATUS_BAD_COLUMN
    keep = (ci >= 0) & (ci < M)
    rows = np.repeat(np.arange(len(rp) - 1), np.diff(rp))
    rp2 = np.zeros_like(rp)
    rp2[1:] = np.cumsum(np.bincount(rows[keep], minlength=len(rp) - 1))
    Or, Lr, _ = oracle.forward(q, k, v, rp2, ci[keep], bs, 0.125, False)
    _compare(O, L, Or, Lr, "bad columns")


def test_largest_supported_M():
    # M = 4096 block rows (N = 131072 at block_size 32), a log-linear pattern
    B, H, N, d, bs = 1, 1, 131072, 64, 32
    M = N // bs
    desc = workloads.PatternDesc(kind=workloads.LOGLINEAR, M=M, H=H, log_kmax=11,
                                 anchors=(0, M // 2, M - 1))
    rp, ci = bsa.build_pattern_from(desc)
    q, k, v = workloads.make_qkv_shape(B, H, N, d, seed=10)
    O, L = _run_gpu(q, k, v, rp, ci, bs, 0.125, False)
    assert bsa.device_status(clear=True) == 0
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(N - 64, N),
                                     np.random.default_rng(1).integers(0, N, 512)]))
    Or, Lr, _ = oracle.forward(q, k, v, rp, ci, bs, 0.125, False, rows=rows)
    _compare(O.reshape(-1, d)[rows], L.reshape(-1)[rows], Or, Lr, "M=4096")


def test_repeated_calls_are_deterministic_and_stream_ordered():
    w = workloads.WORKLOADS["loglinear_4k"]
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    rp, ci = _dev(*bsa.build_pattern_from(w.pattern))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        O1, L1 = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale)
        O2, L2 = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale)
    s.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)

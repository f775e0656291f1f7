"""Seeded synthetic workloads for the block-sparse attention forward.

This module is shared by the CUDA path's tests and benchmark and by the
oracle's tests.  It holds only workload *descriptions* (shapes, pattern
parameters, seeds) and the seeded random draws of Q, K and V.  It contains
none of the method's arithmetic: no pattern enumeration, no softmax, no
attention.

Workload recipe (stands in for the long-text corpora the pages measure on,
which are not needed to exercise the kernel):

* ``torch.Generator('cpu').manual_seed(seed)``; Q, then K, then V are drawn
  as fp32 ``randn`` of shape [B, H, N, d] and cast to bf16 (round to nearest
  even).
* The local+global workload additionally draws ``u ~ U(0, 3)`` of shape
  [B, H, N, 1] after V from the same generator and uses
  ``K = (K_fp32 * (1 + u)).to(bf16)`` to widen the logit range.
* ``scale = 1/sqrt(d)``.

The five workloads follow the block-sparse attention pages: the log-linear
pattern of "Block Sparse Attention with Log-Linear Complexity" (section 3.1,
local + log-stride + 3 global anchor blocks), the Local+Global band of the
SparseFlashAttention article (sections "Local + Global" and "Block-Sparse"),
and the Bernoulli block mask of the RTX 4090 article ("core implementation
logic", step 1).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

# Pattern kinds; the numeric values are the ones of the C-ABI enum bsa_kind.
LOGLINEAR = 0
LOCAL_GLOBAL = 1
BERNOULLI = 2
SLIDING_WINDOW = 3
BIGBIRD = 4
TOPK = 5  # chosen on the device from Q and K (not a host-builder kind)

KIND_NAMES = {LOGLINEAR: "loglinear", LOCAL_GLOBAL: "local_global", BERNOULLI: "bernoulli",
              SLIDING_WINDOW: "sliding_window", BIGBIRD: "bigbird", TOPK: "topk"}


@dataclasses.dataclass(frozen=True)
class PatternDesc:
    """Plain description of a block pattern (mirrors the C struct bsa_pattern_desc)."""

    kind: int
    M: int                      # block rows = block columns = N / block_size
    H: int                      # heads (Bernoulli differs per head; others repeat)
    local_radius: int = 1       # LOGLINEAR: |i-j| <= radius; LOCAL_GLOBAL: band half-width w
    log_kmax: int = 0           # LOGLINEAR: strides 2^k for k = 0..log_kmax
    anchors: Tuple[int, ...] = ()  # LOGLINEAR: anchor columns; LOCAL_GLOBAL: full rows + columns
    p: float = 0.0              # BERNOULLI keep probability
    seed: int = 0               # BERNOULLI counter-based generator seed
    causal: bool = False        # keep only columns j <= i
    dilation: int = 1           # SLIDING_WINDOW: keep j with (i - j) % dilation == 0
    num_random: int = 0         # BIGBIRD: random columns drawn per block row
    top_k: int = 0              # TOPK: blocks kept per row besides the diagonal


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    block_size: int
    pattern: PatternDesc
    seed: int
    key_scale_max: float = 0.0  # >0: K rows scaled by 1 + U(0, key_scale_max)
    causal: bool = False        # token-level causal masking in the forward

    @property
    def M(self) -> int:
        return self.N // self.block_size

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


def _loglinear(M: int, H: int, kmax: int, causal: bool = False) -> PatternDesc:
    return PatternDesc(kind=LOGLINEAR, M=M, H=H, local_radius=1, log_kmax=kmax,
                       anchors=(0, M // 2, M - 1), causal=causal)


WORKLOADS = {
    # B=1 H=2 N=256 d=64 bs=32: strides k=0..2, anchors {0,4,7}
    "tiny_loglinear": Workload("tiny_loglinear", 1, 2, 256, 64, 32, _loglinear(8, 2, 2), seed=0),
    # B=1 H=16 N=4096 d=64 bs=32: strides k=0..6, anchors {0,64,127}
    "loglinear_4k": Workload("loglinear_4k", 1, 16, 4096, 64, 32, _loglinear(128, 16, 6), seed=1),
    # B=2 H=16 N=8192 d=128 bs=64: band w=4 blocks + full rows/cols 0 and M-1
    "local_global_8k": Workload(
        "local_global_8k", 2, 16, 8192, 128, 64,
        PatternDesc(kind=LOCAL_GLOBAL, M=128, H=16, local_radius=4, anchors=(0, 127)),
        seed=2, key_scale_max=3.0),
    # B=16 H=8 N=4096 d=64 bs=64: Bernoulli(0.3) per (h, i, j), seed 7, diagonal forced
    "bernoulli_4k": Workload(
        "bernoulli_4k", 16, 8, 4096, 64, 64,
        PatternDesc(kind=BERNOULLI, M=64, H=8, p=0.3, seed=7), seed=3),
    # B=1 H=32 N=32768 d=128 bs=128: causal log-linear, strides k=0..7, anchors {0,128,255}
    "causal_loglinear_32k": Workload(
        "causal_loglinear_32k", 1, 32, 32768, 128, 128, _loglinear(256, 32, 7, causal=True),
        seed=4, causal=True),
}

# The same five workloads in the order they are usually listed.
ORDER = ["tiny_loglinear", "loglinear_4k", "local_global_8k", "bernoulli_4k", "causal_loglinear_32k"]

# The other pattern kinds of the pages, on shapes of the same scale (the
# kernel is the same; only the block-CSR differs):
#  - dilated sliding window: 512 tokens each side at block 64 (8 blocks),
#    every second block (the SparseFlashAttention article's example);
#  - BigBird: 3-block window, block 0 global, 3 random blocks per row, block 64
#    (the same article's example; random blocks drawn per head);
#  - log-linear with seven anchors instead of three ("Block Sparse Attention
#    with Log-Linear Complexity", section 6.1).
EXTRA = {
    "sliding_window_8k": Workload(
        "sliding_window_8k", 1, 16, 8192, 128, 64,
        PatternDesc(kind=SLIDING_WINDOW, M=128, H=16, local_radius=8, dilation=2), seed=5),
    "bigbird_4k": Workload(
        "bigbird_4k", 2, 16, 4096, 64, 64,
        PatternDesc(kind=BIGBIRD, M=64, H=16, local_radius=1, anchors=(0,), num_random=3, seed=11),
        seed=6),
    "loglinear7_4k": Workload(
        "loglinear7_4k", 1, 16, 4096, 64, 32,
        PatternDesc(kind=LOGLINEAR, M=128, H=16, local_radius=1, log_kmax=6,
                    anchors=(0, 8, 32, 64, 96, 120, 127)), seed=7),
}
WORKLOADS.update(EXTRA)
EXTRA_ORDER = list(EXTRA)

# Content-based selection: each block row of each (b, h) keeps its diagonal
# and the top_k blocks of highest mean-Q . mean-K score, chosen on the device
# (20 % of the row, the RTX 4090 article's "topk = 20%").
TOPK_WORKLOADS = {
    "topk_4k": Workload(
        "topk_4k", 1, 16, 4096, 64, 32,
        PatternDesc(kind=TOPK, M=128, H=16, top_k=25), seed=8),
}
WORKLOADS.update(TOPK_WORKLOADS)


def make_qkv(w: Workload, seed: Optional[int] = None):
    """Draw bf16 Q, K, V of shape [B, H, N, d] on the CPU from the workload's seed."""
    import torch

    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.N, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k32 = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    if w.key_scale_max > 0:
        u = torch.rand((w.B, w.H, w.N, 1), generator=g, dtype=torch.float32) * w.key_scale_max
        k32 = k32 * (1.0 + u)
    k = k32.to(torch.bfloat16)
    return q.contiguous(), k.contiguous(), v.contiguous()


def make_qkv_shape(B: int, H: int, N: int, d: int, seed: int, key_scale_max: float = 0.0):
    """Seeded bf16 Q, K, V for an arbitrary shape (random-shape parity sweeps)."""
    w = Workload("adhoc", B, H, N, d, 32, PatternDesc(kind=LOGLINEAR, M=1, H=H), seed=seed,
                 key_scale_max=key_scale_max)
    return make_qkv(w)



# ---------------------------------------------------------------- decode
# One decode step per (b, h): a new query token at position seq_len[b] - 1
# attends to the cached tokens of the blocks its block row lists (the KV
# cache in the (B, H, L, D) layout of "Block Sparse Attention with Log-Linear
# Complexity", section 5.1).  The cache holds L tokens of room; seq_len draws
# a ragged batch of filled lengths.

@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    L: int                  # cache capacity in tokens
    d: int
    block_size: int
    pattern: PatternDesc    # over M = L // block_size block rows
    seed: int
    min_len: int            # seq_len[b] drawn uniformly from [min_len, L]
    append: bool = True     # the step writes the new token's k and v into the cache

    @property
    def M(self) -> int:
        return self.L // self.block_size

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


DECODE_WORKLOADS = {
    # 8 sequences of 16K-32K tokens, 32 heads, d=128, block 128: the causal
    # log-linear pattern of causal_loglinear_32k (strides k=0..7, anchors
    # {0,128,255}) read by one new token per (b, h)
    "decode_loglinear_32k": DecodeWorkload(
        "decode_loglinear_32k", 8, 32, 32768, 128, 128, _loglinear(256, 32, 7, causal=True),
        seed=9, min_len=16384),
    # a small one for parity: 4 sequences of 1..4096 tokens, block 32, d=64
    "decode_loglinear_4k": DecodeWorkload(
        "decode_loglinear_4k", 4, 16, 4096, 64, 32, _loglinear(128, 16, 6, causal=True),
        seed=10, min_len=1),
}


def make_decode_inputs(w: DecodeWorkload, device="cpu", seed: Optional[int] = None):
    """Seeded decode inputs on `device` (a torch generator of that device).

    Draw order: seq_len [B] int32 uniform in [min_len, L]; q, k_new, v_new
    [B, H, d]; then the K cache and the V cache [B, H, L, d], one batch entry
    at a time; all fp32 randn cast to bf16.  Cache rows at and beyond
    seq_len[b] - 1 hold random values too (stale entries of a reused cache).
    Returns (q, k_new, v_new, k_cache, v_cache, seq_len).
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    lens = torch.randint(w.min_len, w.L + 1, (w.B,), generator=g, device=device,
                         dtype=torch.int64).to(torch.int32)

    def bf16(shape):
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)

    q = bf16((w.B, w.H, w.d))
    k_new = bf16((w.B, w.H, w.d))
    v_new = bf16((w.B, w.H, w.d))
    caches = []
    for _ in range(2):
        c = torch.empty((w.B, w.H, w.L, w.d), dtype=torch.bfloat16, device=device)
        for b in range(w.B):
            c[b] = bf16((w.H, w.L, w.d))
        caches.append(c)
    return q, k_new, v_new, caches[0], caches[1], lens

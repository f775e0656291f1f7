"""GPU parity of top-k block selection and of the forward on its pattern.

The selected CSR must equal the oracle's bit for bit: both sides compute the
block means and scores in fp64 in the same order (see oracle/topk.py), so the
integer decisions agree.  The forward then runs on the batch folded into the
heads and is compared with the fp64 oracle within the usual tolerances.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_38_b200 as bsa
import oracle
from oracle import topk
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bsa.library()
    bsa.device_status(clear=True)
    yield


CASES = [
    # B, H, N, d, bs, top_k, causal
    (1, 2, 256, 64, 32, 2, False),
    (2, 2, 512, 64, 32, 5, True),
    (1, 3, 1024, 128, 64, 4, False),
    (2, 1, 1024, 128, 128, 3, True),
    (1, 2, 4096, 64, 32, 25, False),   # 20 % of 128 blocks
    (1, 1, 64, 64, 64, 0, False),      # M = 1
    (1, 1, 512, 64, 32, 100, True),    # top_k beyond the row: every allowed block
    # more heads and rows; M = 120 and 60 pad the sort to 128 and 64 entries
    (1, 12, 3840, 64, 32, 10, True),
    (2, 5, 2048, 64, 32, 7, False),
    (1, 5, 3840, 128, 64, 3, True),
    # the largest row one warp selects (1024 candidates), and a longer one
    # that takes the one-CTA-per-row kernel (2048)
    (1, 1, 32768, 64, 32, 50, False),
    (1, 1, 65536, 64, 32, 20, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}N{}d{}bs{}k{}c{}".format(*c))
def test_topk_csr_bit_exact_and_forward_parity(case):
    B, H, N, d, bs, k, causal = case
    q, kk, v = workloads.make_qkv_shape(B, H, N, d, seed=N + d + k)
    rp_d, ci_d = bsa.topk_pattern(q.cuda(), kk.cuda(), bs, k, causal)
    torch.cuda.synchronize()
    rp, ci = rp_d.cpu().numpy(), ci_d.cpu().numpy()
    orp, oci = topk.topk_pattern(q.float().numpy(), kk.float().numpy(), bs, k, causal)
    assert np.array_equal(rp, orp)
    assert np.array_equal(ci, oci)
    # forward on the selected pattern, batch folded into the heads
    qf, kf, vf = (t.reshape(1, B * H, N, d).contiguous() for t in (q, kk, v))
    O, L = bsa.forward(qf.cuda(), kf.cuda(), vf.cuda(), rp_d, ci_d, bs, 1.0 / math.sqrt(d), causal)
    torch.cuda.synchronize()
    assert bsa.device_status(clear=True) == 0
    Or, Lr, _ = oracle.forward(qf, kf, vf, orp, oci, bs, 1.0 / math.sqrt(d), causal)
    err = np.abs(O.float().cpu().numpy() - Or)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert np.abs(L.cpu().numpy() - Lr).max() <= 1e-3


@pytest.mark.parametrize("N,bs", [(4096, 32), (65536, 32)])
def test_topk_ties_go_to_the_smaller_column(N, bs):
    """Constant K: every candidate of a row scores the same, so the row keeps
    its smallest allowed columns -- in both selection kernels."""
    B, H, d, k, causal = 1, 2, 64, 7, False
    q, _, _ = workloads.make_qkv_shape(B, H, N, d, seed=5)
    kk = torch.ones_like(q)
    rp_d, ci_d = bsa.topk_pattern(q.cuda(), kk.cuda(), bs, k, causal)
    torch.cuda.synchronize()
    orp, oci = topk.topk_pattern(q.float().numpy(), kk.float().numpy(), bs, k, causal)
    assert np.array_equal(rp_d.cpu().numpy(), orp)
    assert np.array_equal(ci_d.cpu().numpy(), oci)

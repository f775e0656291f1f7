"""bsa_topk_pattern_static, the allocation-free top-k selection.

The entry point takes its fp64 workspace from a static scratch array of the
library rather than from the caller.  The GPU test compares it with
bsa_topk_pattern (caller workspace) on two different calls in a row, so the
second call runs over the scratch the first one left behind; it must give
identical bits and must not change the device's free memory.  The file is
named to be collected last and passes on its own as well.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import block_sparse_attention_38_b200 as bsa
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_python_limit_matches_the_header():
    text = open(os.path.join(ROOT, "include", "bsa.h")).read()
    m = re.search(r"#define BSA_TOPK_STATIC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", text)
    assert m, "limit macro not found"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == bsa.TOPK_STATIC_SCRATCH_BYTES


def test_oversize_and_bad_arguments_are_rejected_before_any_cuda_call():
    # No pointer is dereferenced: every case below fails the host checks.
    lib = bsa.library()
    fake = ctypes.c_void_p(256)
    f = lib.bsa_topk_pattern_static
    # 2 * 64 * 128 * 128 * 8 bytes = 16 MiB of workspace > 4 MiB
    assert f(fake, fake, 64, 4096, 128, 32, 8, 0, fake, fake, None) == bsa.ERR_BUFFER_TOO_SMALL
    # just above the limit: BH * M * d = 1 * 4096 * 65 = 266240 > 262144
    assert f(fake, fake, 1, 4096, 65, 1, 8, 0, fake, fake, None) == bsa.ERR_BUFFER_TOO_SMALL
    assert f(fake, None, 16, 4096, 128, 32, 8, 0, fake, fake, None) == bsa.ERR_INVALID_ARG
    assert f(fake, fake, 1, 4096, 64, 48, 8, 0, fake, fake, None) == bsa.ERR_INVALID_ARG
    assert f(fake, fake, 1, 4096, 300, 32, 8, 0, fake, fake, None) == bsa.ERR_UNSUPPORTED
    assert f(fake, fake, 1, 4096, 64, 32, -1, 0, fake, fake, None) == bsa.ERR_INVALID_ARG
    assert f(fake, fake, 1, 4096, 64, 32, 8, 2, fake, fake, None) == bsa.ERR_INVALID_ARG


def _qk(B, H, N, d, seed, dev):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).to(dev)
    return q, k


# (B, H, N, d, bs, top_k, causal): the topk_4k workload (2 MiB of scratch),
# then a smaller causal case with another layout over the same scratch.
CASES = [
    (1, 16, 4096, 64, 32, 25, False),
    (2, 3, 1024, 128, 64, 5, True),
]


@pytest.mark.gpu
def test_static_scratch_matches_the_workspace_entry_on_calls_in_a_row():
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workloads.WORKLOADS["topk_4k"]
    assert (w.B, w.H, w.N, w.d, w.block_size, w.pattern.top_k) == CASES[0][:6]
    seen = []
    for case_no, (B, H, N, d, bs, top_k, causal) in enumerate(CASES):
        BH, M = B * H, N // bs
        nnz = bsa.topk_nnz(BH, M, top_k, causal)
        rp = torch.full((BH * M + 1,), -7, dtype=torch.int32, device=dev)
        ci = torch.full((nnz,), -7, dtype=torch.int32, device=dev)
        for call, seed in enumerate((100 + 2 * case_no, 101 + 2 * case_no)):
            q, k = _qk(B, H, N, d, seed, dev)
            want_rp, want_ci = bsa.topk_pattern(q, k, bs, top_k, causal)
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info(dev)[0]
            got_rp, got_ci = bsa.topk_pattern_static(q, k, bs, top_k, causal, rp, ci)
            torch.cuda.synchronize()
            if case_no or call:  # after the first call has set the scratch up
                assert torch.cuda.mem_get_info(dev)[0] == free_before
            assert torch.equal(got_rp, want_rp), (case_no, call)
            assert torch.equal(got_ci, want_ci), (case_no, call)
            seen.append(got_ci.cpu().numpy().copy())
        # the two calls of a case chose different blocks: the second did not
        # reuse the first's means
        assert not np.array_equal(seen[-1], seen[-2])
    assert bsa.device_status(clear=True) == 0


@pytest.mark.gpu
def test_oversize_request_leaves_the_outputs_untouched():
    dev = torch.device("cuda", 0)
    q, k = _qk(1, 64, 4096, 128, 5, dev)   # 16 MiB of workspace
    BH, M = 64, 128
    rp = torch.full((BH * M + 1,), -7, dtype=torch.int32, device=dev)
    ci = torch.full((bsa.topk_nnz(BH, M, 8, False),), -7, dtype=torch.int32, device=dev)
    with pytest.raises(bsa.BsaError) as e:
        bsa.topk_pattern_static(q, k, 32, 8, False, rp, ci)
    assert e.value.code == bsa.ERR_BUFFER_TOO_SMALL
    assert "static scratch" in str(e.value)
    torch.cuda.synchronize()
    assert bool((rp == -7).all()) and bool((ci == -7).all())

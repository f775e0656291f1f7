"""Host-side argument checks of bsa_decode (no GPU: every call below fails a
check made before any CUDA call, so the fake pointers are never used)."""
import ctypes

import pytest

import block_sparse_attention_38_b200 as bsa

P = ctypes.c_void_p(4096)  # 16-byte aligned, never dereferenced
P8 = ctypes.c_void_p(4104)  # 8 mod 16


def _call(**kw):
    args = dict(q=P, k_new=P, v_new=P, k_cache=P, v_cache=P, row_ptr=P, col_idx=P, seq_len=P,
                B=2, H=4, L=1024, d=128, bs=64, scale=0.125, O=P, LSE=P)
    args.update(kw)
    return bsa.library().bsa_decode(args["q"], args["k_new"], args["v_new"], args["k_cache"],
                                    args["v_cache"], args["row_ptr"], args["col_idx"],
                                    args["seq_len"], args["B"], args["H"], args["L"], args["d"],
                                    args["bs"], args["scale"], args["O"], args["LSE"], None)


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(k_cache=None), dict(v_cache=None), dict(row_ptr=None),
    dict(col_idx=None), dict(seq_len=None), dict(O=None), dict(LSE=None),
    dict(k_new=None),                 # v_new without k_new
    dict(v_new=None),                 # k_new without v_new
    dict(B=0), dict(H=0), dict(L=0), dict(d=0), dict(bs=0),
    dict(L=1000),                     # L % block_size != 0
    dict(scale=float("nan")), dict(scale=float("inf")),
    dict(q=P8), dict(k_cache=P8), dict(O=P8), dict(k_new=P8),
    dict(LSE=ctypes.c_void_p(4098)),  # LSE not 4-byte aligned
], ids=lambda kw: ",".join(f"{k}={v if not isinstance(v, ctypes.c_void_p) else v.value}"
                           for k, v in kw.items()))
def test_invalid_arguments(kw):
    assert _call(**kw) == bsa.ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [
    dict(d=96), dict(d=256), dict(bs=16), dict(bs=256, L=1024),
    dict(L=4097 * 32, bs=32),         # M = 4097 block rows
])
def test_unsupported_sizes(kw):
    assert _call(**kw) == bsa.ERR_UNSUPPORTED


def test_status_reader_rejects_null():
    assert bsa.library().bsa_decode_status(None, 0) == bsa.ERR_INVALID_ARG

"""B200 block-sparse attention forward: thin Python binding of libbsa.so.

Every step of the computation runs in the library's C++ host code and sm_100a
kernels; this module only marshals arguments (tensor pointers, sizes, the
current CUDA stream) and turns non-zero status codes into exceptions.  There
is no fallback: if libbsa.so is missing or fails to load, every call raises.

    import block_sparse_attention_38_b200 as bsa
    row_ptr, col_idx = bsa.build_pattern(bsa.LOGLINEAR, M=128, H=16, log_kmax=6,
                                         anchors=(0, 64, 127))
    O, LSE = bsa.forward(q, k, v, row_ptr_dev, col_idx_dev, block_size=32)

The C ABI is declared in include/bsa.h.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

# bsa_status
OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_BUFFER_TOO_SMALL = -3
ERR_BAD_PATTERN = -4
ERR_CUDA = -5
STATUS_NAMES = {OK: "BSA_OK", ERR_INVALID_ARG: "BSA_ERR_INVALID_ARG",
                ERR_UNSUPPORTED: "BSA_ERR_UNSUPPORTED",
                ERR_BUFFER_TOO_SMALL: "BSA_ERR_BUFFER_TOO_SMALL",
                ERR_BAD_PATTERN: "BSA_ERR_BAD_PATTERN", ERR_CUDA: "BSA_ERR_CUDA"}

# bsa_kind
LOGLINEAR = 0
LOCAL_GLOBAL = 1
BERNOULLI = 2
SLIDING_WINDOW = 3
BIGBIRD = 4

# device status bits
STATUS_TIMEOUT = 0x1
STATUS_BAD_COLUMN = 0x2
STATUS_BAD_ROW_PTR = 0x4
STATUS_BAD_SEQ_LEN = 0x8


class BsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


class _Desc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("M", ctypes.c_int32), ("H", ctypes.c_int32),
                ("local_radius", ctypes.c_int32), ("log_kmax", ctypes.c_int32),
                ("n_anchors", ctypes.c_int32), ("anchors", ctypes.POINTER(ctypes.c_int32)),
                ("p", ctypes.c_double), ("seed", ctypes.c_uint64), ("causal", ctypes.c_int32),
                ("dilation", ctypes.c_int32), ("num_random", ctypes.c_int32)]


_lib = None


def library() -> ctypes.CDLL:
    """The loaded libbsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m block_sparse_attention_38_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        lib.bsa_build_pattern.restype = ctypes.c_int
        lib.bsa_build_pattern.argtypes = [ctypes.POINTER(_Desc), vp, vp, i64,
                                          ctypes.POINTER(ctypes.c_int64)]
        lib.bsa_validate_pattern.restype = ctypes.c_int
        lib.bsa_validate_pattern.argtypes = [vp, vp, i64, i32, i32, i32]
        lib.bsa_forward.restype = ctypes.c_int
        lib.bsa_forward.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                    vp, vp, vp]
        lib.bsa_forward_workspace_bytes.restype = ctypes.c_size_t
        lib.bsa_forward_workspace_bytes.argtypes = [ctypes.c_int]
        lib.bsa_forward_ws.restype = ctypes.c_int
        lib.bsa_forward_ws.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                       vp, vp, vp, ctypes.c_size_t, vp]
        lib.bsa_device_status.restype = ctypes.c_int
        lib.bsa_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
        lib.bsa_version.restype = ctypes.c_int
        lib.bsa_version.argtypes = []
        lib.bsa_topk_nnz.restype = ctypes.c_int64
        lib.bsa_topk_nnz.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.bsa_topk_workspace_bytes.restype = ctypes.c_size_t
        lib.bsa_topk_workspace_bytes.argtypes = [ctypes.c_int] * 4
        lib.bsa_topk_pattern.restype = ctypes.c_int
        lib.bsa_topk_pattern.argtypes = [vp, vp] + [ctypes.c_int] * 6 + [vp, vp, vp,
                                                                          ctypes.c_size_t, vp]
        lib.bsa_transpose_pattern.restype = ctypes.c_int
        lib.bsa_transpose_pattern.argtypes = [vp, vp, i32, i32, vp, vp, i64,
                                              ctypes.POINTER(ctypes.c_int64)]
        lib.bsa_backward_workspace_bytes.restype = ctypes.c_size_t
        lib.bsa_backward_workspace_bytes.argtypes = [ctypes.c_int] * 3
        lib.bsa_backward.restype = ctypes.c_int
        lib.bsa_backward.argtypes = [vp] * 10 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int,
                                                                    vp, vp, vp, vp,
                                                                    ctypes.c_size_t, vp]
        lib.bsa_backward_status.restype = ctypes.c_int
        lib.bsa_backward_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
        lib.bsa_decode.restype = ctypes.c_int
        lib.bsa_decode.argtypes = [vp] * 8 + [ctypes.c_int] * 5 + [ctypes.c_float, vp, vp, vp]
        lib.bsa_decode_status.restype = ctypes.c_int
        lib.bsa_decode_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
        lib.bsa_topk_pattern_static.restype = ctypes.c_int
        lib.bsa_topk_pattern_static.argtypes = [vp, vp] + [ctypes.c_int] * 6 + [vp, vp, vp]
        _lib = lib
    return _lib


def _check(code: int, what: str) -> None:
    if code != OK:
        raise BsaError(code, what)


def build_pattern(kind: int, M: int, H: int, local_radius: int = 1, log_kmax: int = 0,
                  anchors: Sequence[int] = (), p: float = 0.0, seed: int = 0,
                  causal: bool = False, dilation: int = 1,
                  num_random: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Block-CSR of a pattern, built on the host by bsa_build_pattern.

    Returns (row_ptr int32 [H*M+1], col_idx int32 [nnz]) as numpy arrays.
    """
    lib = library()
    anc = np.ascontiguousarray(np.asarray(anchors, dtype=np.int32).reshape(-1))
    d = _Desc(int(kind), int(M), int(H), int(local_radius), int(log_kmax), int(anc.size),
              anc.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if anc.size else None,
              float(p), int(seed) & ((1 << 64) - 1), int(bool(causal)), int(dilation),
              int(num_random))
    nnz = ctypes.c_int64(0)
    _check(lib.bsa_build_pattern(ctypes.byref(d), None, None, 0, ctypes.byref(nnz)),
           "bsa_build_pattern")
    row_ptr = np.empty(int(H) * int(M) + 1, dtype=np.int32)
    col_idx = np.empty(max(int(nnz.value), 1), dtype=np.int32)
    _check(lib.bsa_build_pattern(ctypes.byref(d), row_ptr.ctypes.data, col_idx.ctypes.data,
                                 col_idx.size, ctypes.byref(nnz)), "bsa_build_pattern")
    return row_ptr, col_idx[: int(nnz.value)]


def build_pattern_from(desc) -> Tuple[np.ndarray, np.ndarray]:
    """build_pattern for any object with the bsa_pattern_desc field names."""
    return build_pattern(desc.kind, desc.M, desc.H, desc.local_radius, desc.log_kmax,
                         desc.anchors, desc.p, desc.seed, desc.causal,
                         getattr(desc, "dilation", 1), getattr(desc, "num_random", 0))


def validate_pattern(row_ptr: np.ndarray, col_idx: np.ndarray, H: int, M: int,
                     causal: bool = False) -> int:
    """Status code of bsa_validate_pattern for a host CSR (BSA_OK = 0)."""
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    if rp.size != int(H) * int(M) + 1:
        return ERR_INVALID_ARG
    return library().bsa_validate_pattern(rp.ctypes.data, ci.ctypes.data if ci.size else None,
                                          ci.size, int(H), int(M), int(bool(causal)))


def forward_workspace_bytes(d: int) -> int:
    """Bytes of the chunk workspace bsa_forward_ws can use for head dim d."""
    return int(library().bsa_forward_workspace_bytes(int(d)))


def forward(q, k, v, row_ptr, col_idx, block_size: int, scale: Optional[float] = None,
            causal: bool = False, out=None, lse=None, split: bool = True, workspace=None):
    """Block-sparse attention forward on q's device and current stream.

    q, k, v: CUDA bf16 tensors [B, H, N, d], contiguous.  row_ptr [H*M+1] and
    col_idx [nnz]: CUDA int32 tensors.  Returns (O bf16 [B,H,N,d], LSE fp32 [B,H,N]).
    With split (the default) the call is bsa_forward_ws, which may cut long
    tiles into chunks; `workspace` is then a CUDA tensor of at least
    forward_workspace_bytes(d) bytes (allocated on the current stream when
    not given).  split=False calls bsa_forward.
    """
    import torch

    lib = library()
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one shape [B, H, N, d]")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor")
    for name, t in (("row_ptr", row_ptr), ("col_idx", col_idx)):
        if not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA int32 tensor")
    B, H, N, d = (int(s) for s in q.shape)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    col_ptr = col_idx.data_ptr() if col_idx.numel() else row_ptr.data_ptr()
    with torch.cuda.device(q.device):
        stream = torch.cuda.current_stream(q.device).cuda_stream
        if not split:
            rc = lib.bsa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), row_ptr.data_ptr(),
                                 col_ptr, B, H, N, d, int(block_size), float(scale),
                                 int(bool(causal)), out.data_ptr(), lse.data_ptr(), stream)
            _check(rc, "bsa_forward")
            return out, lse
        if workspace is None:
            nbytes = int(lib.bsa_forward_workspace_bytes(d))
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
        if not workspace.is_cuda or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        rc = lib.bsa_forward_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), row_ptr.data_ptr(),
                                col_ptr, B, H, N, d, int(block_size), float(scale),
                                int(bool(causal)), out.data_ptr(), lse.data_ptr(),
                                workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                stream)
    _check(rc, "bsa_forward_ws")
    return out, lse


def topk_nnz(BH: int, M: int, top_k: int, causal: bool = False) -> int:
    """Stored blocks of a top-k pattern over BH heads (bsa_topk_nnz)."""
    n = int(library().bsa_topk_nnz(int(BH), int(M), int(top_k), int(bool(causal))))
    if n < 0:
        raise BsaError(ERR_INVALID_ARG, "bsa_topk_nnz")
    return n


def topk_pattern(q, k, block_size: int, top_k: int, causal: bool = False, workspace=None):
    """Content-based top-k block selection on q's device (bsa_topk_pattern).

    q, k: CUDA bf16 [B, H, N, d] contiguous.  Returns device int32 (row_ptr
    [B*H*M+1], col_idx) with one CSR row per (b*H + h, block row): run
    `forward` on q.view(1, B*H, N, d) etc. with it.  The fp64 workspace is a
    caller-owned CUDA tensor (allocated here when not given).
    """
    import torch

    lib = library()
    if q.dim() != 4 or k.shape != q.shape:
        raise ValueError("q, k must share one shape [B, H, N, d]")
    for name, t in (("q", q), ("k", k)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor")
    B, H, N, d = (int(x) for x in q.shape)
    BH, M = B * H, N // int(block_size)
    nbytes = int(lib.bsa_topk_workspace_bytes(BH, N, d, int(block_size)))
    if nbytes == 0:
        raise BsaError(ERR_INVALID_ARG, "bsa_topk_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(nbytes // 8, dtype=torch.float64, device=q.device)
    nnz = topk_nnz(BH, M, top_k, causal)
    row_ptr = torch.empty(BH * M + 1, dtype=torch.int32, device=q.device)
    col_idx = torch.empty(max(nnz, 1), dtype=torch.int32, device=q.device)
    with torch.cuda.device(q.device):
        stream = torch.cuda.current_stream(q.device).cuda_stream
        rc = lib.bsa_topk_pattern(q.data_ptr(), k.data_ptr(), BH, N, d, int(block_size),
                                  int(top_k), int(bool(causal)), row_ptr.data_ptr(),
                                  col_idx.data_ptr(), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), stream)
    _check(rc, "bsa_topk_pattern")
    return row_ptr, col_idx[:nnz]


TOPK_STATIC_SCRATCH_BYTES = 4 * 1024 * 1024


def topk_pattern_static(q, k, block_size: int, top_k: int, causal: bool, row_ptr, col_idx):
    """bsa_topk_pattern_static: the top-k selection with the library's own
    static scratch, writing into the caller's device int32 row_ptr
    [B*H*M+1] and col_idx [topk_nnz(...)].  Allocates nothing.

    Requests needing more than TOPK_STATIC_SCRATCH_BYTES of workspace raise
    BsaError(ERR_BUFFER_TOO_SMALL); calls overlapping in time on one device race.
    """
    import torch

    lib = library()
    if q.dim() != 4 or k.shape != q.shape:
        raise ValueError("q, k must share one shape [B, H, N, d]")
    for name, t in (("q", q), ("k", k)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor")
    B, H, N, d = (int(x) for x in q.shape)
    BH, M = B * H, N // int(block_size)
    nnz = topk_nnz(BH, M, top_k, causal)
    for name, t, n in (("row_ptr", row_ptr, BH * M + 1), ("col_idx", col_idx, nnz)):
        if (not t.is_cuda or t.device != q.device or t.dtype != torch.int32
                or not t.is_contiguous() or t.numel() < n):
            raise ValueError(f"{name} must be a contiguous int32 tensor on q's device "
                             f"with at least {n} elements")
    need = int(lib.bsa_topk_workspace_bytes(BH, N, d, int(block_size)))
    with torch.cuda.device(q.device):
        stream = torch.cuda.current_stream(q.device).cuda_stream
        rc = lib.bsa_topk_pattern_static(q.data_ptr(), k.data_ptr(), BH, N, d, int(block_size),
                                         int(top_k), int(bool(causal)), row_ptr.data_ptr(),
                                         col_idx.data_ptr(), stream)
    if rc == ERR_BUFFER_TOO_SMALL:
        raise BsaError(rc, f"bsa_topk_pattern_static (needs {need} bytes of scratch, the "
                           f"static scratch holds {TOPK_STATIC_SCRATCH_BYTES})")
    _check(rc, "bsa_topk_pattern_static")
    return row_ptr, col_idx[:nnz]


def transpose_pattern(row_ptr, col_idx, H: int, M: int) -> Tuple[np.ndarray, np.ndarray]:
    """Column-major copy of a host block-CSR (bsa_transpose_pattern): (col_ptr, row_idx)."""
    lib = library()
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    if rp.size != int(H) * int(M) + 1:
        raise ValueError("row_ptr must have H*M+1 entries")
    cp = np.empty(rp.size, dtype=np.int32)
    ri = np.empty(max(int(rp[-1]), 1), dtype=np.int32)
    nnz = ctypes.c_int64(0)
    _check(lib.bsa_transpose_pattern(rp.ctypes.data, ci.ctypes.data if ci.size else None, int(H),
                                     int(M), cp.ctypes.data, ri.ctypes.data, ri.size,
                                     ctypes.byref(nnz)), "bsa_transpose_pattern")
    return cp, ri[:nnz.value].copy()


def backward(q, k, v, o, do, lse, row_ptr, col_idx, col_ptr, row_idx, block_size: int,
             scale: float, causal: bool = False, workspace=None):
    """Gradients of `forward` (bsa_backward) on q's device and current stream.

    q, k, v, o, do: CUDA bf16 [B, H, N, d] contiguous (o, lse from `forward`);
    lse: CUDA fp32 [B, H, N]; row_ptr / col_idx: the forward's CSR and
    col_ptr / row_idx its `transpose_pattern`, all CUDA int32.  Returns
    (dQ, dK, dV) as CUDA bf16 [B, H, N, d].
    """
    import torch

    lib = library()
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = (int(x) for x in q.shape)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} must have q's shape")
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor on q's device")
    if (tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous()
            or lse.device != q.device):
        raise ValueError("lse must be a contiguous fp32 [B, H, N] tensor on q's device")
    for name, t in (("row_ptr", row_ptr), ("col_idx", col_idx), ("col_ptr", col_ptr),
                    ("row_idx", row_idx)):
        if not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous int32 tensor on q's device")
    nbytes = int(lib.bsa_backward_workspace_bytes(B, H, N))
    if workspace is None:
        workspace = torch.empty(max(nbytes // 4, 1), dtype=torch.float32, device=q.device)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    with torch.cuda.device(q.device):
        stream = torch.cuda.current_stream(q.device).cuda_stream
        rc = lib.bsa_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                              lse.data_ptr(), row_ptr.data_ptr(), col_idx.data_ptr(),
                              col_ptr.data_ptr(), row_idx.data_ptr(), B, H, N, d, int(block_size),
                              float(scale), int(bool(causal)), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), stream)
    _check(rc, "bsa_backward")
    return dq, dk, dv


def backward_status(clear: bool = True) -> int:
    """OR of STATUS_* bits raised by the backward kernels on the current device (synchronises it)."""
    v = ctypes.c_uint32(0)
    _check(library().bsa_backward_status(ctypes.byref(v), int(bool(clear))), "bsa_backward_status")
    return int(v.value)


def decode(q, k_cache, v_cache, seq_len, row_ptr, col_idx, block_size: int, scale: float,
           k_new=None, v_new=None, out=None, lse=None):
    """One decode step (bsa_decode) on q's device and current stream.

    q: CUDA bf16 [B, H, d]; k_cache, v_cache: CUDA bf16 [B, H, L, d] (with
    k_new / v_new [B, H, d] given, row seq_len[b] - 1 of each cache is
    overwritten with them first); seq_len: CUDA int32 [B]; row_ptr, col_idx:
    CUDA int32 block-CSR over L // block_size block rows per head.  Returns
    (O bf16 [B, H, d], LSE fp32 [B, H]).
    """
    import torch

    lib = library()
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q must be [B, H, d] and the caches [B, H, L, d]")
    B, H, L, d = (int(x) for x in k_cache.shape)
    if tuple(q.shape) != (B, H, d):
        raise ValueError("q must be [B, H, d] with the caches' B, H, d")
    named = [("q", q), ("k_cache", k_cache), ("v_cache", v_cache)]
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    if k_new is not None:
        named += [("k_new", k_new), ("v_new", v_new)]
        if tuple(k_new.shape) != (B, H, d) or tuple(v_new.shape) != (B, H, d):
            raise ValueError("k_new, v_new must be [B, H, d]")
    for name, t in named:
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor")
        if t.device != q.device:
            raise ValueError(f"{name} must be on q's device")
    for name, t in (("seq_len", seq_len), ("row_ptr", row_ptr), ("col_idx", col_idx)):
        if not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous int32 tensor on q's device")
    if seq_len.numel() != B:
        raise ValueError("seq_len must hold B entries")
    if row_ptr.numel() != H * (L // int(block_size)) + 1:
        raise ValueError("row_ptr must have H*M+1 entries")
    O = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device) if out is None else out
    LSE = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    with torch.cuda.device(q.device):
        stream = torch.cuda.current_stream(q.device).cuda_stream
        rc = lib.bsa_decode(q.data_ptr(), None if k_new is None else k_new.data_ptr(),
                            None if v_new is None else v_new.data_ptr(), k_cache.data_ptr(),
                            v_cache.data_ptr(), row_ptr.data_ptr(), col_idx.data_ptr(),
                            seq_len.data_ptr(), B, H, L, d, int(block_size), float(scale),
                            O.data_ptr(), LSE.data_ptr(), stream)
    _check(rc, "bsa_decode")
    return O, LSE


def decode_status(clear: bool = True) -> int:
    """OR of STATUS_* bits raised by the decode kernel on the current device (synchronises it)."""
    v = ctypes.c_uint32(0)
    _check(library().bsa_decode_status(ctypes.byref(v), int(bool(clear))), "bsa_decode_status")
    return int(v.value)


def device_status(clear: bool = True) -> int:
    """OR of STATUS_* bits raised by kernels on the current device (synchronises it)."""
    v = ctypes.c_uint32(0)
    _check(library().bsa_device_status(ctypes.byref(v), int(bool(clear))), "bsa_device_status")
    return int(v.value)


def version() -> int:
    return int(library().bsa_version())

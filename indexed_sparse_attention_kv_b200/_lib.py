"""Thin ctypes binding of liblsa.so (include/lsa.h), same names as the C ABI.

Argument marshalling only: shapes are read from the tensors, pointers and the
current CUDA stream are passed through, outputs and workspaces are allocated
with torch when the caller does not pass them, and a non-zero lsa_status is
raised as LsaError. Every step of the computation runs in liblsa's kernels;
there is no fallback of any kind: without liblsa.so or a CUDA device the calls
raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lsa.h")

LSA_OK = 0
STATUS_NAMES = {0: "LSA_OK", -1: "LSA_ERR_ARG", -2: "LSA_ERR_ALIGN", -3: "LSA_ERR_SHAPE",
                -4: "LSA_ERR_WORKSPACE", -5: "LSA_ERR_CUDA", -6: "LSA_ERR_TIMEOUT", -7: "LSA_ERR_UNSUPPORTED",
                -8: "LSA_ERR_SCRATCH"}
NOALLOC_SCRATCH_BYTES = 8 << 20   # LSA_NOALLOC_SCRATCH_BYTES
DEV_BAD_INDEX = 1
DEV_TIMEOUT = 2


class LsaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


class lsa_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("hq", ctypes.c_int), ("hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("r", ctypes.c_int), ("T", ctypes.c_int)]

    def __repr__(self):
        return "lsa_dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class lsa_proj_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("d", ctypes.c_int), ("r", ctypes.c_int), ("nbases", ctypes.c_int)]

    def __repr__(self):
        return "lsa_proj_dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_DIMS = ctypes.POINTER(lsa_dims)
_SIGS = {
    "lsa_version": (_I, []),
    "lsa_status_string": (ctypes.c_char_p, [_I]),
    "lsa_workspace_size": (_SZ, [_DIMS, _I, _I, _I]),
    "lsa_score": (_I, [_DIMS, _P, _P, _P, _P]),
    "lsa_topk": (_I, [_DIMS, _P, _I, _P, _P, _SZ, _P]),
    "lsa_indexed_attn": (_I, [_DIMS, _P, _P, _P, _P, _I, ctypes.c_float, _P, _P, _SZ, _P]),
    "lsa_indexed_attn_noalloc": (_I, [_DIMS, _P, _P, _P, _P, _I, ctypes.c_float, _P, _P, _P]),
    "lsa_score_fp8": (_I, [_DIMS, _P, _P, _P, _P]),
    "lsa_decode_step_fp8": (_I, [_DIMS, _P, _P, _P, _P, _P, _I, ctypes.c_float, _P, _P, _P, _SZ, _P]),
    "lsa_decode_step": (_I, [_DIMS, _P, _P, _P, _P, _P, _P, _I, _I, _I, ctypes.c_float, _P, _P, _P, _SZ, _P]),
    "lsa_block_centroids": (_I, [_DIMS, _P, _I, _P, _P]),
    "lsa_indexed_attn_paged": (_I, [_DIMS, _P, _P, _P, _I, _P, _P, _I, ctypes.c_float, _P, _P, _SZ, _P]),
    "lsa_decode_step_paged": (_I, [_DIMS, _P, _P, _P, _P, _I, _P, _P, _I, ctypes.c_float, _P, _P, _P, _SZ, _P]),
    "lsa_project": (_I, [ctypes.POINTER(lsa_proj_dims), _P, _P, _I, _I, _P, _P, _P]),
    "lsa_project_fp8": (_I, [ctypes.POINTER(lsa_proj_dims), _P, _P, _I, _I, _P, _P, _P]),
    "lsa_update_centroids": (_I, [_DIMS, _P, _I, _I, _I, _P, _P]),
    "lsa_prefill_workspace_size": (_SZ, [_DIMS, _I, _I]),
    "lsa_prefill_index": (_I, [_DIMS, _P, _I, _I, _P, _I, _P, _P, _SZ, _P]),
    "lsa_prefill_attn": (_I, [_DIMS, _P, _I, _P, _P, _P, _I, ctypes.c_float, _P, _P, _SZ, _P]),
    "lsa_read_device_status": (_I, [_P, _P, _P]),
    "lsa_clear_device_status": (_I, [_P, _P]),
    "lsa_debug_set_wait_limit": (None, [ctypes.c_longlong]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load liblsa.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"liblsa.so is not built ({LIB_PATH}); run "
                               "`python -m indexed_sparse_attention_kv_b200.csrc.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/lsa.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"LSA_API\s+[\w\s\*]+?\b(lsa_\w+)\s*\(", text)


def _check(fn: str, status: int) -> None:
    if status != LSA_OK:
        msg = lib().lsa_status_string(status).decode()
        raise LsaError(fn, status, msg)


def _cuda(t: torch.Tensor, name: str, dtype: torch.dtype) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (liblsa has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def make_dims(batch, hq, hkv, d, r, T) -> lsa_dims:
    return lsa_dims(int(batch), int(hq), int(hkv), int(d), int(r), int(T))


def decode_dims(q: torch.Tensor, qt: torch.Tensor, k: torch.Tensor) -> lsa_dims:
    batch, hq, d = q.shape
    r = qt.shape[-1]
    _, T, hkv, _ = k.shape
    return make_dims(batch, hq, hkv, d, r, T)


def lsa_workspace_size(dims: lsa_dims, B: int, blk: int = 0, keep: int = 0) -> int:
    return int(lib().lsa_workspace_size(ctypes.byref(dims), int(B), int(blk), int(keep)))


def workspace(dims: lsa_dims, B: int, blk: int = 0, keep: int = 0, device="cuda") -> torch.Tensor:
    """A zeroed uint8 workspace of lsa_workspace_size bytes (256-byte aligned)."""
    n = lsa_workspace_size(dims, B, blk, keep)
    if n == 0:
        raise LsaError("lsa_workspace_size", -1, f"invalid sizes {dims} B={B} blk={blk} keep={keep}")
    ws = torch.zeros(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def lsa_score(qt: torch.Tensor, kt: torch.Tensor, scores: torch.Tensor | None = None) -> torch.Tensor:
    """Group-mean scores [batch, hkv, T] fp32 of kt [batch, T, hkv, r] (lsa.h: lsa_score)."""
    _cuda(qt, "qt", torch.bfloat16)
    _cuda(kt, "kt", torch.bfloat16)
    batch, T, hkv, r = kt.shape
    dims = make_dims(batch, qt.shape[1], hkv, 128, r, T)
    if scores is None:
        scores = torch.empty((batch, hkv, T), dtype=torch.float32, device=kt.device)
    _cuda(scores, "scores", torch.float32)
    _check("lsa_score", lib().lsa_score(ctypes.byref(dims), _ptr(qt), _ptr(kt), _ptr(scores), _stream(kt)))
    return scores


def lsa_topk(scores: torch.Tensor, B: int, idx: torch.Tensor | None = None) -> torch.Tensor:
    """Top-B positions per row of scores [..., T] (lsa.h: lsa_topk); returns int32 [..., B]."""
    _cuda(scores, "scores", torch.float32)
    T = scores.shape[-1]
    rows = scores.numel() // T
    dims = make_dims(rows, 1, 1, 128, 16, T)
    if idx is None:
        idx = torch.empty((*scores.shape[:-1], B), dtype=torch.int32, device=scores.device)
    _cuda(idx, "idx", torch.int32)
    _check("lsa_topk", lib().lsa_topk(ctypes.byref(dims), _ptr(scores), int(B), _ptr(idx), None, 0,
                                      _stream(scores)))
    return idx


def lsa_indexed_attn(q, k, v, idx, scale: float | None = None, out=None, ws=None) -> torch.Tensor:
    """Indexed attention of q [batch, hq, d] over k/v rows idx [batch, hkv, B] (lsa.h: lsa_indexed_attn)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda(t, n, torch.bfloat16)
    _cuda(idx, "idx", torch.int32)
    batch, hq, d = q.shape
    _, T, hkv, _ = k.shape
    B = idx.shape[-1]
    dims = make_dims(batch, hq, hkv, d, 16, T)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    _cuda(out, "out", torch.bfloat16)
    if ws is None:
        ws = workspace(dims, B, device=q.device)
    _check("lsa_indexed_attn", lib().lsa_indexed_attn(
        ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), int(B), ctypes.c_float(scale), _ptr(out),
        _ptr(ws), ws.numel(), _stream(q)))
    return out


def lsa_indexed_attn_noalloc(q, k, v, idx, scale: float | None = None, out=None, dev_status=None) -> torch.Tensor:
    """lsa_indexed_attn with the library's fixed per-device scratch instead of a
    workspace (lsa.h: lsa_indexed_attn_noalloc). dev_status: optional device
    int32 [1] receiving LSA_DEV_* bits."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda(t, n, torch.bfloat16)
    _cuda(idx, "idx", torch.int32)
    batch, hq, d = q.shape
    _, T, hkv, _ = k.shape
    B = idx.shape[-1]
    dims = make_dims(batch, hq, hkv, d, 16, T)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    _cuda(out, "out", torch.bfloat16)
    if dev_status is not None:
        _cuda(dev_status, "dev_status", torch.int32)
    _check("lsa_indexed_attn_noalloc", lib().lsa_indexed_attn_noalloc(
        ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), int(B), ctypes.c_float(scale), _ptr(out),
        _ptr(dev_status), _stream(q)))
    return out


def lsa_decode_step(q, qt, k, v, kt, B: int, scale: float | None = None, centroids=None, blk: int = 0,
                    keep: int = 0, idx_out=None, out=None, ws=None, return_idx: bool = True):
    """One decode step (lsa.h: lsa_decode_step). Returns (idx [batch, hkv, B] or None, out [batch, hq, d])."""
    for t, n in ((q, "q"), (qt, "qt"), (k, "k"), (v, "v"), (kt, "kt")):
        _cuda(t, n, torch.bfloat16)
    dims = decode_dims(q, qt, k)
    scale = 1.0 / math.sqrt(dims.d) if scale is None else float(scale)
    if centroids is not None:
        _cuda(centroids, "centroids", torch.bfloat16)
        nblk = -(-dims.T // blk)
        keep = min(int(keep), nblk)
    else:
        blk, keep = 0, 0
    if out is None:
        out = torch.empty_like(q)
    if idx_out is None and return_idx:
        idx_out = torch.empty((dims.batch, dims.hkv, B), dtype=torch.int32, device=q.device)
    if idx_out is not None:
        _cuda(idx_out, "idx_out", torch.int32)
    if ws is None:
        ws = workspace(dims, B, blk, keep, device=q.device)
    _check("lsa_decode_step", lib().lsa_decode_step(
        ctypes.byref(dims), _ptr(q), _ptr(qt), _ptr(k), _ptr(v), _ptr(kt), _ptr(centroids), int(blk), int(keep),
        int(B), ctypes.c_float(scale), _ptr(idx_out), _ptr(out), _ptr(ws), ws.numel(), _stream(q)))
    return idx_out, out


def _paged_dims(q, k_pool, page_table, r):
    batch, hq, d = q.shape
    nslots, hkv, _ = k_pool.shape
    T = page_table.shape[1]
    return make_dims(batch, hq, hkv, d, r, T), nslots


def lsa_indexed_attn_paged(q, k_pool, v_pool, page_table, idx, scale: float | None = None, out=None,
                           ws=None) -> torch.Tensor:
    """Indexed attention over a paged KV cache (lsa.h: lsa_indexed_attn_paged): k_pool / v_pool
    [nslots, hkv, d], page_table [batch, T] int32 (pool slot of each logical position), idx
    [batch, hkv, B] logical positions."""
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _cuda(t, n, torch.bfloat16)
    _cuda(page_table, "page_table", torch.int32)
    _cuda(idx, "idx", torch.int32)
    dims, nslots = _paged_dims(q, k_pool, page_table, 16)
    B = idx.shape[-1]
    scale = 1.0 / math.sqrt(dims.d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    _cuda(out, "out", torch.bfloat16)
    if ws is None:
        ws = workspace(dims, B, device=q.device)
    _check("lsa_indexed_attn_paged", lib().lsa_indexed_attn_paged(
        ctypes.byref(dims), _ptr(q), _ptr(k_pool), _ptr(v_pool), int(nslots), _ptr(page_table), _ptr(idx), int(B),
        ctypes.c_float(scale), _ptr(out), _ptr(ws), ws.numel(), _stream(q)))
    return out


def lsa_decode_step_paged(q, qt, k_pool, v_pool, page_table, kt, B: int, scale: float | None = None, idx_out=None,
                          out=None, ws=None, return_idx: bool = True):
    """One flat decode step over a paged KV cache (lsa.h: lsa_decode_step_paged); kt [batch, T, hkv, r]
    stays contiguous. Returns (idx [batch, hkv, B] or None, out [batch, hq, d])."""
    for t, n in ((q, "q"), (qt, "qt"), (k_pool, "k_pool"), (v_pool, "v_pool"), (kt, "kt")):
        _cuda(t, n, torch.bfloat16)
    _cuda(page_table, "page_table", torch.int32)
    dims, nslots = _paged_dims(q, k_pool, page_table, kt.shape[-1])
    scale = 1.0 / math.sqrt(dims.d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if idx_out is None and return_idx:
        idx_out = torch.empty((dims.batch, dims.hkv, B), dtype=torch.int32, device=q.device)
    if idx_out is not None:
        _cuda(idx_out, "idx_out", torch.int32)
    if ws is None:
        ws = workspace(dims, B, device=q.device)
    _check("lsa_decode_step_paged", lib().lsa_decode_step_paged(
        ctypes.byref(dims), _ptr(q), _ptr(qt), _ptr(k_pool), _ptr(v_pool), int(nslots), _ptr(page_table), _ptr(kt),
        int(B), ctypes.c_float(scale), _ptr(idx_out), _ptr(out), _ptr(ws), ws.numel(), _stream(q)))
    return idx_out, out


def _fp8(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (liblsa has no CPU path)")
    if t.dtype != torch.float8_e4m3fn:
        raise TypeError(f"{name} must be torch.float8_e4m3fn, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def lsa_score_fp8(qt: torch.Tensor, kt: torch.Tensor, scores: torch.Tensor | None = None) -> torch.Tensor:
    """Group-mean scores [batch, hkv, T] of an FP8 E4M3 projected-key cache kt [batch, T, hkv, r]
    (lsa.h: lsa_score_fp8)."""
    _cuda(qt, "qt", torch.bfloat16)
    _fp8(kt, "kt")
    batch, T, hkv, r = kt.shape
    dims = make_dims(batch, qt.shape[1], hkv, 128, r, T)
    if scores is None:
        scores = torch.empty((batch, hkv, T), dtype=torch.float32, device=kt.device)
    _cuda(scores, "scores", torch.float32)
    _check("lsa_score_fp8", lib().lsa_score_fp8(ctypes.byref(dims), _ptr(qt), _ptr(kt), _ptr(scores), _stream(kt)))
    return scores


def lsa_decode_step_fp8(q, qt, k, v, kt, B: int, scale: float | None = None, idx_out=None, out=None, ws=None,
                        return_idx: bool = True):
    """One flat decode step over an FP8 E4M3 projected-key cache (lsa.h: lsa_decode_step_fp8).
    Returns (idx [batch, hkv, B] or None, out [batch, hq, d])."""
    for t, n in ((q, "q"), (qt, "qt"), (k, "k"), (v, "v")):
        _cuda(t, n, torch.bfloat16)
    _fp8(kt, "kt")
    dims = decode_dims(q, qt, k)
    scale = 1.0 / math.sqrt(dims.d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if idx_out is None and return_idx:
        idx_out = torch.empty((dims.batch, dims.hkv, B), dtype=torch.int32, device=q.device)
    if idx_out is not None:
        _cuda(idx_out, "idx_out", torch.int32)
    if ws is None:
        ws = workspace(dims, B, device=q.device)
    _check("lsa_decode_step_fp8", lib().lsa_decode_step_fp8(
        ctypes.byref(dims), _ptr(q), _ptr(qt), _ptr(k), _ptr(v), _ptr(kt), int(B), ctypes.c_float(scale),
        _ptr(idx_out), _ptr(out), _ptr(ws), ws.numel(), _stream(q)))
    return idx_out, out


def lsa_block_centroids(kt: torch.Tensor, blk: int, centroids=None) -> torch.Tensor:
    """Block centroids [batch, ceil(T/blk), hkv, r] of kt [batch, T, hkv, r] (lsa.h: lsa_block_centroids)."""
    _cuda(kt, "kt", torch.bfloat16)
    batch, T, hkv, r = kt.shape
    dims = make_dims(batch, hkv, hkv, 128, r, T)
    if centroids is None:
        centroids = torch.empty((batch, -(-T // blk), hkv, r), dtype=torch.bfloat16, device=kt.device)
    _cuda(centroids, "centroids", torch.bfloat16)
    _check("lsa_block_centroids", lib().lsa_block_centroids(ctypes.byref(dims), _ptr(kt), int(blk),
                                                            _ptr(centroids), _stream(kt)))
    return centroids


def _project(fn, x, P, t0, n, y, ydtype, dev_status):
    _cuda(x, "x", torch.bfloat16)
    _cuda(P, "P", torch.bfloat16)
    if x.dim() != 4 or P.dim() != 3:
        raise LsaError(fn, -1, "x must be [batch, T, H, d] and P [nbases, r, d]")
    batch, T, H, d = x.shape
    nbases, r, _ = P.shape
    if y is None:
        y = torch.zeros((batch, T, H, r), dtype=ydtype, device=x.device)
    _cuda(y, "y", ydtype)
    if dev_status is not None:
        _cuda(dev_status, "dev_status", torch.int32)
    dims = lsa_proj_dims(batch, T, H, d, r, nbases)
    t0 = 0 if t0 is None else int(t0)
    n = T - t0 if n is None else int(n)
    _check(fn, getattr(lib(), fn)(ctypes.byref(dims), _ptr(x), _ptr(P), t0, n, _ptr(y), _ptr(dev_status),
                                  _stream(x)))
    return y


def lsa_project(x, P, t0: int | None = None, n: int | None = None, y=None, dev_status=None) -> torch.Tensor:
    """Project rows t0 .. t0+n-1 of x [batch, T, H, d] onto the bases P [nbases, r, d]
    (row i uses basis i // (H // nbases)) into y [batch, T, H, r] bf16 (lsa.h: lsa_project)."""
    return _project("lsa_project", x, P, t0, n, y, torch.bfloat16, dev_status)


def lsa_project_fp8(x, P, t0: int | None = None, n: int | None = None, y=None, dev_status=None) -> torch.Tensor:
    """lsa_project into an FP8 E4M3 y [batch, T, H, r] (lsa.h: lsa_project_fp8)."""
    return _project("lsa_project_fp8", x, P, t0, n, y, torch.float8_e4m3fn, dev_status)


def lsa_update_centroids(kt: torch.Tensor, centroids: torch.Tensor, blk: int, t0: int, n: int) -> torch.Tensor:
    """Add kt rows t0 .. t0+n-1 [batch, T, hkv, r] to their block centroids
    [batch, ceil(T/blk), hkv, r] in place, bf16 after every add (lsa.h: lsa_update_centroids)."""
    _cuda(kt, "kt", torch.bfloat16)
    _cuda(centroids, "centroids", torch.bfloat16)
    batch, T, hkv, r = kt.shape
    dims = make_dims(batch, hkv, hkv, 128, r, T)
    _check("lsa_update_centroids", lib().lsa_update_centroids(ctypes.byref(dims), _ptr(kt), int(blk), int(t0),
                                                              int(n), _ptr(centroids), _stream(kt)))
    return centroids


def lsa_prefill_workspace_size(dims: lsa_dims, nq: int, B: int) -> int:
    return int(lib().lsa_prefill_workspace_size(ctypes.byref(dims), int(nq), int(B)))


def prefill_workspace(dims: lsa_dims, nq: int, B: int, device="cuda") -> torch.Tensor:
    """A zeroed uint8 prefill workspace (256-byte aligned)."""
    n = lsa_prefill_workspace_size(dims, nq, B)
    if n == 0:
        raise LsaError("lsa_prefill_workspace_size", -1, f"invalid sizes {dims} nq={nq} B={B}")
    ws = torch.zeros(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def prefill_dims(hq: int, kt: torch.Tensor, d: int = 128) -> lsa_dims:
    T, hkv, r = kt.shape
    return make_dims(1, hq, hkv, d, r, T)


def lsa_prefill_index(qt, kt, q_start: int, B: int, idx=None, ws=None) -> torch.Tensor:
    """Causal top-B index sets [nq, hkv, B] of queries qt [nq, hq, r] at positions
    q_start .. q_start + nq - 1 over kt [T, hkv, r] (lsa.h: lsa_prefill_index)."""
    _cuda(qt, "qt", torch.bfloat16)
    _cuda(kt, "kt", torch.bfloat16)
    nq, hq, _ = qt.shape
    dims = prefill_dims(hq, kt)
    if idx is None:
        idx = torch.empty((nq, dims.hkv, B), dtype=torch.int32, device=qt.device)
    _cuda(idx, "idx", torch.int32)
    if ws is None:
        ws = prefill_workspace(dims, nq, B, device=qt.device)
    _check("lsa_prefill_index", lib().lsa_prefill_index(
        ctypes.byref(dims), _ptr(qt), int(nq), int(q_start), _ptr(kt), int(B), _ptr(idx), _ptr(ws), ws.numel(),
        _stream(qt)))
    return idx


def lsa_prefill_attn(q, k, v, idx, scale: float | None = None, out=None, ws=None) -> torch.Tensor:
    """Indexed attention of every prefill query q [nq, hq, d] over k/v [T, hkv, d]
    rows idx [nq, hkv, B] (lsa.h: lsa_prefill_attn)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda(t, n, torch.bfloat16)
    _cuda(idx, "idx", torch.int32)
    nq, hq, d = q.shape
    T, hkv, _ = k.shape
    B = idx.shape[-1]
    dims = make_dims(1, hq, hkv, d, 16, T)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    _cuda(out, "out", torch.bfloat16)
    if ws is None:
        ws = prefill_workspace(dims, nq, B, device=q.device)
    _check("lsa_prefill_attn", lib().lsa_prefill_attn(
        ctypes.byref(dims), _ptr(q), int(nq), _ptr(k), _ptr(v), _ptr(idx), int(B), ctypes.c_float(scale), _ptr(out),
        _ptr(ws), ws.numel(), _stream(q)))
    return out


def lsa_read_device_status(ws: torch.Tensor) -> int:
    """Synchronously read the workspace's device status word (LSA_DEV_* bits)."""
    host = torch.zeros(1, dtype=torch.int32).pin_memory()
    _check("lsa_read_device_status", lib().lsa_read_device_status(_ptr(ws), _ptr(host), _stream(ws)))
    torch.cuda.current_stream(ws.device).synchronize()
    return int(host.item())


def lsa_clear_device_status(ws: torch.Tensor) -> None:
    _check("lsa_clear_device_status", lib().lsa_clear_device_status(_ptr(ws), _stream(ws)))


def lsa_debug_set_wait_limit(ns: int) -> None:
    """Device-time limit of every bounded wait in later launches (0: give up at the
    first failed probe; negative: restore the default of 2 s)."""
    lib().lsa_debug_set_wait_limit(int(ns))

"""Python binding of libkvc: window-attention token scoring, top-k selection
that keeps the window, and K/V / hidden-state compaction on B200 (sm_100a).

Argument marshalling only.  Every step runs in the CUDA kernels of
``libkvc.so`` (built in-tree by ``python -m long_context_kv_window_b200.build``);
PyTorch supplies device memory and the current stream.  There is no CPU path:
if the library is missing, importing the functions raises.

Names follow the C ABI in ``include/kvc.h``.  Tensors are CUDA tensors; bf16
inputs may be ``torch.bfloat16`` or raw ``int16``/``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvc.so")

KVC_OK = 0
KVC_DEV_ERR_INDEX = 1
KVC_DEV_ERR_SEQLENS = 2
KVC_DEV_ERR_TIMEOUT = 4
KVC_DEV_ERR_ORDER = 8


class KvcError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {status_string(status)} ({detail})")
        self.status = status


class ScoreParams(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32), ("scale", ctypes.c_float)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t

_SIGS = {
    "kvc_abi_version": ([], _I32),
    "kvc_status_string": ([_I32], ctypes.c_char_p),
    "kvc_last_error": ([], ctypes.c_char_p),
    "kvc_launch_count": ([], _I64),
    "kvc_score_workspace_size": ([_P, _I32, _I64, _P], _I32),
    "kvc_score": ([_P, _I64, _I64, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _SZ, _P, _P], _I32),
    "kvc_score_varlen": ([_P, _I64, _I64, _I64, _P, _I64, _I64, _P, _I32, _I64, _I64, _P, _P, _P, _P,
                          _P, _SZ, _P, _P], _I32),
    "kvc_score_noalloc": ([_P, _I64, _I64, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P], _I32),
    "kvc_score_lse": ([_P, _I64, _I64, _P, _I64, _I64, _I64, _P, _P, _I64, _I64, _P, _P, _P, _P, _SZ, _P, _P],
                      _I32),
    "kvc_prefill_attention": ([_P, _P, _P, _I64, _I32, _I32, _I32, ctypes.c_float, _P, _P, _P, _P], _I32),
    "kvc_select_workspace_size": ([_I32, _I32, _I64, _P], _I32),
    "kvc_select_topk": ([_P, _I32, _I64, _I32, _I64, _I32, _I32, _I64, _P, _I64, _P, _P, _SZ, _P], _I32),
    "kvc_select_topk_varlen": ([_P, _I32, _I64, _I32, _P, _I32, _I64, _I64, _I32, _I32, _I64, _P, _P, _P,
                                _SZ, _P, _P], _I32),
    "kvc_gather_kv": ([_P, _P, _I64, _I64, _I64, _I32, _I32, _P, _I64, _I64, _P, _P, _P, _P], _I32),
    "kvc_gather_kv_varlen": ([_P, _P, _I64, _I64, _P, _I32, _I64, _I32, _I32, _P, _I64, _P, _P, _P, _P],
                             _I32),
    "kvc_gather_hidden": ([_P, _I64, _I64, _I64, _P, _I64, _P, _P, _P], _I32),
    "kvc_stats_workspace_size": ([_I32, _I64, _P], _I32),
    "kvc_layer_stats": ([_P, _I32, _I64, _I64, ctypes.c_float, _P, _P, _SZ, _P], _I32),
    "kvc_pivot_update": ([_P, _I32, _I32, ctypes.c_double, _I32, _I32, _P, _P, _P], _I32),
    "kvc_rvq_encode": ([_P, _I64, _I64, _I32, _P, _I32, _I32, _P, _P, _P, _P], _I32),
    "kvc_decode_workspace_size": ([_I32, _I32, _I32, _I64, _P], _I32),
    "kvc_decode_attention": ([_P, _I64, _P, _P, _I64, _I32, _I32, _I32, ctypes.c_float, _P, _P, _SZ, _P, _P],
                             _I32),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libkvc.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m long_context_kv_window_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().kvc_status_string(s).decode()


def last_error() -> str:
    return lib().kvc_last_error().decode()


def launch_count() -> int:
    """Kernels launched by libkvc in this process."""
    return int(lib().kvc_launch_count())


def abi_version() -> int:
    return int(lib().kvc_abi_version())


def _check(status: int, where: str) -> None:
    if status != KVC_OK:
        raise KvcError(status, where, last_error())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream], dev: torch.device):
    """The launch stream: the given one, else the current stream of `dev`
    (the device every tensor of the call lives on)."""
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    if s.device != dev:
        raise ValueError(f"stream is on {s.device}, the tensors on {dev}")
    return ctypes.c_void_p(s.cuda_stream)


def _call(dev: torch.device, fn, *args) -> int:
    """Run one libkvc entry point with `dev` current (kernel launches and the
    per-device function attributes refer to the current device)."""
    with torch.cuda.device(dev):
        return fn(*args)


# The C entry points take raw pointers and sizes and cannot see a tensor's
# extent; the checks below make every pointer passed cover what the call
# reads or writes through it.
_BF16_BITS = (torch.bfloat16, torch.int16, torch.uint16)  # 2-byte storage of bf16 values


def _dense(t: torch.Tensor, name: str, shape, dtype, dev: torch.device) -> torch.Tensor:
    """A caller-supplied output the kernels address densely: exact shape,
    contiguous.  dtype: one dtype, or a tuple of accepted ones."""
    ok = t.dtype in dtype if isinstance(dtype, tuple) else t.dtype == dtype
    if not ok or t.device != dev:
        raise TypeError(f"{name} must be a {dtype} tensor on {dev}")
    if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor of shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _vector(t: Optional[torch.Tensor], name: str, numel: int, dtype: torch.dtype, dev: torch.device):
    """An optional contiguous array of exactly `numel` elements (any shape)."""
    if t is None:
        return None
    if t.dtype != dtype or t.device != dev:
        raise TypeError(f"{name} must be a {dtype} tensor on {dev}")
    if t.numel() != numel or not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous with {numel} elements, got shape {tuple(t.shape)}")
    return t


def _rows(t: torch.Tensor, name: str, rows: int, min_cols: int, dtype: torch.dtype, dev: torch.device):
    """A [rows][>= min_cols] matrix addressed by its row stride (unit column stride)."""
    if t.dtype != dtype or t.device != dev:
        raise TypeError(f"{name} must be a {dtype} tensor on {dev}")
    if t.dim() != 2 or t.shape[0] != rows or t.shape[1] < min_cols or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be [{rows}][>= {min_cols}] with unit column stride, got {tuple(t.shape)}")
    return t


def _err_word(t: Optional[torch.Tensor], dev: torch.device):
    if t is not None and (t.dtype != torch.int32 or t.device != dev or t.numel() < 1):
        raise TypeError(f"dev_err must be an int32 tensor on {dev} with at least one element")
    return t


def _ws_bytes(t: torch.Tensor, dev: torch.device) -> int:
    if t.device != dev or not t.is_contiguous():
        raise ValueError(f"ws must be a contiguous tensor on {dev}")
    return t.numel() * t.element_size()


def _same_device(dev: torch.device, **ts) -> None:
    for name, t in ts.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other inputs on {dev}")


def _bf16(t: torch.Tensor, name: str, dim: int) -> torch.Tensor:
    if t.dtype not in _BF16_BITS:
        raise TypeError(f"{name} must hold bf16 values (bfloat16 or int16/uint16 bits)")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions, got shape {tuple(t.shape)}")
    if t.stride(-1) != 1:
        raise ValueError(f"{name} must be contiguous in its last dimension")
    return t


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# --------------------------------------------------------------------------- #
# scoring
# --------------------------------------------------------------------------- #
def score_params(H: int, Hkv: int, d: int, w: int, scale: Optional[float] = None) -> ScoreParams:
    return ScoreParams(H, Hkv, d, w, float(1.0 / math.sqrt(d) if scale is None else scale))


def score_workspace_size(p: ScoreParams, batch: int, total: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().kvc_score_workspace_size(ctypes.byref(p), batch, total, ctypes.byref(out)),
           "kvc_score_workspace_size")
    return int(out.value)


def _score_outputs(dev, Hkv: int, total: int, scores, tsp, accum, dev_err):
    if scores is None:
        scores = torch.empty((Hkv, total), dtype=torch.float32, device=dev)
    _dense(scores, "scores", (Hkv, total), torch.float32, dev)
    _vector(tsp, "tsp", total, torch.float32, dev)
    if accum is not None:
        _dense(accum, "accum", (Hkv, total), torch.float32, dev)
    _err_word(dev_err, dev)
    return scores


def kvc_score(q_win: torch.Tensor, k: torch.Tensor, scale: Optional[float] = None,
              scores: Optional[torch.Tensor] = None, tsp: Optional[torch.Tensor] = None,
              accum: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
              dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Window-attention aggregate A [Hkv][n] (fp32) of q_win [w][H][d] over k [n][Hkv][d]."""
    _bf16(q_win, "q_win", 3)
    _bf16(k, "k", 3)
    dev = k.device
    _same_device(dev, q_win=q_win)
    w, H, d = q_win.shape
    n, Hkv, dk = k.shape
    if dk != d:
        raise ValueError("head_dim of q_win and k differ")
    p = score_params(H, Hkv, d, w, scale)
    scores = _score_outputs(dev, Hkv, n, scores, tsp, accum, dev_err)
    if ws is None:
        ws = _workspace(score_workspace_size(p, 1, n), dev)
    _check(_call(dev, lib().kvc_score, _ptr(q_win), q_win.stride(0), q_win.stride(1), _ptr(k), k.stride(0),
                 k.stride(1), n, ctypes.byref(p), _ptr(scores), _ptr(tsp), _ptr(accum), _ptr(ws),
                 _ws_bytes(ws, dev), _ptr(dev_err), _stream(stream, dev)), "kvc_score")
    return scores


def kvc_score_lse(q_win: torch.Tensor, k: torch.Tensor, lse: torch.Tensor, scale: Optional[float] = None,
                  scores: Optional[torch.Tensor] = None, tsp: Optional[torch.Tensor] = None,
                  accum: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                  dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """kvc_score with the window rows' softmax normalisers given: lse fp32
    [w][H] (any strides), lse[i, h] = ln of the sum of exp(scale * q . k) over
    the keys window row i of query head h sees -- the log-sum-exp a causal
    prefill attention returns, e.g. its [H][n] output viewed as
    ``lse_full[:, n - w:].t()``.  One pass over K instead of two."""
    _bf16(q_win, "q_win", 3)
    _bf16(k, "k", 3)
    dev = k.device
    _same_device(dev, q_win=q_win)
    w, H, d = q_win.shape
    n, Hkv, dk = k.shape
    if dk != d:
        raise ValueError("head_dim of q_win and k differ")
    if lse.dtype != torch.float32 or lse.device != dev:
        raise TypeError(f"lse must be a float32 tensor on {dev}")
    if tuple(lse.shape) != (w, H):
        raise ValueError(f"lse must be [{w}][{H}] (window row, query head), got {tuple(lse.shape)}")
    p = score_params(H, Hkv, d, w, scale)
    scores = _score_outputs(dev, Hkv, n, scores, tsp, accum, dev_err)
    if ws is None:
        ws = _workspace(score_workspace_size(p, 1, n), dev)
    _check(_call(dev, lib().kvc_score_lse, _ptr(q_win), q_win.stride(0), q_win.stride(1), _ptr(k), k.stride(0),
                 k.stride(1), n, ctypes.byref(p), _ptr(lse), lse.stride(0), lse.stride(1), _ptr(scores), _ptr(tsp),
                 _ptr(accum), _ptr(ws), _ws_bytes(ws, dev), _ptr(dev_err), _stream(stream, dev)), "kvc_score_lse")
    return scores


def kvc_score_noalloc(q_win: torch.Tensor, k: torch.Tensor, scale: Optional[float] = None,
                      scores: Optional[torch.Tensor] = None, tsp: Optional[torch.Tensor] = None,
                      accum: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """kvc_score without a caller workspace: the library's static device
    scratch is used instead (for callers that cannot allocate; calls that
    overlap on the GPU race on that scratch).  Pass `scores` to avoid even the
    output allocation here."""
    _bf16(q_win, "q_win", 3)
    _bf16(k, "k", 3)
    dev = k.device
    _same_device(dev, q_win=q_win)
    w, H, d = q_win.shape
    n, Hkv, dk = k.shape
    if dk != d:
        raise ValueError("head_dim of q_win and k differ")
    p = score_params(H, Hkv, d, w, scale)
    scores = _score_outputs(dev, Hkv, n, scores, tsp, accum, dev_err)
    _check(_call(dev, lib().kvc_score_noalloc, _ptr(q_win), q_win.stride(0), q_win.stride(1), _ptr(k),
                 k.stride(0), k.stride(1), n, ctypes.byref(p), _ptr(scores), _ptr(tsp), _ptr(accum),
                 _ptr(dev_err), _stream(stream, dev)), "kvc_score_noalloc")
    return scores


def kvc_score_varlen(q_win: torch.Tensor, k: torch.Tensor, cu_seqlens: torch.Tensor, max_seqlen: int,
                     scale: Optional[float] = None, scores: Optional[torch.Tensor] = None,
                     tsp: Optional[torch.Tensor] = None, accum: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Ragged batch: q_win [B][w][H][d], k [total][Hkv][d] packed, cu_seqlens int32 [B+1]."""
    _bf16(q_win, "q_win", 4)
    _bf16(k, "k", 3)
    dev = k.device
    _same_device(dev, q_win=q_win)
    B, w, H, d = q_win.shape
    total, Hkv, dk = k.shape
    if dk != d:
        raise ValueError("head_dim of q_win and k differ")
    _vector(cu_seqlens, "cu_seqlens", B + 1, torch.int32, dev)
    p = score_params(H, Hkv, d, w, scale)
    scores = _score_outputs(dev, Hkv, total, scores, tsp, accum, dev_err)
    if ws is None:
        ws = _workspace(score_workspace_size(p, B, total), dev)
    _check(_call(dev, lib().kvc_score_varlen, _ptr(q_win), q_win.stride(0), q_win.stride(1), q_win.stride(2),
                 _ptr(k), k.stride(0), k.stride(1), _ptr(cu_seqlens), B, total, int(max_seqlen),
                 ctypes.byref(p), _ptr(scores), _ptr(tsp), _ptr(accum), _ptr(ws), _ws_bytes(ws, dev),
                 _ptr(dev_err), _stream(stream, dev)), "kvc_score_varlen")
    return scores


# --------------------------------------------------------------------------- #
# selection
# --------------------------------------------------------------------------- #
def select_workspace_size(out_rows: int, batch: int, total: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().kvc_select_workspace_size(out_rows, batch, total, ctypes.byref(out)),
           "kvc_select_workspace_size")
    return int(out.value)


def _out_rows(rows: int, row_group: int) -> int:
    if row_group < 1 or rows % row_group:
        raise ValueError(f"row_group {row_group} must divide the {rows} score rows")
    return rows // row_group


def kvc_select_topk(scores: torch.Tensor, window: int, pool_kernel: int, k: int, row_group: int = 1,
                    n: Optional[int] = None, idx: Optional[torch.Tensor] = None,
                    pooled: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Per output row: the k - window best (pooled) prefix positions plus the
    window, ascending.  scores [rows][>= n] fp32; returns int32 [rows/row_group][min(k, n)]."""
    dev = scores.device
    if scores.dim() != 2:
        raise ValueError(f"scores must be [rows][n], got shape {tuple(scores.shape)}")
    rows = scores.shape[0]
    n = scores.shape[1] if n is None else int(n)
    _rows(scores, "scores", rows, n, torch.float32, dev)
    out_rows = _out_rows(rows, row_group)
    kout = min(k, n)
    if idx is None:
        idx = torch.empty((out_rows, kout), dtype=torch.int32, device=dev)
    _rows(idx, "idx", out_rows, kout, torch.int32, dev)
    if pooled is not None:
        _dense(pooled, "pooled", (out_rows, n - window), torch.float32, dev)
    if ws is None and pooled is None:
        ws = _workspace(select_workspace_size(out_rows, 1, n), dev)
    nbytes = 0 if ws is None else _ws_bytes(ws, dev)
    _check(_call(dev, lib().kvc_select_topk, _ptr(scores), rows, scores.stride(0), row_group, n, window,
                 pool_kernel, k, _ptr(idx), idx.stride(0), _ptr(pooled), _ptr(ws), nbytes, _stream(stream, dev)),
           "kvc_select_topk")
    return idx


def kvc_select_topk_varlen(scores: torch.Tensor, cu_seqlens: torch.Tensor, max_seqlen: int, window: int,
                           pool_kernel: int, k: int, row_group: int = 1, idx: Optional[torch.Tensor] = None,
                           counts: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                           dev_err: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Ragged batch; returns (idx int32 [B][rows/row_group][k] local positions, -1 padded,
    counts int32 [B])."""
    dev = scores.device
    if scores.dim() != 2:
        raise ValueError(f"scores must be [rows][total], got shape {tuple(scores.shape)}")
    rows, total = scores.shape[0], scores.shape[1]
    _rows(scores, "scores", rows, total, torch.float32, dev)
    B = cu_seqlens.numel() - 1
    _vector(cu_seqlens, "cu_seqlens", B + 1, torch.int32, dev)
    out_rows = _out_rows(rows, row_group)
    if idx is None:
        idx = torch.empty((B, out_rows, k), dtype=torch.int32, device=dev)
    _dense(idx, "idx", (B, out_rows, k), torch.int32, dev)
    if counts is None:
        counts = torch.empty((B,), dtype=torch.int32, device=dev)
    _vector(counts, "counts", B, torch.int32, dev)
    _err_word(dev_err, dev)
    if ws is None:
        ws = _workspace(select_workspace_size(out_rows, B, total), dev)
    _check(_call(dev, lib().kvc_select_topk_varlen, _ptr(scores), rows, scores.stride(0), row_group,
                 _ptr(cu_seqlens), B, total, int(max_seqlen), window, pool_kernel, k, _ptr(idx), _ptr(counts),
                 _ptr(ws), _ws_bytes(ws, dev), _ptr(dev_err), _stream(stream, dev)), "kvc_select_topk_varlen")
    return idx, counts


# --------------------------------------------------------------------------- #
# gathers
# --------------------------------------------------------------------------- #
def _kv_pair(k: torch.Tensor, v: Optional[torch.Tensor]) -> torch.device:
    _bf16(k, "k", 3)
    if v is not None:
        _bf16(v, "v", 3)
        _same_device(k.device, v=v)
        if v.stride() != k.stride() or v.shape != k.shape:
            raise ValueError("k and v must have the same shape and strides")
    return k.device


def kvc_gather_kv(k: torch.Tensor, v: Optional[torch.Tensor], idx: torch.Tensor,
                  k_out: Optional[torch.Tensor] = None, v_out: Optional[torch.Tensor] = None,
                  dev_err: Optional[torch.Tensor] = None, stream=None):
    """k, v [n][Hkv][d]; idx int32 [Hkv][kk] (or [1][kk] broadcast) -> k_out, v_out [Hkv][kk][d]."""
    dev = _kv_pair(k, v)
    n, Hkv, d = k.shape
    if idx.dim() != 2 or idx.shape[0] not in (1, Hkv):
        raise ValueError(f"idx must be [{Hkv}][kk] or [1][kk], got shape {tuple(idx.shape)}")
    kk = idx.shape[1]
    _rows(idx, "idx", idx.shape[0], kk, torch.int32, dev)
    irs = 0 if idx.shape[0] == 1 and Hkv > 1 else idx.stride(0)
    if k_out is None:
        k_out = torch.empty((Hkv, kk, d), dtype=k.dtype, device=dev)
    _dense(k_out, "k_out", (Hkv, kk, d), _BF16_BITS, dev)
    if v is not None:
        if v_out is None:
            v_out = torch.empty((Hkv, kk, d), dtype=v.dtype, device=dev)
        _dense(v_out, "v_out", (Hkv, kk, d), _BF16_BITS, dev)
    _err_word(dev_err, dev)
    _check(_call(dev, lib().kvc_gather_kv, _ptr(k), _ptr(v), k.stride(0), k.stride(1), n, Hkv, d, _ptr(idx),
                 irs, kk, _ptr(k_out), _ptr(v_out if v is not None else None), _ptr(dev_err),
                 _stream(stream, dev)), "kvc_gather_kv")
    return k_out, v_out


def kvc_gather_kv_varlen(k: torch.Tensor, v: Optional[torch.Tensor], cu_seqlens: torch.Tensor,
                         idx: torch.Tensor, k_out: Optional[torch.Tensor] = None,
                         v_out: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                         stream=None):
    """k, v [total][Hkv][d]; idx int32 [B][Hkv][kk] local positions -> [B][Hkv][kk][d]."""
    dev = _kv_pair(k, v)
    total, Hkv, d = k.shape
    if idx.dim() != 3 or idx.shape[1] != Hkv:
        raise ValueError(f"idx must be [B][{Hkv}][kk], got shape {tuple(idx.shape)}")
    B, _, kk = idx.shape
    _dense(idx, "idx", (B, Hkv, kk), torch.int32, dev)
    _vector(cu_seqlens, "cu_seqlens", B + 1, torch.int32, dev)
    if k_out is None:
        k_out = torch.empty((B, Hkv, kk, d), dtype=k.dtype, device=dev)
    _dense(k_out, "k_out", (B, Hkv, kk, d), _BF16_BITS, dev)
    if v is not None:
        if v_out is None:
            v_out = torch.empty((B, Hkv, kk, d), dtype=v.dtype, device=dev)
        _dense(v_out, "v_out", (B, Hkv, kk, d), _BF16_BITS, dev)
    _err_word(dev_err, dev)
    _check(_call(dev, lib().kvc_gather_kv_varlen, _ptr(k), _ptr(v), k.stride(0), k.stride(1), _ptr(cu_seqlens),
                 B, total, Hkv, d, _ptr(idx), kk, _ptr(k_out), _ptr(v_out if v is not None else None),
                 _ptr(dev_err), _stream(stream, dev)), "kvc_gather_kv_varlen")
    return k_out, v_out


def kvc_gather_hidden(x: torch.Tensor, idx: torch.Tensor, out: Optional[torch.Tensor] = None,
                      dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x [n][D] -> out [kk][D] = x[idx]."""
    _bf16(x, "x", 2)
    dev = x.device
    n, D = x.shape
    kk = idx.numel()
    _vector(idx, "idx", kk, torch.int32, dev)
    if out is None:
        out = torch.empty((kk, D), dtype=x.dtype, device=dev)
    _dense(out, "out", (kk, D), _BF16_BITS, dev)
    _err_word(dev_err, dev)
    _check(_call(dev, lib().kvc_gather_hidden, _ptr(x), x.stride(0), n, D, _ptr(idx), kk, _ptr(out),
                 _ptr(dev_err), _stream(stream, dev)), "kvc_gather_hidden")
    return out


# --------------------------------------------------------------------------- #
# decode over the compacted cache
# --------------------------------------------------------------------------- #
def decode_workspace_size(H: int, Hkv: int, d: int, kk: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().kvc_decode_workspace_size(H, Hkv, d, kk, ctypes.byref(out)), "kvc_decode_workspace_size")
    return int(out.value)


def kvc_decode_attention(q: torch.Tensor, k_c: torch.Tensor, v_c: torch.Tensor, scale: Optional[float] = None,
                         out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                         dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode query per head, q [H][d], over the compacted cache
    k_c, v_c [Hkv][kk][d] (every retained entry visible); returns fp32 [H][d].
    A caller's ws must have been zero-filled once (the call leaves it so)."""
    _bf16(q, "q", 2)
    _bf16(k_c, "k_c", 3)
    _bf16(v_c, "v_c", 3)
    dev = k_c.device
    _same_device(dev, q=q, v_c=v_c)
    H, d = q.shape
    Hkv, kk, dk = k_c.shape
    if dk != d or tuple(v_c.shape) != (Hkv, kk, d):
        raise ValueError("q [H][d], k_c and v_c [Hkv][kk][d] must agree")
    if not (k_c.is_contiguous() and v_c.is_contiguous()):
        raise ValueError("k_c and v_c must be contiguous")
    if out is None:
        out = torch.empty((H, d), dtype=torch.float32, device=dev)
    _dense(out, "out", (H, d), torch.float32, dev)
    _err_word(dev_err, dev)
    if ws is None:  # starts with per-KV-head counters, which must be zero before the first call
        ws = torch.zeros(max(decode_workspace_size(H, Hkv, d, kk), 1), dtype=torch.uint8, device=dev)
    sc = float(1.0 / math.sqrt(d) if scale is None else scale)
    _check(_call(dev, lib().kvc_decode_attention, _ptr(q), q.stride(0), _ptr(k_c), _ptr(v_c), kk, H, Hkv, d, sc,
                 _ptr(out), _ptr(ws), _ws_bytes(ws, dev), _ptr(dev_err), _stream(stream, dev)),
           "kvc_decode_attention")
    return out


def kvc_prefill_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
                          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                          want_out: bool = True, dev_err: Optional[torch.Tensor] = None,
                          stream=None) -> Tuple[Optional[torch.Tensor], torch.Tensor]:
    """Causal attention of one sequence, q [n][H][d], k and v [n][Hkv][d]
    (bf16, contiguous): returns (out bf16 [n][H][d] or None when want_out is
    False and none was passed, lse fp32 [n][H], the rows' log-sum-exp)."""
    _bf16(q, "q", 3)
    _bf16(k, "k", 3)
    _bf16(v, "v", 3)
    dev = q.device
    _same_device(dev, k=k, v=v)
    n, H, d = q.shape
    if tuple(k.shape[::2]) != (n, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q [n][H][d], k and v [n][Hkv][d] must agree")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k and v must be contiguous")
    Hkv = k.shape[1]
    if out is None and want_out:
        out = torch.empty((n, H, d), dtype=torch.bfloat16, device=dev)
    if out is not None:
        _dense(out, "out", (n, H, d), _BF16_BITS, dev)
    if lse is None:
        lse = torch.empty((n, H), dtype=torch.float32, device=dev)
    _dense(lse, "lse", (n, H), torch.float32, dev)
    _err_word(dev_err, dev)
    sc = float(1.0 / math.sqrt(d) if scale is None else scale)
    _check(_call(dev, lib().kvc_prefill_attention, _ptr(q), _ptr(k), _ptr(v), n, H, Hkv, d, sc, _ptr(out),
                 _ptr(lse), _ptr(dev_err), _stream(stream, dev)), "kvc_prefill_attention")
    return out, lse


# --------------------------------------------------------------------------- #
# residual vector quantisation
# --------------------------------------------------------------------------- #
def kvc_rvq_encode(x: torch.Tensor, codebooks: torch.Tensor, codes: Optional[torch.Tensor] = None,
                   residual: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Residual VQ of rows x [n][d] (bf16) against fp32 codebooks [S][M][d]:
    returns (codes int32 [n][S], residual fp32 [n][d] if one was passed)."""
    _bf16(x, "x", 2)
    dev = x.device
    _same_device(dev, codebooks=codebooks)
    n, d = x.shape
    if codebooks.dtype != torch.float32 or codebooks.dim() != 3 or codebooks.shape[2] != d:
        raise ValueError(f"codebooks must be float32 [S][M][{d}]")
    if not codebooks.is_contiguous():
        raise ValueError("codebooks must be contiguous")
    S, M = codebooks.shape[0], codebooks.shape[1]
    if codes is None:
        codes = torch.empty((n, S), dtype=torch.int32, device=dev)
    _dense(codes, "codes", (n, S), torch.int32, dev)
    if residual is not None:
        _dense(residual, "residual", (n, d), torch.float32, dev)
    _err_word(dev_err, dev)
    _check(_call(dev, lib().kvc_rvq_encode, _ptr(x), x.stride(0), n, d, _ptr(codebooks), S, M, _ptr(codes),
                 _ptr(residual), _ptr(dev_err), _stream(stream, dev)), "kvc_rvq_encode")
    return codes, residual


# --------------------------------------------------------------------------- #
# statistics
# --------------------------------------------------------------------------- #
def kvc_layer_stats(scores: torch.Tensor, mass_norm: float, n: Optional[int] = None,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per row of scores: [entropy, top-1% mass, variance] of scores/mass_norm."""
    dev = scores.device
    if scores.dim() != 2:
        raise ValueError(f"scores must be [rows][n], got shape {tuple(scores.shape)}")
    rows = scores.shape[0]
    n = scores.shape[1] if n is None else int(n)
    _rows(scores, "scores", rows, n, torch.float32, dev)
    if out is None:
        out = torch.empty((rows, 3), dtype=torch.float32, device=dev)
    _dense(out, "out", (rows, 3), torch.float32, dev)
    _check(_call(dev, lib().kvc_layer_stats, _ptr(scores), rows, scores.stride(0), n, float(mass_norm),
                 _ptr(out), None, 0, _stream(stream, dev)), "kvc_layer_stats")
    return out


# --------------------------------------------------------------------------- #
# pivot detection
# --------------------------------------------------------------------------- #
def pivot_state(device) -> torch.Tensor:
    """A zeroed device kvc_pivot_state (24 bytes: two float64, two int32),
    held as three int64."""
    return torch.zeros(3, dtype=torch.int64, device=device)


def pivot_layer(state: torch.Tensor) -> int:
    """The decided pivot layer (0 while undecided); reads the device state."""
    return int(state.view(torch.int32)[4].item())


def kvc_pivot_update(stats: torch.Tensor, layer: int, tau: float, l_min: int, l_max: int, state: torch.Tensor,
                     dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Fold layer `layer`'s statistics (kvc_layer_stats' [rows][3] output) into
    the online pivot rule held in `state` (see pivot_state); layers in order."""
    dev = stats.device
    if stats.dim() != 2 or stats.shape[1] != 3:
        raise ValueError(f"stats must be [rows][3], got shape {tuple(stats.shape)}")
    _dense(stats, "stats", (stats.shape[0], 3), torch.float32, dev)
    _vector(state, "state", 3, torch.int64, dev)
    _err_word(dev_err, dev)
    _check(_call(dev, lib().kvc_pivot_update, _ptr(stats), stats.shape[0], int(layer), float(tau), int(l_min),
                 int(l_max), _ptr(state), _ptr(dev_err), _stream(stream, dev)), "kvc_pivot_update")
    return state


# --------------------------------------------------------------------------- #
# one layer of the method, composed from the calls above
# --------------------------------------------------------------------------- #
@dataclass
class LayerOutputs:
    scores: torch.Tensor                    # [Hkv][n] fp32
    idx_kv: torch.Tensor                    # [Hkv][k_kv] int32
    k_c: torch.Tensor                       # [Hkv][k_kv][d]
    v_c: Optional[torch.Tensor]
    idx_tsp: Optional[torch.Tensor] = None  # [1][k_tsp] int32
    x_c: Optional[torch.Tensor] = None      # [k_tsp][D]
    tsp: Optional[torch.Tensor] = None      # [n] fp32 (when requested)


class LayerPlan:
    """Pre-allocated buffers for repeated calls of ``compress_layer`` on one shape."""

    def __init__(self, n: int, H: int, Hkv: int, d: int, w: int, k_kv: int, k_tsp: Optional[int],
                 hidden: Optional[int], with_v: bool, device, pool_kernel: int = 1, tsp_row: bool = False):
        self.n, self.H, self.Hkv, self.d, self.w = n, H, Hkv, d, w
        self.k_kv, self.k_tsp, self.hidden, self.pool = k_kv, k_tsp, hidden, pool_kernel
        f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
        self.params = score_params(H, Hkv, d, w)
        self.scores = torch.empty((Hkv, n), dtype=f32, device=device)
        self.ws_score = _workspace(score_workspace_size(self.params, 1, n), device)
        self.ws_sel_kv = _workspace(select_workspace_size(Hkv, 1, n), device)
        self.idx_kv = torch.empty((Hkv, min(k_kv, n)), dtype=i32, device=device)
        self.k_c = torch.empty((Hkv, min(k_kv, n), d), dtype=bf, device=device)
        self.v_c = torch.empty_like(self.k_c) if with_v else None
        self.dev_err = torch.zeros(1, dtype=i32, device=device)
        self.tsp = None
        self.tsp_row = tsp_row
        if k_tsp is not None:
            if tsp_row:  # the scoring call also writes the all-head sum row, which the TSP selection ranks
                self.tsp = torch.empty((1, n), dtype=f32, device=device)
            self.ws_sel_tsp = _workspace(select_workspace_size(1, 1, n), device)
            self.idx_tsp = torch.empty((1, min(k_tsp, n)), dtype=i32, device=device)
            self.x_c = (torch.empty((min(k_tsp, n), hidden), dtype=bf, device=device)
                        if hidden else None)
        self.side = torch.cuda.Stream(device=device)
        self._ev_scores = torch.cuda.Event()
        self._ev_side = torch.cuda.Event()

    def run(self, q_win, k, v=None, x=None, stream=None, lse=None) -> LayerOutputs:
        """Score -> per-KV-head top-k -> K/V gather; with a TSP budget also the
        all-head top-k -> hidden-state gather.  With lse (the window rows'
        log-sum-exp [w][H], as kvc_prefill_attention returns it for the last w
        rows) the scores come from kvc_score_lse: one read of K.

        The TSP selection ranks the sum of the KV-head score rows, formed as it
        stages them (heads in order, the same fp32 sum as the scoring call's
        optional head-sum row, which it writes to out.tsp when the plan was
        made with tsp_row=True).  The two selection -> gather chains only
        share the scores, so the K/V chain runs on a side stream concurrently
        with the TSP chain (enqueued first: it leads to the longer gather);
        both join the calling stream before returning.  Nothing is
        synchronised with the host; inputs must stay alive until the work
        completes."""
        main = stream if stream is not None else torch.cuda.current_stream(self.scores.device)
        if lse is None:
            kvc_score(q_win, k, scores=self.scores, tsp=self.tsp, ws=self.ws_score, dev_err=self.dev_err,
                      stream=main)
        else:
            kvc_score_lse(q_win, k, lse, scores=self.scores, tsp=self.tsp, ws=self.ws_score, dev_err=self.dev_err,
                          stream=main)
        out = LayerOutputs(self.scores, self.idx_kv, self.k_c, self.v_c)
        if self.k_tsp is None:
            self._kv_chain(k, v, main)
            return out
        self._ev_scores.record(main)
        if self.tsp_row:
            kvc_select_topk(self.tsp, self.w, self.pool, self.k_tsp, idx=self.idx_tsp, ws=self.ws_sel_tsp,
                            stream=main)
        else:
            kvc_select_topk(self.scores, self.w, self.pool, self.k_tsp, row_group=self.Hkv, idx=self.idx_tsp,
                            ws=self.ws_sel_tsp, stream=main)
        self.side.wait_event(self._ev_scores)
        self._kv_chain(k, v, self.side)
        out.idx_tsp = self.idx_tsp
        out.tsp = self.tsp
        if x is not None and self.x_c is not None:
            kvc_gather_hidden(x, self.idx_tsp.view(-1), out=self.x_c, dev_err=self.dev_err, stream=main)
            out.x_c = self.x_c
        self._ev_side.record(self.side)
        main.wait_event(self._ev_side)
        return out

    def _kv_chain(self, k, v, stream):
        kvc_select_topk(self.scores, self.w, self.pool, self.k_kv, idx=self.idx_kv, ws=self.ws_sel_kv,
                        stream=stream)
        kvc_gather_kv(k, v, self.idx_kv, k_out=self.k_c, v_out=self.v_c, dev_err=self.dev_err, stream=stream)

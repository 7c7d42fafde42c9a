"""Thin Python binding of libmxfa.so (fused attention forward for B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/mxfa.h``.  PyTorch provides device
memory (outputs, workspace) and the current stream.  There is no fallback:
if the library is missing, or a call fails, an exception is raised.

Functions carry the C entry points' names:
    mxfa_attn_fwd(q, k, v, causal=..., softmax_scale=...)              -> (o, lse)
    mxfa_attn_varlen_fwd(q, k, v, cu_q, cu_k, max_q, max_k, ...)       -> (o, lse)
    mxfa_attn_decode_splitkv(q, k, v, qo_indptr, kv_indptr, ...)       -> (o, lse)
    mxfa_attn_decode_mla_fp8kv(q, kv, kv_scale, qo_indptr, kv_indptr, ...) -> (o, lse)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxfa.so")

MXFA_OK, MXFA_ERR_INVALID_ARG, MXFA_ERR_UNSUPPORTED, MXFA_ERR_WORKSPACE, MXFA_ERR_CUDA, MXFA_ERR_TIMEOUT = range(6)
_DT = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}

_lock = threading.Lock()
_lib = None


class MxfaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"mxfa status {status}: {msg}")
        self.status = status


def load():
    """Load libmxfa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with `python -m tiled_attention_21_b200.build_ext`")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
            lib.mxfa_attn_fwd.argtypes = [vp] * 5 + [i32] * 7 + [i64] * 8 + [f32, i32, vp, sz, vp]
            lib.mxfa_attn_fwd.restype = i32
            lib.mxfa_attn_fwd_workspace_size.argtypes = [i32] * 7
            lib.mxfa_attn_fwd_workspace_size.restype = sz
            lib.mxfa_attn_varlen_fwd.argtypes = [vp] * 7 + [i32] * 9 + [f32, i32, vp, sz, vp]
            lib.mxfa_attn_varlen_fwd.restype = i32
            lib.mxfa_attn_varlen_fwd_workspace_size.argtypes = [i32] * 6
            lib.mxfa_attn_varlen_fwd_workspace_size.restype = sz
            lib.mxfa_attn_decode_splitkv.argtypes = [vp] * 7 + [i32] * 9 + [i64, i64, i32, f32, i32, i32, vp, sz, vp]
            lib.mxfa_attn_decode_splitkv.restype = i32
            lib.mxfa_attn_decode_splitkv_workspace_size.argtypes = [i32] * 8
            lib.mxfa_attn_decode_splitkv_workspace_size.restype = sz
            lib.mxfa_attn_decode_mla_fp8kv.argtypes = [vp, vp, f32] + [vp] * 4 + [i32] * 6 + [i64, f32, i32, i32,
                                                                                        vp, sz, vp]
            lib.mxfa_attn_decode_mla_fp8kv.restype = i32
            lib.mxfa_attn_decode_mla_fp8kv_workspace_size.argtypes = [i32] * 5
            lib.mxfa_attn_decode_mla_fp8kv_workspace_size.restype = sz
            lib.mxfa_attn_decode_kvcache.argtypes = [vp] * 7 + [i32] * 10 + [i32, f32, i32, i32, vp, vp, vp, sz, vp]
            lib.mxfa_attn_decode_kvcache.restype = i32
            lib.mxfa_attn_decode_kvcache_workspace_size.argtypes = [i32] * 8
            lib.mxfa_attn_decode_kvcache_workspace_size.restype = sz
            lib.mxfa_last_error.argtypes = []
            lib.mxfa_last_error.restype = ctypes.c_char_p
            lib.mxfa_read_device_status.argtypes = [vp, vp]
            lib.mxfa_read_device_status.restype = i32
            lib.mxfa_device_status_detail.argtypes = []
            lib.mxfa_device_status_detail.restype = ctypes.c_uint32
            lib.mxfa_version.argtypes = []
            lib.mxfa_version.restype = ctypes.c_uint32
            lib.mxfa_attn_varlen_fwd_noalloc.argtypes = [vp] * 7 + [i32] * 9 + [f32, i32, vp]
            lib.mxfa_attn_varlen_fwd_noalloc.restype = i32
            lib.mxfa_read_noalloc_status.argtypes = [vp]
            lib.mxfa_read_noalloc_status.restype = i32
            lib.mxfa_test_hooks.argtypes = [ctypes.c_uint64, i32]
            lib.mxfa_test_hooks.restype = None
            _lib = lib
    return _lib


def _check(status: int):
    if status != MXFA_OK:
        raise MxfaError(status, load().mxfa_last_error().decode())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


_ws_cache: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-initialised byte buffer of at least ``nbytes`` (cached per device).
    The library keeps a sticky status word at its head, cleared by
    ``read_device_status``."""
    dev = torch.device(device)
    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device())
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 256) + 256, dtype=torch.uint8, device=dev)
        _ws_cache[key] = buf
    return buf


def _ws_view(buf: torch.Tensor) -> tuple[int, int]:
    p = buf.data_ptr()
    off = (-p) % 256
    return p + off, buf.numel() - off


def read_device_status(ws: torch.Tensor | None = None, device=None) -> tuple[int, int]:
    """(status, site) recorded on the device since the last read; clears it."""
    lib = load()
    if ws is None:
        ws = workspace(256, device or torch.device("cuda"))
    p, _ = _ws_view(ws)
    st = lib.mxfa_read_device_status(ctypes.c_void_p(p), _stream(None))
    return st, lib.mxfa_device_status_detail()


def read_noalloc_status(stream=None) -> tuple[int, int]:
    """(status, site) of the no-allocation varlen entry point's last call on
    the current device (its scratch array's status word); clears it."""
    lib = load()
    st = lib.mxfa_read_noalloc_status(_stream(stream))
    return st, lib.mxfa_device_status_detail()


def _scale(s):
    return float("nan") if s is None else float(s)


def mxfa_attn_fwd(q, k, v, causal: bool = False, softmax_scale: float | None = None, out=None, lse=None,
                  return_lse: bool = True, ws: torch.Tensor | None = None, stream=None):
    """Batched attention, q [B, Sq, Hq, D], k/v [B, Sk, Hkv, D] (last dim contiguous,
    batches contiguous).  Returns (o [B, Sq, Hq, D], lse [B, Sq, Hq] fp32)."""
    lib = load()
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Sq, Hq), dtype=torch.float32, device=q.device)
    for name, t, S in (("q", q, Sq), ("k", k, Sk), ("v", v, Sk), ("o", out, Sq)):
        if t.stride(-1) != 1 or (t.shape[0] > 1 and t.stride(0) != S * t.stride(1)):
            raise ValueError(f"{name}: last dim must be contiguous and batches contiguous")
    dt = _DT[q.dtype]
    need = lib.mxfa_attn_fwd_workspace_size(B, Sq, Sk, Hq, Hkv, D, dt)
    ws = ws if ws is not None else workspace(need, q.device)
    wp, wn = _ws_view(ws)
    _check(lib.mxfa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Sk, Hq, Hkv, D, dt,
                             q.stride(1), q.stride(2), k.stride(1), k.stride(2), v.stride(1), v.stride(2),
                             out.stride(1), out.stride(2), _scale(softmax_scale), int(bool(causal)),
                             wp, wn, _stream(stream)))
    return out, lse


def mxfa_attn_varlen_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                         causal: bool = False, softmax_scale: float | None = None, out=None, lse=None,
                         return_lse: bool = True, ws: torch.Tensor | None = None, stream=None):
    """Packed attention, q [total_q, Hq, D], k/v [total_k, Hkv, D] contiguous,
    cu_seqlens int32 on the device.  Returns (o [total_q, Hq, D], lse [total_q, Hq])."""
    lib = load()
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    batch = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((total_q, Hq), dtype=torch.float32, device=q.device)
    dt = _DT[q.dtype]
    need = lib.mxfa_attn_varlen_fwd_workspace_size(batch, max_seqlen_q, max_seqlen_k, Hq, D, dt)
    ws = ws if ws is not None else workspace(need, q.device)
    wp, wn = _ws_view(ws)
    _check(lib.mxfa_attn_varlen_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                                    _ptr(cu_seqlens_k), batch, total_q, total_k, int(max_seqlen_q),
                                    int(max_seqlen_k), Hq, Hkv, D, dt, _scale(softmax_scale), int(bool(causal)),
                                    wp, wn, _stream(stream)))
    return out, lse


def mxfa_attn_decode_splitkv(q, k, v, qo_indptr, kv_indptr, max_q_len: int, max_kv_len: int,
                             softmax_scale: float | None = None, causal: bool = False, num_splits: int = 0,
                             out=None, lse=None, return_lse: bool = True, ws: torch.Tensor | None = None,
                             stream=None):
    """Split-KV decode.  q [total_q, Hq, Dqk] contiguous; k [total_kv, Hkv, Dqk] and
    v [total_kv, Hkv, Dv] with unit stride inside a row (they may be views of one
    MLA cache: k = kv, v = kv[..., :512]).  Returns (o [total_q, Hq, Dv], lse)."""
    lib = load()
    total_q, Hq, Dqk = q.shape
    total_kv, Hkv, Dv = v.shape
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    for name, t, d in (("k", k, Dqk), ("v", v, Dv)):
        if t.stride(2) != 1 or (Hkv > 1 and t.stride(1) != d):
            raise ValueError(f"{name}: rows must be [Hkv, D] contiguous")
    batch = qo_indptr.numel() - 1
    if out is None:
        out = torch.empty((total_q, Hq, Dv), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((total_q, Hq), dtype=torch.float32, device=q.device)
    dt = _DT[q.dtype]
    need = lib.mxfa_attn_decode_splitkv_workspace_size(batch, max_q_len, Hq, Hkv, Dv, max_kv_len, num_splits, dt)
    ws = ws if ws is not None else workspace(need, q.device)
    wp, wn = _ws_view(ws)
    _check(lib.mxfa_attn_decode_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(qo_indptr),
                                        _ptr(kv_indptr), batch, total_q, total_kv, int(max_q_len), int(max_kv_len),
                                        Hq, Hkv, Dqk, Dv, k.stride(0), v.stride(0), dt, _scale(softmax_scale),
                                        int(bool(causal)), int(num_splits), wp, wn, _stream(stream)))
    return out, lse


def mxfa_attn_decode_mla_fp8kv(q, kv, kv_scale: float, qo_indptr, kv_indptr, max_q_len: int, max_kv_len: int,
                               softmax_scale: float | None = None, causal: bool = False, num_splits: int = 0,
                               out=None, lse=None, return_lse: bool = True, ws: torch.Tensor | None = None,
                               stream=None):
    """MLA decode over an E4M3 latent cache.  q [total_q, Hq, 576] bf16 contiguous;
    kv [total_kv, 576] torch.float8_e4m3fn or uint8 codes (unit stride inside a
    row); element value = kv_scale * code value.  Returns (o [total_q, Hq, 512]
    bf16, lse [total_q, Hq])."""
    lib = load()
    total_q, Hq, Dqk = q.shape
    total_kv = kv.shape[0]
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16")
    if kv.dtype not in (torch.uint8, torch.float8_e4m3fn) or kv.dim() != 2 or kv.stride(1) != 1:
        raise ValueError("kv must be [total_kv, 576] E4M3 codes with unit stride inside a row")
    batch = qo_indptr.numel() - 1
    if out is None:
        out = torch.empty((total_q, Hq, 512), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((total_q, Hq), dtype=torch.float32, device=q.device)
    need = lib.mxfa_attn_decode_mla_fp8kv_workspace_size(batch, max_q_len, Hq, max_kv_len, num_splits)
    ws = ws if ws is not None else workspace(need, q.device)
    wp, wn = _ws_view(ws)
    _check(lib.mxfa_attn_decode_mla_fp8kv(_ptr(q), _ptr(kv), float(kv_scale), _ptr(out), _ptr(lse),
                                          _ptr(qo_indptr), _ptr(kv_indptr), batch, total_q, total_kv,
                                          int(max_q_len), int(max_kv_len), Hq, kv.stride(0),
                                          _scale(softmax_scale), int(bool(causal)), int(num_splits), wp, wn,
                                          _stream(stream)))
    return out, lse


def mxfa_attn_decode_kvcache(q, k_cache, v_cache, cache_seqlens, k_new=None, v_new=None, block_table=None,
                             softmax_scale: float | None = None, causal: bool = False, num_splits: int = 0,
                             max_len: int | None = None, out=None, lse=None, return_lse: bool = True,
                             ws: torch.Tensor | None = None, stream=None):
    """Decode over a KV cache.  q [B, Sq, Hq, D]; k_cache / v_cache [B, cache_len,
    Hkv, D] (dense, block_table None) or [num_pages, page_size, Hkv, D] with
    block_table [B, max_blocks] int32 (paged); cache_seqlens [B] int32 on the
    device.  k_new / v_new [B, Snew, Hkv, D] are appended at cache_seqlens
    first, and cache_seqlens is advanced by Snew in place.  All contiguous.
    Returns (o [B, Sq, Hq, D], lse [B, Sq, Hq])."""
    lib = load()
    B, Sq, Hq, D = q.shape
    num_pages, page_size, Hkv, _ = k_cache.shape
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("k_new", k_new), ("v_new", v_new),
                    ("cache_seqlens", cache_seqlens), ("block_table", block_table)):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if cache_seqlens.dtype != torch.int32 or (block_table is not None and block_table.dtype != torch.int32):
        raise ValueError("cache_seqlens and block_table must be int32")
    Snew = 0 if k_new is None else k_new.shape[1]
    max_blocks = 0 if block_table is None else block_table.shape[1]
    if max_len is None:
        max_len = page_size * max_blocks if block_table is not None else page_size
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Sq, Hq), dtype=torch.float32, device=q.device)
    dt = _DT[q.dtype]
    need = lib.mxfa_attn_decode_kvcache_workspace_size(B, Sq, Hq, Hkv, D, int(max_len), num_splits, dt)
    ws = ws if ws is not None else workspace(need, q.device)
    wp, wn = _ws_view(ws)
    _check(lib.mxfa_attn_decode_kvcache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new),
                                        _ptr(cache_seqlens), _ptr(block_table), B, Sq, Snew, Hq, Hkv, D, num_pages,
                                        page_size, max_blocks, int(max_len), dt, _scale(softmax_scale),
                                        int(bool(causal)), int(num_splits), _ptr(out), _ptr(lse), wp, wn,
                                        _stream(stream)))
    return out, lse


__all__ = ["load", "mxfa_attn_fwd", "mxfa_attn_varlen_fwd", "mxfa_attn_decode_splitkv", "mxfa_attn_decode_mla_fp8kv",
           "mxfa_attn_decode_kvcache", "read_device_status", "read_noalloc_status", "workspace", "MxfaError",
           "LIB_PATH"]

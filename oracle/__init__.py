"""fp64 CPU oracle for the attention forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product path never does; the CUDA library and this
oracle share no code, headers, tables or helpers.

``attention`` evaluates the plain definition (see ``attn_oracle.c``) for a
list of (token, head) pairs: a materialised score row per pair, fp64
throughout, O and the natural-log LSE returned as float64 tensors.  The pure
Python ``brute`` module is a second, independent restatement used on tiny
inputs to pin this one.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_DTYPE_CODE = {torch.float64: 0, torch.float32: 1, torch.float16: 2, torch.bfloat16: 3}


def build(out_path: str | None = None, mutant: int = 0) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, so IEEE fp64 holds)."""
    out_path = out_path or _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           f"-DORACLE_MUTANT={int(mutant)}", _SRC, "-o", out_path, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return out_path


def _bind(lib):
    f = lib.oracle_attention
    i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    f.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64, vp, vp, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, dbl, ctypes.c_int,
                  vp, i64, vp, vp, vp, ctypes.c_int]
    f.restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_q, cu_k, scale: float,
              causal: bool, pairs: torch.Tensor | None = None, threads: int | None = None,
              lib=None, return_psum: bool = False):
    """O and LSE of softmax(scale*q k^T + mask) v for packed inputs.

    q: [total_q, Hq, Dqk]; k: [total_k, Hkv, Dqk]; v: [total_k, Hkv, Dv] (CPU
    tensors of one dtype: f64, f32, f16 or bf16; any token/head strides, last
    dim contiguous).  cu_q / cu_k: cumulative lengths [batch+1].  pairs:
    [n, 2] int64 (token, head); None means every token and head, in which
    case O is returned as [total_q, Hq, Dv] and LSE as [total_q, Hq].
    """
    lib = lib or load()
    assert q.dtype == k.dtype == v.dtype and q.dtype in _DTYPE_CODE
    for t in (q, k, v):
        assert t.device.type == "cpu" and t.dim() == 3 and t.stride(2) == 1
    cu_q = torch.as_tensor(cu_q, dtype=torch.int64).contiguous()
    cu_k = torch.as_tensor(cu_k, dtype=torch.int64).contiguous()
    total_q, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    full = pairs is None
    if full:
        tok = torch.arange(total_q, dtype=torch.int64).repeat_interleave(hq)
        hd = torch.arange(hq, dtype=torch.int64).repeat(total_q)
        pairs = torch.stack([tok, hd], 1)
    pairs = pairs.to(torch.int64).contiguous()
    n = pairs.shape[0]
    o = torch.empty((n, dv), dtype=torch.float64)
    lse = torch.empty((n,), dtype=torch.float64)
    psum = torch.empty((n,), dtype=torch.float64)
    rc = lib.oracle_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), _DTYPE_CODE[q.dtype],
                              q.stride(0), q.stride(1), k.stride(0), k.stride(1), v.stride(0), v.stride(1),
                              cu_q.data_ptr(), cu_k.data_ptr(), cu_q.numel() - 1, hq, hkv, dqk, dv,
                              float(scale), int(bool(causal)), pairs.data_ptr(), n,
                              o.data_ptr(), lse.data_ptr(), psum.data_ptr(),
                              int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError("oracle_attention rejected its arguments")
    if full:
        o = o.view(total_q, hq, dv)
        lse = lse.view(total_q, hq)
        psum = psum.view(total_q, hq)
    return (o, lse, psum) if return_psum else (o, lse)


def problem(p, pairs=None, threads=None, lib=None, return_psum=False):
    """Run the oracle on a ``workloads.Problem`` (inputs in their stored dtype).
    An E4M3 latent cache (``p.kv_scale`` set, ``p.kv`` the codes) is first
    dequantised exactly in fp64 (``e4m3.dequantize``); q is then taken in fp64
    too (exact), since the oracle wants one dtype for q, k and v."""
    if getattr(p, "kv_scale", None) is not None:
        from . import e4m3
        kv = e4m3.dequantize(p.kv, p.kv_scale)
        tk = kv.shape[0]
        return attention(p.q.double(), kv.view(tk, 1, p.dqk), kv[:, :p.dv].view(tk, 1, p.dv), p.cu_q, p.cu_k,
                         p.scale, p.causal, pairs=pairs, threads=threads, lib=lib, return_psum=return_psum)
    return attention(p.q, p.k, p.v, p.cu_q, p.cu_k, p.scale, p.causal, pairs=pairs,
                     threads=threads, lib=lib, return_psum=return_psum)

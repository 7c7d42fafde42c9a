"""mxfa_attn_varlen_fwd_noalloc: the varlen forward for callers that cannot
allocate device memory when they run attention (plugins and services with a
fixed, pre-planned device memory budget, or code without access to the
allocator that owns the device).  Its scratch is a fixed array inside the
library, so the caller passes only inputs and outputs.

The GPU test calls the entry point through the C ABI twice in a row, on two
different problems, and checks each result against mxfa_attn_varlen_fwd (the
entry point that takes a caller workspace) within the parity tolerances.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import workloads

FAKE = 0x100000


def _bind(lib):
    f = lib.mxfa_attn_varlen_fwd_noalloc
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [vp] * 7 + [i32] * 9 + [f32, i32, vp]
    f.restype = i32
    return f


def _lib():
    import tiled_attention_21_b200 as mx
    from tiled_attention_21_b200 import build_ext
    try:
        build_ext.build()
    except RuntimeError:
        pass
    return mx, mx.load()


def test_rejects_problems_beyond_the_scratch_limit():
    """A schedule larger than the fixed 1 MiB scratch is refused before any launch."""
    mx, lib = _lib()
    f = _bind(lib)
    r = f(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 4096, 1 << 24, 1 << 24, 65536, 65536, 8, 2, 128, 2,
          float("nan"), 1, None)
    assert r == mx.MXFA_ERR_WORKSPACE
    assert b"no-allocation" in lib.mxfa_last_error()


def _call_noalloc(f, p, q, k, v, cu_q, cu_k, stream):
    o = torch.full_like(q, float("nan"))
    lse = torch.full((q.shape[0], p.hq), float("nan"), dtype=torch.float32, device=q.device)
    r = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), cu_q.data_ptr(), cu_k.data_ptr(),
          p.batch, p.total_q, p.total_k, max(p.seqlens_q()), max(p.seqlens_k()), p.hq, p.hkv, p.dqk,
          {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}[q.dtype], float("nan"), int(p.causal),
          ctypes.c_void_p(stream.cuda_stream))
    return r, o, lse


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mx, lib = _lib()
    f = _bind(lib)
    stream = torch.cuda.current_stream()
    problems = [
        workloads.varlen(31, [300, 17, 512, 1, 129], [300, 40, 512, 1, 129], 8, 2, 128, "bf16", True),
        workloads.varlen(32, [64, 700, 3], [80, 700, 3], 4, 4, 64, "f16", False),
    ]
    for p in problems:
        q, k, v = p.q.cuda(), p.k.cuda(), p.v.cuda()
        cu_q, cu_k = p.cu_q.cuda(), p.cu_k.cuda()
        ref_o, ref_l = mx.mxfa_attn_varlen_fwd(q, k, v, cu_q, cu_k, max(p.seqlens_q()), max(p.seqlens_k()),
                                               causal=p.causal)
        r, o, lse = _call_noalloc(f, p, q, k, v, cu_q, cu_k, stream)
        assert r == mx.MXFA_OK, lib.mxfa_last_error()
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all()
        assert (o.float() - ref_o.float()).abs().max().item() <= 1e-2
        fin = torch.isfinite(ref_l)
        assert torch.equal(torch.isfinite(lse), fin)
        assert (lse[fin] - ref_l[fin]).abs().max().item() <= 1e-3

"""mxfa_attn_varlen_fwd_noalloc: the varlen forward for callers that cannot
allocate device memory when they run attention (plugins and services with a
fixed, pre-planned device memory budget, or code without access to the
allocator that owns the device).  Its scratch is a fixed array inside the
library, so the caller passes only inputs and outputs.

The GPU test calls the entry point through the C ABI on several problems in
a row (bf16 and f16 on the tensor cores, f32 on the CUDA cores, a batch with
an empty sequence).  Each result is checked against the fp64 oracle with the
parity tolerances and against mxfa_attn_varlen_fwd (the entry point that
takes a caller workspace), and the scratch array's status word is read
after every call.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import oracle
import workloads
from parity import compare

FAKE = 0x100000
DT = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


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
    r = lib.mxfa_attn_varlen_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 4096, 1 << 24, 1 << 24, 65536,
                                         65536, 8, 2, 128, 2, float("nan"), 1, None)
    assert r == mx.MXFA_ERR_WORKSPACE
    assert b"no-allocation" in lib.mxfa_last_error()


def test_rejected_arguments_are_reported_before_the_scratch_is_touched():
    """The argument checks of mxfa_attn_varlen_fwd come first (no device is
    needed to see them: nothing is launched, not even the header memset)."""
    mx, lib = _lib()
    # NULL cu_seqlens, Hq not a multiple of Hkv, an unsupported head dim
    assert lib.mxfa_attn_varlen_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, None, None, None, 2, 64, 64, 32, 32, 8, 2, 128,
                                            2, float("nan"), 1, None) == mx.MXFA_ERR_INVALID_ARG
    assert lib.mxfa_attn_varlen_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 64, 64, 32, 32, 6, 4, 128,
                                            2, float("nan"), 1, None) == mx.MXFA_ERR_INVALID_ARG
    assert lib.mxfa_attn_varlen_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 64, 64, 32, 32, 8, 2, 96,
                                            2, float("nan"), 1, None) == mx.MXFA_ERR_UNSUPPORTED


def _call_noalloc(lib, p, q, k, v, cu_q, cu_k, stream):
    o = torch.full_like(q, float("nan"))
    lse = torch.full((q.shape[0], p.hq), float("nan"), dtype=torch.float32, device=q.device)
    r = lib.mxfa_attn_varlen_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                         cu_q.data_ptr(), cu_k.data_ptr(), p.batch, p.total_q, p.total_k,
                                         max(p.seqlens_q()), max(p.seqlens_k()), p.hq, p.hkv, p.dqk, DT[q.dtype],
                                         float("nan"), int(p.causal), ctypes.c_void_p(stream.cuda_stream))
    return r, o, lse


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_workspace_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mx, lib = _lib()
    stream = torch.cuda.current_stream()
    problems = [
        workloads.varlen(31, [300, 17, 512, 1, 129], [300, 40, 512, 1, 129], 8, 2, 128, "bf16", True),
        workloads.varlen(32, [64, 700, 3], [80, 700, 3], 4, 4, 64, "f16", False),
        workloads.varlen(33, [40, 0, 97], [40, 12, 97], 4, 2, 64, "f32", True),  # CUDA-core path, an empty sequence
        workloads.varlen(34, [129, 0, 300], [129, 0, 310], 4, 1, 128, "bf16", True),  # a sequence without keys
    ]
    for p in problems:
        q, k, v = p.q.cuda(), p.k.cuda(), p.v.cuda()
        cu_q, cu_k = p.cu_q.cuda(), p.cu_k.cuda()
        ref_o, ref_l = mx.mxfa_attn_varlen_fwd(q, k, v, cu_q, cu_k, max(p.seqlens_q()), max(p.seqlens_k()),
                                               causal=p.causal)
        r, o, lse = _call_noalloc(lib, p, q, k, v, cu_q, cu_k, stream)
        assert r == mx.MXFA_OK, lib.mxfa_last_error()
        torch.cuda.synchronize()
        assert mx.read_noalloc_status(stream) == (mx.MXFA_OK, 0)
        ro, rl = oracle.problem(p)
        compare(o, lse, ro, rl, q.dtype, f"noalloc {p.name} {q.dtype}")
        tol = 1e-5 if q.dtype == torch.float32 else 1e-2
        assert (o.float() - ref_o.float()).abs().max().item() <= tol
        fin = torch.isfinite(ref_l)
        assert torch.equal(torch.isfinite(lse), fin)
        assert (lse[fin] - ref_l[fin]).abs().max().item() <= (1e-5 if q.dtype == torch.float32 else 1e-3)


@pytest.mark.gpu
def test_noalloc_status_reports_a_short_max_seqlen():
    """The scratch array's status word is readable: a sequence longer than
    max_seqlen_q is reported (MXFA_ERR_INVALID_ARG, site 0x201), and the next
    correct call starts clean."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mx, lib = _lib()
    stream = torch.cuda.current_stream()
    p = workloads.varlen(35, [1000, 10], [1000, 10], 4, 4, 128, "bf16", True)
    q, k, v = p.q.cuda(), p.k.cuda(), p.v.cuda()
    cu_q, cu_k = p.cu_q.cuda(), p.cu_k.cuda()
    o = torch.empty_like(q)
    r = lib.mxfa_attn_varlen_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), None,
                                         cu_q.data_ptr(), cu_k.data_ptr(), 2, p.total_q, p.total_k, 300, 1000, 4, 4,
                                         128, 2, float("nan"), 1, ctypes.c_void_p(stream.cuda_stream))
    assert r == mx.MXFA_OK
    assert mx.read_noalloc_status(stream) == (mx.MXFA_ERR_INVALID_ARG, 0x201)
    r, o, lse = _call_noalloc(lib, p, q, k, v, cu_q, cu_k, stream)
    assert r == mx.MXFA_OK
    assert mx.read_noalloc_status(stream) == (mx.MXFA_OK, 0)
    ro, rl = oracle.problem(p)
    compare(o, lse, ro, rl, q.dtype, "noalloc after a reported call")

"""Run a workloads.Problem through the library's public entry points (test/bench helper)."""
import tiled_attention_21_b200 as mx
from workloads import to_device as to_dev  # noqa: F401  (re-exported for the tests)


def run(p, d, entry=None, num_splits=0, stream=None, out=None, lse=None):
    """Returns (o, lse) in packed layout [total_q, Hq, Dv] / [total_q, Hq]."""
    entry = entry or ("decode" if p.mla else ("fwd" if p.batched else "varlen"))
    if entry == "fwd":
        B = p.batch
        Sq, Sk = p.total_q // B, p.total_k // B
        o, l = mx.mxfa_attn_fwd(d["q"].view(B, Sq, p.hq, p.dqk), d["k"].view(B, Sk, p.hkv, p.dqk),
                                d["v"].view(B, Sk, p.hkv, p.dv), causal=p.causal, softmax_scale=p.scale,
                                stream=stream,
                                out=None if out is None else out.view(B, Sq, p.hq, p.dv),
                                lse=None if lse is None else lse.view(B, Sq, p.hq))
        return o.view(p.total_q, p.hq, p.dv), l.view(p.total_q, p.hq)
    if entry == "varlen":
        return mx.mxfa_attn_varlen_fwd(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"], max(p.seqlens_q()),
                                       max(p.seqlens_k()), causal=p.causal, softmax_scale=p.scale, stream=stream,
                                       out=out, lse=lse)
    if p.kv_scale is not None:
        return mx.mxfa_attn_decode_mla_fp8kv(d["q"], d["kv"], p.kv_scale, d["cu_q"], d["cu_k"], max(p.seqlens_q()),
                                             max(p.seqlens_k()), softmax_scale=p.scale, causal=p.causal,
                                             num_splits=num_splits, stream=stream, out=out, lse=lse)
    return mx.mxfa_attn_decode_splitkv(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"], max(p.seqlens_q()),
                                       max(p.seqlens_k()), softmax_scale=p.scale, causal=p.causal,
                                       num_splits=num_splits, stream=stream, out=out, lse=lse)

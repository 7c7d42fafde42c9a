"""Host-side pieces of bench.py that need no GPU: the oracle baseline of the
MLA decode over an E4M3 cache, taken on whole sequences of the workload
(the oracle dequantises the cache it is given, so the sequences are cut out
of the workload first)."""
import importlib.util
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_sub_problem_rows_equal_the_full_problem_rows():
    """The oracle on sequences cut out of the workload gives, bit for bit, the
    rows the oracle gives for them in the whole workload (one sequence has
    no keys)."""
    b = _bench()
    p = workloads.mla_decode_fp8(3, 6, 2, 0, lens_kv=[5, 9, 0, 7, 3, 11])
    seqs = [4, 2, 1]
    sub = b._sub_problem(p, seqs)
    assert sub.kv_scale == p.kv_scale and sub.batch == len(seqs)
    assert sub.seqlens_k() == [p.seqlens_k()[s] for s in seqs]
    o_full, l_full = oracle.problem(p)
    o_sub, l_sub = oracle.problem(sub)
    cq = p.cu_q.tolist()
    idx = torch.tensor([r for s in seqs for r in range(cq[s], cq[s + 1])])
    assert torch.equal(o_sub, o_full[idx])
    assert torch.equal(l_sub, l_full[idx])


def test_fp8_decode_baseline_runs_whole_sequences():
    b = _bench()
    p = workloads.mla_decode_fp8(3, 8, 4, 256)
    cb = b.cpu_baseline_seqs(p, full_units=1e9, target_s=0.2, max_seqs=3)
    assert cb["kind"] == "oracle" and cb["unit"] == "GB/s" and cb["value"] > 0 and cb["cores"] >= 1
    assert "whole sequences" in cb["sample"]

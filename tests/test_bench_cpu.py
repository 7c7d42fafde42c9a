"""Host-side pieces of bench.py that need no GPU: the oracle baseline of the
MLA decode over an E4M3 cache, taken on whole sequences of the workload
(the oracle dequantises the cache it is given, so the sequences are cut out
of the workload first), and the roofline bookkeeping -- the causal-adjusted
work count, the visible keys of a sampled row, the algorithmic bytes of a
decode, and the recorded DRAM traffic that is reported only while the
kernel's sources are the ones it was captured on."""
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


def test_causal_adjusted_flops():
    """4*B*H*S^2*D/2 for a causal problem: the long-context headline is
    8.796 TFLOP, the batched 2K workload 68.72 GFLOP; a varlen problem is the
    sum of its sequences' counts."""
    b = _bench()
    assert b.prefill_flops(1, 32, 32768, 128) == 8796093022208.0
    assert round(b.prefill_flops(4, 16, 2048, 128) / 1e9, 2) == 68.72
    assert b.prefill_flops(2, 3, 10, 8, causal=False) == 2 * b.prefill_flops(2, 3, 10, 8)
    p = workloads.varlen(5, [3, 40, 17], [3, 40, 17], 4, 2, 64, "bf16", True)
    assert b.varlen_flops(p) == sum(b.prefill_flops(1, 4, L, 64) for L in (3, 40, 17))


def test_visible_keys_match_the_causal_mask():
    """The work count of a sampled row is its number of visible keys under the
    bottom-right causal mask (query i of a sequence sees key j iff
    j <= i + Sk - Sq), counted here by brute force."""
    b = _bench()
    p = workloads.varlen(6, [5, 9, 1, 12], [7, 9, 4, 3], 2, 2, 64, "bf16", True)
    pairs = torch.tensor([[t, 0] for t in range(p.total_q)])
    cq, ck = p.cu_q.tolist(), p.cu_k.tolist()
    want = []
    for s in range(p.batch):
        sq, sk = cq[s + 1] - cq[s], ck[s + 1] - ck[s]
        for i in range(sq):
            want.append(sum(1 for j in range(sk) if j <= i + sk - sq))
    assert b._visible_keys(p, pairs) == want


def test_decode_bytes_of_an_e4m3_cache():
    """The E4M3 cache counts one byte per element, the bf16 cache two; q, O
    and LSE are the same."""
    b = _bench()
    pf = workloads.mla_decode_fp8(3, 3, 4, 100)
    pb = workloads.mla_decode(3, 3, 4, 100)
    assert b.decode_bytes(pb) - b.decode_bytes(pf) == pf.kv.numel()


def test_recorded_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    """A recorded DRAM traffic figure is reported only while the sources it
    was captured on are unchanged (hash of the kernel's own headers)."""
    import json
    import shutil
    b = _bench()
    csrc = tmp_path / "tiled_attention_21_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "tiled_attention_21_b200", "csrc"), csrc)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    h = b.kernel_hash("decode_gqa")
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"decode_gqa": {"w": {"dram_bytes_per_launch": 123, "source_hash": h}}}))
    assert b.recorded_traffic("decode_gqa", "w") == 123
    assert b.recorded_traffic("decode_gqa", "other") is None
    with open(csrc / "decode_gqa.cuh", "a") as f:
        f.write("\n// changed\n")
    assert b.recorded_traffic("decode_gqa", "w") is None

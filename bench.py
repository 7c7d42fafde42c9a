"""Benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxfa|reference]

The headline step is one attention forward of the long-context causal
prefill (bf16, B=1, Hq=Hkv=32, Sq=Sk=32768, D=128, seed 4), the largest
workload that fits one GPU, through the library's tensor-core path; the
metric is causal-adjusted TFLOP/s (4*B*H*S^2*D / 2 per step).  The same run
measures, each as a sub-object of the one JSON line with its own roofline,
end-to-end number, oracle CPU baseline and clock record:
  batched_causal    bf16, B=4, H=16, S=2048, D=128, causal (seed 1)
  varlen_gqa        bf16 varlen, 16 sequences U[128, 4096] (seed 2),
                    Hq=32, Hkv=8, D=128, causal; the schedule kernel that
                    precedes the attention kernel is inside the timed call
  single_head_fp32  fp32, B=1, H=1, S=128, D=64, non-causal (seed 0): us
                    per call on the exact CUDA-core kernel
  decode            MLA split-KV decode, bf16, batch 128, q_len 4, 16 heads,
                    576/512, kv_len 8192 (seed 3), in KV GB/s
  decode_mla_q8     the same with q_len 8 (128 query rows per sequence:
                    two head groups), batch 64
  decode_gqa        grouped-query decode, q_len 1, Hq 32, Hkv 4, D 128, kv 8192
  decode_fp8        the MLA decode over an E4M3 cache
Inputs are synthetic (workloads.py).  L2 is flushed (a 512 MiB write)
before every timed prefill step, outside the timed interval; the decode
inputs (0.6-1.2 GB) are larger than L2.  With --gpus N (under torchrun)
every rank runs its own replica (no collective on the data path; weak
scaling) and each time is the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores on bounded
samples of the headline workload (the reference arm; there is no reference
library to run).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import itertools
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "attn fwd TFLOP/s (causal-adjusted) & decode KV GB/s, % of B200 roofline"
HEADLINE = dict(B=1, H=32, S=32768, D=128)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def prefill_flops(B, H, S, D, causal=True):
    f = 4.0 * B * H * S * S * D
    return f / 2 if causal else f


def varlen_flops(p):
    """Conventional causal-adjusted work of a varlen problem: 4*Hq*D*L^2/2 per sequence."""
    f = sum(4.0 * p.hq * p.dqk * L * L for L in p.seqlens_q())
    return f / 2 if p.causal else f


def decode_bytes(p):
    """Algorithmic bytes of one decode: the KV cache once (MLA: the shared
    latent rows; grouped-query: K and V), q, O and LSE."""
    es = 2
    if p.kv_scale is not None:  # E4M3 latent cache: one byte per element
        kv = p.kv.numel()
    else:
        kv = p.kv.numel() * es if p.mla else (p.k.numel() + p.v.numel()) * es
    return kv + p.q.numel() * es + p.total_q * p.hq * p.dv * es + p.total_q * p.hq * 4


# Source files that define each measured kernel (its own header and the
# headers it includes); a recorded ncu capture is valid while they are unchanged.
KERNEL_SOURCES = {
    "attn_fwd_tc_kernel": ["prefill_tc.cuh", "exp2_poly.cuh", "ptx.cuh", "common.cuh"],
    "decode": ["decode_tc.cuh", "ptx.cuh", "common.cuh"],
    "decode_gqa": ["decode_gqa.cuh", "decode_tc.cuh", "ptx.cuh", "common.cuh"],
}


def kernel_hash(kernel: str):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_attention_21_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on
    the current sources of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != kernel_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n):
    """One process per GPU (RANK / WORLD_SIZE / LOCAL_RANK / MASTER_* from the
    launcher).  The data path has no collective: the process group carries
    only the timing barrier and the max over ranks.  NCCL on GPUs; gloo on a
    host without one (the multi-process tests)."""
    if n <= 1 and "RANK" not in os.environ:
        return 0, 1, 0
    import torch.distributed as dist
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    from datetime import timedelta
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_rate(units_per_step, steps, world, t_ms):
    """Whole-job throughput of `world` replicas that each process
    `units_per_step` per step: all ranks' units over the slowest rank's time
    (`t_ms`, the max over ranks of the timed steps)."""
    return units_per_step * steps * world / (t_ms / 1e3)


def time_steps(fn, steps, warmup, flush, stream, world):
    """Per-step CUDA-event times (ms) on `stream`; `flush` before each step,
    outside the timed interval."""
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


# ---------------------------------------------------------------- CPU baseline (the oracle, timed)
def _visible_keys(p, pairs):
    """Visible keys of each sampled (token, head) row (bottom-right causal)."""
    cq, ck = p.cu_q.tolist(), p.cu_k.tolist()
    out = []
    import bisect
    for tok in pairs[:, 0].tolist():
        b = bisect.bisect_right(cq, tok) - 1
        sq, sk, i = cq[b + 1] - cq[b], ck[b + 1] - ck[b], tok - cq[b]
        out.append(sk if not p.causal else max(0, min(sk, i + 1 + sk - sq)))
    return out


def _sample_pairs(p, n, seed):
    """n (token, head) rows of problem p drawn uniformly with a seeded generator."""
    g = torch.Generator("cpu").manual_seed(seed)
    tok = torch.randint(0, p.total_q, (n,), generator=g)
    hd = torch.randint(0, p.hq, (n,), generator=g)
    return torch.stack([tok, hd], 1)


def cpu_baseline(p, kind: str, target_s: float = 8.0, full_units=None):
    """The fp64 oracle as it stands on the host cores over a bounded random
    sample of (token, head) rows of workload `p`, scaled to the metric's
    unit.  kind "flops": TFLOP/s of the contraction work of the rows
    evaluated, 2*(Dqk+Dv) per visible (query, key) pair (4*D for Dqk = Dv,
    as in the causal-adjusted metric); kind "bytes": the workload's
    algorithmic bytes `full_units` in proportion to the rows evaluated, in
    GB/s."""
    import oracle
    threads = oracle.default_threads()
    n_rows = p.total_q * p.hq

    def run(n, seed):
        pairs = _sample_pairs(p, n, seed)
        t0 = time.perf_counter()
        oracle.problem(p, pairs=pairs, threads=threads)
        return time.perf_counter() - t0, pairs

    t, pairs = run(4 * threads, 7)
    n = int(max(threads, min(n_rows, pairs.shape[0] * target_s / max(t, 1e-3))))
    t, pairs = run(n, 8)
    rows = pairs.shape[0]
    if kind == "flops":
        work = sum(2.0 * (p.dqk + p.dv) * nv for nv in _visible_keys(p, pairs))
        value, unit = work / t / 1e12, "TFLOP/s"
    else:
        value, unit = full_units * rows / n_rows / t / 1e9, "GB/s"
    return {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
            "sample": f"{rows} random (token, head) rows of the {n_rows} of {p.name}, fp64, {t:.1f} s wall" +
                      ("; rate = the workload's algorithmic bytes x rows evaluated / all rows" if kind == "bytes"
                       else "; work = 2*(Dqk+Dv) per visible (query, key) pair")}


def _sub_problem(p, seqs):
    """Decode workload `p` cut down to the sequences `seqs`: their query rows
    and their rows of the latent cache, with the cumulative lengths rebuilt
    (input selection only; the oracle does all the arithmetic)."""
    cq, ck = p.cu_q.tolist(), p.cu_k.tolist()
    cu = lambda lens: torch.tensor([0] + list(itertools.accumulate(lens)), dtype=torch.int32)
    q = torch.cat([p.q[cq[b]:cq[b + 1]] for b in seqs])
    kv = torch.cat([p.kv[ck[b]:ck[b + 1]] for b in seqs])
    tk = kv.shape[0]
    return dataclasses.replace(p, name=f"{p.name}[{len(seqs)} sequences]", q=q, kv=kv,
                               k=kv.view(tk, 1, p.dqk), v=kv[:, :p.dv].view(tk, 1, p.dv),
                               cu_q=cu([cq[b + 1] - cq[b] for b in seqs]),
                               cu_k=cu([ck[b + 1] - ck[b] for b in seqs]), check_rows=None, meta={})


def cpu_baseline_seqs(p, full_units, target_s: float = 6.0, max_seqs: int = 16):
    """The fp64 oracle on a seeded random sample of whole sequences of the
    MLA decode workload `p` over an E4M3 cache, all their rows.  The oracle
    dequantises the cache it is given, so a row sample of the whole workload
    would decode all its codes per call; a sub-problem of a few sequences
    decodes only theirs (at most max_seqs, to bound the fp64 copy in host
    memory).  GB/s: the workload's algorithmic bytes `full_units` in
    proportion to the (token, head) rows evaluated."""
    import oracle
    threads = oracle.default_threads()
    order = torch.randperm(p.batch, generator=torch.Generator("cpu").manual_seed(9)).tolist()

    def run(k):
        sub = _sub_problem(p, order[:k])
        t0 = time.perf_counter()
        oracle.problem(sub, threads=threads)
        return time.perf_counter() - t0, sub

    t, _ = run(1)
    k = int(max(1, min(p.batch, max_seqs, target_s / max(t, 1e-3))))
    t, sub = run(k)
    rows, n_rows = sub.total_q * sub.hq, p.total_q * p.hq
    return {"value": full_units * rows / n_rows / t / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{k} random whole sequences of {p.name} ({rows} of its {n_rows} (token, head) rows, "
                      f"their {sub.total_k} cache rows dequantised), fp64, {t:.1f} s wall; rate = the workload's "
                      f"algorithmic bytes x rows evaluated / all rows"}


def cpu_baseline_full_us(p, target_s: float = 3.0):
    """The oracle on the whole (small) problem, repeated for about target_s: us per call."""
    import oracle
    threads = oracle.default_threads()
    oracle.problem(p, threads=threads)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < target_s:
        oracle.problem(p, threads=threads)
        n += 1
    t = time.perf_counter() - t0
    return {"value": t / n * 1e6, "unit": "us", "cores": threads, "kind": "oracle",
            "sample": f"the whole problem ({p.total_q * p.hq} rows), {n} calls, fp64, {t:.1f} s wall"}


def headline_problem():
    return workloads.cfg_long_causal(S=HEADLINE["S"], H=HEADLINE["H"])


def headline_config(p, flops, world):
    return headline_config_of(p.name, flops, world)


def headline_config_of(name, flops, world):
    return {"workload": name, "B": HEADLINE["B"], "H": HEADLINE["H"], "seq_len": HEADLINE["S"],
            "head_dim": HEADLINE["D"], "causal": True, "flops_per_step": flops,
            "l2": "flushed before every step (512 MiB write); inputs (805 MB q, k, v) are larger than L2",
            "parallelism": f"replicas x{world}"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    p = headline_problem()
    flops = prefill_flops(HEADLINE["B"], HEADLINE["H"], HEADLINE["S"], HEADLINE["D"])
    per_step = args.sample_seconds if args.sample_seconds else max(2.0, 60.0 / max(1, args.steps + args.warmup))
    res = [cpu_baseline(p, "flops", target_s=per_step) for _ in range(args.warmup + args.steps)]
    vals = [r["value"] for r in res[args.warmup:]]
    v = statistics.mean(vals)
    cb = dict(res[-1])
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": headline_config(p, flops, world),
            "host_note": "the oracle runs on the host cores on sampled rows of this workload; "
                         "the config's L2 policy is the GPU arm's",
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- legs
class Bench:
    def __init__(self, args, world, local, dev, stream):
        import tiled_attention_21_b200 as mx
        self.mx = mx
        self.args, self.world, self.local, self.dev, self.stream = args, world, local, dev, stream
        self.flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.pk, self.pk_kind = peaks()
        self.rank0_cpu = world == 1 and not args.no_cpu_baseline

    def flush(self):
        self.flush_buf.zero_()

    def timed(self, fn, steps, warmup=3, flush=True):
        """(per-step times, clock summary); the times of the slowest rank."""
        with ClockSampler(self.local) as clk:
            times = time_steps(fn, steps, warmup, self.flush if flush else (lambda: None), self.stream,
                               self.world)
        return times, clk.summary()

    def check_status(self, ws):
        st, site = self.mx.read_device_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {st} at site 0x{site:x}")

    def tensor_roofline(self, flops, kern_ms, kernel, workload):
        achieved = flops / (kern_ms / 1e3) / 1e12
        peak = self.pk["bf16_tflops"]
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": recorded_traffic("attn_fwd_tc_kernel", workload), "kernel": kernel,
                "peak_kind": f"{self.pk_kind} burst dense bf16 (cuBLAS)"}

    def hbm_roofline(self, nbytes, kern_ms, kernel_key, workload):
        gbs = nbytes / (kern_ms / 1e3) / 1e9
        peak = self.pk["hbm_gbs"]
        return {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                "traffic": recorded_traffic(kernel_key, workload), "peak_kind": f"{self.pk_kind} HBM copy"}

    # -------- batched prefill (headline and batched_causal)
    def batched_prefill(self, p, steps, cpu=True):
        mx, dev, stream, world = self.mx, self.dev, self.stream, self.world
        B = p.meta["B"]
        S, H, D = p.meta["Sq"], p.hq, p.dqk
        q = p.q.view(B, S, H, D).to(dev)
        k = p.k.view(B, S, H, D).to(dev)
        v = p.v.view(B, S, H, D).to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((B, S, H), dtype=torch.float32, device=dev)
        ws = mx.workspace(256, dev)

        def step():
            mx.mxfa_attn_fwd(q, k, v, causal=True, out=o, lse=lse, ws=ws, stream=stream)

        flops = prefill_flops(B, H, S, D)
        times, clocks = self.timed(step, steps, self.args.warmup)
        self.check_status(ws)
        t_ms = max_over_ranks(sum(times), world)
        kern_ms = max_over_ranks(statistics.mean(times), world)  # one kernel launch per step
        res = {"workload": p.name, "value": job_rate(flops, steps, world, t_ms) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": t_ms / steps, "steps": steps, "flops_per_step": flops,
               "roofline": self.tensor_roofline(flops, kern_ms, f"attn_fwd_tc_kernel<{D},bf16>", p.name),
               "clocks": clocks, "gpu_launches": steps}
        # end to end through the public API with host buffers
        hq, hk, hv = (t.view(B, S, H, D).pin_memory() for t in (p.q, p.k, p.v))
        ho = torch.empty((B, S, H, D), dtype=torch.bfloat16).pin_memory()
        hl = torch.empty((B, S, H), dtype=torch.float32).pin_memory()
        dq, dk, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv_.copy_(hv, non_blocking=True)
            mx.mxfa_attn_fwd(dq, dk, dv_, causal=True, out=o, lse=lse, ws=ws, stream=stream)
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        n_e2e = max(5, steps // 3)
        e2e_times, _ = self.timed(e2e_step, n_e2e, 2)
        e2e_ms = max_over_ranks(sum(e2e_times), world)
        res["e2e"] = {"value": job_rate(flops, n_e2e, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
                      "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o.numel() * 2 + lse.numel() * 4}
        res["cpu_baseline"] = cpu_baseline(p, "flops") if (cpu and self.rank0_cpu) else None
        del q, k, v, o, dq, dk, dv_
        return res

    # -------- varlen prefill (varlen_gqa)
    def varlen_prefill(self, p, steps):
        mx, dev, stream, world = self.mx, self.dev, self.stream, self.world
        d = workloads.to_device(p, dev)
        o = torch.empty_like(d["q"])
        lse = torch.empty((p.total_q, p.hq), dtype=torch.float32, device=dev)
        max_q, max_k = max(p.seqlens_q()), max(p.seqlens_k())
        ws = mx.workspace(mx.load().mxfa_attn_varlen_fwd_workspace_size(p.batch, max_q, max_k, p.hq, p.dqk, 2), dev)

        def step():
            mx.mxfa_attn_varlen_fwd(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"], max_q, max_k, causal=True,
                                    out=o, lse=lse, ws=ws, stream=stream)

        flops = varlen_flops(p)
        times, clocks = self.timed(step, steps, self.args.warmup)
        self.check_status(ws)
        t_ms = max_over_ranks(sum(times), world)
        kern_ms = max_over_ranks(statistics.mean(times), world)
        res = {"workload": p.name, "value": job_rate(flops, steps, world, t_ms) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": t_ms / steps, "steps": steps, "flops_per_step": flops,
               "roofline": self.tensor_roofline(flops, kern_ms, "attn_fwd_tc_kernel<128,bf16> (+ prefill_prep_kernel)",
                                                p.name),
               "clocks": clocks, "gpu_launches": 2 * steps,
               "l2": "flushed before every step (512 MiB write)"}
        hq, hk, hv = p.q.pin_memory(), p.k.pin_memory(), p.v.pin_memory()
        hcq, hck = p.cu_q.pin_memory(), p.cu_k.pin_memory()
        ho, hl = torch.empty_like(hq).pin_memory(), torch.empty((p.total_q, p.hq), dtype=torch.float32).pin_memory()
        dq, dk, dv_ = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
        dcq, dck = torch.empty_like(d["cu_q"]), torch.empty_like(d["cu_k"])

        def e2e_step():
            for dst, src in ((dq, hq), (dk, hk), (dv_, hv), (dcq, hcq), (dck, hck)):
                dst.copy_(src, non_blocking=True)
            mx.mxfa_attn_varlen_fwd(dq, dk, dv_, dcq, dck, max_q, max_k, causal=True, out=o, lse=lse, ws=ws,
                                    stream=stream)
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        n_e2e = max(5, steps // 3)
        e2e_times, _ = self.timed(e2e_step, n_e2e, 2)
        e2e_ms = max_over_ranks(sum(e2e_times), world)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcq, hck))
        res["e2e"] = {"value": job_rate(flops, n_e2e, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": ho.numel() * 2 + hl.numel() * 4}
        res["cpu_baseline"] = cpu_baseline(p, "flops") if self.rank0_cpu else None
        return res

    # -------- the fp32 single-head problem (us per call)
    def single_head(self, p, steps):
        mx, dev, stream, world = self.mx, self.dev, self.stream, self.world
        S, D = p.meta["Sq"], p.dqk
        q, k, v = (t.view(1, S, 1, D).to(dev) for t in (p.q, p.k, p.v))
        o = torch.empty_like(q)
        lse = torch.empty((1, S, 1), dtype=torch.float32, device=dev)
        ws = mx.workspace(256, dev)

        def call():  # on the current stream: the capture stream inside the graph capture below
            mx.mxfa_attn_fwd(q, k, v, causal=False, softmax_scale=p.scale, out=o, lse=lse, ws=ws)

        # A call is a few microseconds of GPU work, less than the host time of
        # the binding's argument marshalling: each timed step replays the call
        # from a CUDA graph, so the interval measures the device, not Python.
        for _ in range(2):
            call()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call()
        times, clocks = self.timed(graph.replay, steps, self.args.warmup)
        self.check_status(ws)
        us = max_over_ranks(statistics.mean(times), world) * 1e3
        flops = prefill_flops(1, 1, S, D, causal=False)
        res = {"workload": p.name, "value": us, "unit": "us", "higher_is_better": False, "steps": steps,
               "tflops": flops / (us / 1e6) / 1e12, "kernel": "attn_fwd_simt_kernel<float> (fp32, CUDA cores)",
               "timing": "each step one replay of the call captured in a CUDA graph (device time per call)",
               "bound": "launch latency (4.19 MFLOP)", "clocks": clocks, "gpu_launches": steps,
               "l2": "flushed before every call (512 MiB write)"}
        hq, hk, hv = (t.view(1, S, 1, D).pin_memory() for t in (p.q, p.k, p.v))
        ho, hl = torch.empty_like(hq).pin_memory(), torch.empty((1, S, 1), dtype=torch.float32).pin_memory()
        dq, dk, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv_.copy_(hv, non_blocking=True)
            mx.mxfa_attn_fwd(dq, dk, dv_, causal=False, softmax_scale=p.scale, out=o, lse=lse, ws=ws, stream=stream)
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        e2e_times, _ = self.timed(e2e_step, steps, 2)
        res["e2e"] = {"value": max_over_ranks(statistics.mean(e2e_times), world) * 1e3, "unit": "us",
                      "h2d_bytes_per_step": 3 * q.numel() * 4, "d2h_bytes_per_step": o.numel() * 4 + lse.numel() * 4}
        res["cpu_baseline"] = cpu_baseline_full_us(p) if self.rank0_cpu else None
        return res

    # -------- decode legs
    def decode(self, p, steps, kind):
        mx, dev, stream, world = self.mx, self.dev, self.stream, self.world
        lib = mx.load()
        d = workloads.to_device(p, dev)
        od = torch.empty((p.total_q, p.hq, p.dv), dtype=torch.bfloat16, device=dev)
        ld = torch.empty((p.total_q, p.hq), dtype=torch.float32, device=dev)
        max_q, max_k = max(p.seqlens_q()), max(p.seqlens_k())
        if kind == "fp8":
            need = lib.mxfa_attn_decode_mla_fp8kv_workspace_size(p.batch, max_q, p.hq, max_k, 0)
        else:
            need = lib.mxfa_attn_decode_splitkv_workspace_size(p.batch, max_q, p.hq, p.hkv, p.dv, max_k, 0, 2)
        wsd = torch.zeros(need + 256, dtype=torch.uint8, device=dev)

        def call(dd, out, lse):
            if kind == "fp8":
                mx.mxfa_attn_decode_mla_fp8kv(dd["q"], dd["kv"], p.kv_scale, dd["cu_q"], dd["cu_k"], max_q, max_k,
                                              softmax_scale=p.scale, out=out, lse=lse, ws=wsd, stream=stream)
            else:
                mx.mxfa_attn_decode_splitkv(dd["q"], dd["k"], dd["v"], dd["cu_q"], dd["cu_k"], max_q, max_k,
                                            softmax_scale=p.scale, out=out, lse=lse, ws=wsd, stream=stream)

        times, clocks = self.timed(lambda: call(d, od, ld), steps, 3, flush=False)
        self.check_status(wsd)
        nbytes = decode_bytes(p)
        ms = max_over_ranks(statistics.mean(times), world)
        gbs = nbytes / (ms / 1e3) / 1e9
        key = "decode_gqa" if kind == "gqa" else "decode"
        res = {"workload": p.name, "value": gbs * world, "unit": "GB/s", "ms_per_step": ms, "steps": steps,
               "algorithmic_bytes": nbytes, "kv_rows_per_s": p.total_k * world / (ms / 1e3),
               "l2": "inputs larger than L2", "roofline": self.hbm_roofline(nbytes, ms, key, p.name),
               "clocks": clocks, "gpu_launches": 3 * steps}
        # end to end: every input (q, the KV cache, the indptr arrays) copied
        # from pinned host memory and O, LSE read back, every step
        hsrc = {"q": p.q, "cu_q": p.cu_q, "cu_k": p.cu_k}
        if p.mla:
            hsrc["kv"] = p.kv
        else:
            hsrc["k"], hsrc["v"] = p.k, p.v
        hsrc = {n: t.contiguous().pin_memory() for n, t in hsrc.items()}
        dsrc = {n: torch.empty_like(t, device=dev) for n, t in hsrc.items()}
        if p.mla:
            dsrc["k"] = dsrc["kv"].view(-1, 1, p.dqk)
            dsrc["v"] = dsrc["kv"][:, :p.dv].view(-1, 1, p.dv)
        ho, hl = torch.empty(od.shape, dtype=od.dtype).pin_memory(), torch.empty(ld.shape).pin_memory()

        def e2e_step():
            for n, t in hsrc.items():
                dsrc[n].copy_(t, non_blocking=True)
            call(dsrc, od, ld)
            ho.copy_(od, non_blocking=True)
            hl.copy_(ld, non_blocking=True)

        n_e2e = 5
        e2e_times, _ = self.timed(e2e_step, n_e2e, 2, flush=False)
        e2e_ms = max_over_ranks(statistics.mean(e2e_times), world)
        res["e2e"] = {"value": nbytes * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                      "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hsrc.values()),
                      "d2h_bytes_per_step": ho.numel() * 2 + hl.numel() * 4,
                      "note": "the KV cache crosses PCIe every step here; in serving it stays resident"}
        if not self.rank0_cpu:
            res["cpu_baseline"] = None
        elif kind == "fp8":
            res["cpu_baseline"] = cpu_baseline_seqs(p, nbytes)
        else:
            res["cpu_baseline"] = cpu_baseline(p, "bytes", full_units=nbytes)
        del d, dsrc
        return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mxfa", choices=["mxfa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None,
                    choices=["headline", "batched_causal", "varlen_gqa", "single_head_fp32", "decode", "mla_q8", "gqa",
                             "fp8"],
                    help="time one workload only (used for profiling captures; no JSON contract line)")
    ap.add_argument("--sample-seconds", type=float, default=None,
                    help="reference arm: seconds of oracle work per step (default: about a minute in all)")
    ap.add_argument("--decode-batch", type=int, default=128,
                    help="sequences of the MLA decode workloads (128 = the full workload; smaller for captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        run_reference(args, rank, int(os.environ.get("WORLD_SIZE", 1)))
        return

    rank, world, local = dist_setup(args.gpus)
    import tiled_attention_21_b200 as mx
    mx.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    bn = Bench(args, world, local, dev, stream)
    want = (lambda name: args.only in (None, name))
    out = {}

    if want("headline"):
        out["headline"] = bn.batched_prefill(headline_problem(), args.steps)
    if want("batched_causal"):
        out["batched_causal"] = bn.batched_prefill(workloads.cfg_batched_causal(), args.steps)
    if want("varlen_gqa"):
        out["varlen_gqa"] = bn.varlen_prefill(workloads.cfg_varlen_gqa(), args.steps)
    if want("single_head_fp32"):
        out["single_head_fp32"] = bn.single_head(workloads.cfg_single_head_fp32(), args.steps)
    dsteps = max(5, args.steps // 2)
    if want("decode"):
        pdc = (workloads.cfg_mla_decode() if args.decode_batch == 128 else
               workloads.mla_decode(3, args.decode_batch, 4, 8192,
                                    name=f"mla_decode_b{args.decode_batch}_q4_h16_kv8192_bf16"))
        out["decode"] = bn.decode(pdc, dsteps, "mla")
    if want("mla_q8"):
        # 8 queries x 16 heads = 128 query rows per sequence: two head groups
        # on the tensor-core kernel, each streaming the latent cache
        out["decode_mla_q8"] = bn.decode(workloads.mla_decode(3, 64, 8, 8192, name="mla_decode_b64_q8_h16_kv8192_bf16"),
                                         dsteps, "mla")
        out["decode_mla_q8"]["note"] = ("algorithmic bytes count the cache once; the two head groups of a sequence "
                                        "each stream it, the second mostly from L2")
    if want("gqa"):
        out["decode_gqa"] = bn.decode(workloads.cfg_gqa_decode(), dsteps, "gqa")
    if want("fp8"):
        pf = (workloads.cfg_mla_decode_fp8() if args.decode_batch == 128 else
              workloads.mla_decode_fp8(3, args.decode_batch, 4, 8192,
                                       name=f"mla_decode_b{args.decode_batch}_q4_h16_kv8192_fp8kv"))
        out["decode_fp8"] = bn.decode(pf, dsteps, "fp8")
        out["decode_fp8"]["mma_tflops"] = (2.0 * pf.total_q * pf.hq * (pf.total_k // pf.batch) * (pf.dqk + pf.dv)
                                           / (out["decode_fp8"]["ms_per_step"] / 1e3) / 1e12)

    if rank == 0:
        if args.only is not None:
            print(json.dumps(out), flush=True)
        else:
            h = out.pop("headline")
            line = {"metric": METRIC, "value": h["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                    "warmup": args.warmup, "ms_per_step": h["ms_per_step"], "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                    "config": headline_config_of(h["workload"], h["flops_per_step"], world),
                    "roofline": h["roofline"], "cpu_baseline": h["cpu_baseline"], "e2e": h["e2e"],
                    "gpu_launches": h["gpu_launches"], "clocks": h["clocks"]}
            line.update(out)
            print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

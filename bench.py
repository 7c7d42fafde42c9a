"""Benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxfa|reference]

One step = one attention forward of the batched causal prefill workload
(bf16, B=4, Hq=Hkv=16, Sq=Sk=2048, D=128, seed 1) through the library's
tensor-core path; the metric is causal-adjusted TFLOP/s (4*B*H*S^2*D / 2
per step).  The same run also measures the MLA split-KV decode workload
(bf16, batch 128, q_len 4, 16 heads, 576/512, kv_len 8192, seed 3) in KV
GB/s, reported under "decode".  Inputs are synthetic (workloads.py); L2 is
flushed (a 512 MiB write) before every timed step, outside the timed
interval.  With --gpus N (under torchrun) every rank runs its own replica
(no collective on the data path; weak scaling) and the time is the max
over ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the reference arm; there is no reference
library to run).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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
PREFILL_CFG = dict(B=4, H=16, S=2048, D=128)
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
    """Per-step CUDA-event times (ms) on `stream`; L2 flushed before each step."""
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


def cpu_baseline_prefill(target_s: float = 12.0):
    """The fp64 oracle on host cores over a bounded sample of the prefill
    workload: random (token, head) rows, throughput in causal-adjusted
    TFLOP/s of the rows evaluated (4*D*visible keys per row)."""
    import oracle
    p = workloads.cfg_batched_causal()
    threads = oracle.default_threads()
    S, D = PREFILL_CFG["S"], PREFILL_CFG["D"]

    def run(n, seed):
        pairs = workloads.sample_rows(p, max(1, n // p.hq), seed)
        i_local = pairs[:, 0] % S
        flops = float((4 * D * (i_local + 1)).sum())
        t0 = time.perf_counter()
        oracle.problem(p, pairs=pairs, threads=threads)
        return time.perf_counter() - t0, flops, pairs.shape[0]

    t, f, n = run(256, 7)
    n2 = int(max(256, min(200000, n * target_s / max(t, 1e-3))))
    t, f, n = run(n2, 8)
    return {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} random (token, head) rows of the B=4 H=16 S=2048 D=128 causal workload "
                      f"(plus first/last rows), fp64, {t:.1f} s wall"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    res = [cpu_baseline_prefill(target_s=max(2.0, 60.0 / max(1, args.steps + args.warmup))) for _ in
           range(args.warmup + args.steps)]
    vals = [r["value"] for r in res[args.warmup:]]
    v = statistics.mean(vals)
    cb = dict(res[-1])
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "batched_causal_b4_h16_s2048_d128_bf16", "l2": "n/a (host)"},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mxfa", choices=["mxfa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=128,
                    help="sequences of the MLA decode workload (128 = the full workload; smaller for captures)")
    ap.add_argument("--only", choices=["prefill", "decode", "gqa", "fp8"], default=None,
                    help="time one workload only (used for profiling captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        run_reference(args, rank, int(os.environ.get("WORLD_SIZE", 1)))
        return

    rank, world, local = dist_setup(args.gpus)
    import tiled_attention_21_b200 as mx
    mx.load()
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from runners import to_dev

    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.zero_()

    pk, pk_kind = peaks()

    # ---------------- prefill (the step)
    B, H, S, D = PREFILL_CFG["B"], PREFILL_CFG["H"], PREFILL_CFG["S"], PREFILL_CFG["D"]
    p = workloads.cfg_batched_causal()
    q = p.q.view(B, S, H, D).to(dev)
    k = p.k.view(B, S, H, D).to(dev)
    v = p.v.view(B, S, H, D).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, S, H), dtype=torch.float32, device=dev)
    ws = mx.workspace(256, dev)

    def step():
        mx.mxfa_attn_fwd(q, k, v, causal=True, out=o, lse=lse, ws=ws, stream=stream)

    flops = prefill_flops(B, H, S, D)
    if args.only in ("decode", "gqa", "fp8"):
        args.steps = 0
    with ClockSampler(local) as clk:
        times = time_steps(step, args.steps, args.warmup, flush, stream, world)
    st, site = mx.read_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} at site 0x{site:x}")
    t_ms = max_over_ranks(sum(times), world) if times else float("nan")
    ms_per_step = t_ms / max(1, args.steps)
    value = job_rate(flops, args.steps, world, t_ms) / 1e12 if times else float("nan")
    kern_ms = statistics.mean(times) if times else float("nan")  # one kernel launch per step
    achieved = flops / (kern_ms / 1e3) / 1e12
    traffic = recorded_traffic("attn_fwd_tc_kernel", "batched_causal_b4_h16_s2048_d128_bf16")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"], "traffic": traffic, "kernel": "attn_fwd_tc_kernel<128,bf16>",
                "peak_kind": f"{pk_kind} burst dense bf16 (cuBLAS)"}

    # ---------------- e2e through the public API with host buffers
    hq = p.q.view(B, S, H, D).pin_memory()
    hk = p.k.view(B, S, H, D).pin_memory()
    hv = p.v.view(B, S, H, D).pin_memory()
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

    e2e_times = time_steps(e2e_step, max(5, args.steps // 3), 3, flush, stream, world) if args.only is None else [1.0]
    e2e_ms = max_over_ranks(sum(e2e_times), world)
    e2e_val = flops * len(e2e_times) * world / (e2e_ms / 1e3) / 1e12
    h2d = 3 * q.numel() * 2
    d2h = o.numel() * 2 + lse.numel() * 4

    # ---------------- decode (secondary measurement)
    decode = None
    if not args.no_decode and args.only in (None, "decode"):
        pdc = (workloads.cfg_mla_decode() if args.decode_batch == 128 else
               workloads.mla_decode(3, args.decode_batch, 4, 8192, name=f"mla_decode_b{args.decode_batch}_q4_h16_kv8192_bf16"))
        dd = to_dev(pdc, dev)
        od = torch.empty((pdc.total_q, pdc.hq, pdc.dv), dtype=torch.bfloat16, device=dev)
        ld = torch.empty((pdc.total_q, pdc.hq), dtype=torch.float32, device=dev)
        need = mx.load().mxfa_attn_decode_splitkv_workspace_size(pdc.batch, 4, pdc.hq, 1, pdc.dv, 8192, 0, 2)
        wsd = torch.zeros(need + 256, dtype=torch.uint8, device=dev)

        def dstep():
            mx.mxfa_attn_decode_splitkv(dd["q"], dd["k"], dd["v"], dd["cu_q"], dd["cu_k"], 4, 8192,
                                        softmax_scale=pdc.scale, out=od, lse=ld, ws=wsd, stream=stream)

        dsteps = max(5, args.steps // 3)
        dtimes = time_steps(dstep, dsteps, 3, lambda: None, stream, world)  # KV (1.2 GB) >> L2
        dbytes = decode_bytes(pdc)
        dms = max_over_ranks(statistics.mean(dtimes), world)
        dgbs = dbytes / (dms / 1e3) / 1e9
        decode = {"workload": pdc.name, "value": dgbs * world, "unit": "GB/s", "ms_per_step": dms,
                  "algorithmic_bytes": dbytes, "l2": "inputs (1.2 GB KV) larger than L2",
                  "roofline": {"bound": "hbm", "achieved": dgbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                               "frac": dgbs / pk["hbm_gbs"],
                               "traffic": recorded_traffic("decode", "mla_decode_b128_q4_h16_kv8192_bf16"),
                               "peak_kind": f"{pk_kind} HBM copy"}}

    # ---------------- grouped-query decode (next scope row; secondary measurement)
    decode_gqa = None
    if not args.no_decode and args.only in (None, "gqa"):
        pg = workloads.cfg_gqa_decode()
        dg = to_dev(pg, dev)
        og = torch.empty((pg.total_q, pg.hq, pg.dv), dtype=torch.bfloat16, device=dev)
        lg = torch.empty((pg.total_q, pg.hq), dtype=torch.float32, device=dev)
        kvl = pg.total_k // pg.batch
        need = mx.load().mxfa_attn_decode_splitkv_workspace_size(pg.batch, 1, pg.hq, pg.hkv, pg.dv, kvl, 0, 2)
        wsg = torch.zeros(need + 256, dtype=torch.uint8, device=dev)

        def gstep():
            mx.mxfa_attn_decode_splitkv(dg["q"], dg["k"], dg["v"], dg["cu_q"], dg["cu_k"], 1, kvl,
                                        softmax_scale=pg.scale, out=og, lse=lg, ws=wsg, stream=stream)

        gtimes = time_steps(gstep, max(5, args.steps // 3), 3, lambda: None, stream, world)  # KV 1.07 GB >> L2
        gbytes = decode_bytes(pg)
        gms = max_over_ranks(statistics.mean(gtimes), world)
        ggbs = gbytes / (gms / 1e3) / 1e9
        decode_gqa = {"workload": pg.name, "value": ggbs * world, "unit": "GB/s", "ms_per_step": gms,
                      "algorithmic_bytes": gbytes, "l2": "inputs (1.07 GB K+V) larger than L2",
                      "roofline": {"bound": "hbm", "achieved": ggbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                   "frac": ggbs / pk["hbm_gbs"],
                                   "traffic": recorded_traffic("decode_gqa", pg.name),
                                   "peak_kind": f"{pk_kind} HBM copy"}}

    # ---------------- MLA decode over an E4M3 cache (next scope row; secondary measurement)
    decode_fp8 = None
    if not args.no_decode and args.only in (None, "fp8"):
        pf = workloads.cfg_mla_decode_fp8()
        df = to_dev(pf, dev)
        of = torch.empty((pf.total_q, pf.hq, pf.dv), dtype=torch.bfloat16, device=dev)
        lf = torch.empty((pf.total_q, pf.hq), dtype=torch.float32, device=dev)
        need = mx.load().mxfa_attn_decode_mla_fp8kv_workspace_size(pf.batch, 4, pf.hq, 8192, 0)
        wsf = torch.zeros(need + 256, dtype=torch.uint8, device=dev)

        def fstep():
            mx.mxfa_attn_decode_mla_fp8kv(df["q"], df["kv"], pf.kv_scale, df["cu_q"], df["cu_k"], 4, 8192,
                                          softmax_scale=pf.scale, out=of, lse=lf, ws=wsf, stream=stream)

        ftimes = time_steps(fstep, max(5, args.steps // 3), 3, lambda: None, stream, world)  # 604 MB codes >> L2
        fbytes = decode_bytes(pf)
        fms = max_over_ranks(statistics.mean(ftimes), world)
        fgbs = fbytes / (fms / 1e3) / 1e9
        fflops = 2.0 * pf.total_q * pf.hq * (pf.total_k // pf.batch) * (pf.dqk + pf.dv)
        decode_fp8 = {"workload": pf.name, "value": fgbs * world, "unit": "GB/s", "ms_per_step": fms,
                      "algorithmic_bytes": fbytes, "l2": "inputs (604 MB of codes) larger than L2",
                      "kv_rows_per_s": pf.total_k * world / (fms / 1e3),
                      "mma_tflops": fflops / (fms / 1e3) / 1e12,
                      "limit": "not HBM: the same M = 64 bf16 MMAs per KV row as the bf16 cache, plus the "
                               "shared-memory traffic of widening the codes; compare kv_rows_per_s with decode's",
                      "roofline": {"bound": "hbm", "achieved": fgbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                   "frac": fgbs / pk["hbm_gbs"],
                                   "traffic": recorded_traffic("decode", pf.name),
                                   "peak_kind": f"{pk_kind} HBM copy"}}
        if decode is not None:
            decode["kv_rows_per_s"] = pdc.total_k * world / (decode["ms_per_step"] / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only is None:
        cpu = cpu_baseline_prefill()

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": p.name, "B": B, "H": H, "seq_len": S, "head_dim": D, "causal": True,
                           "flops_per_step": flops, "l2": "flushed before every step (512 MiB write)",
                           "parallelism": f"replicas x{world}"},
                "roofline": roofline, "cpu_baseline": cpu,
                "e2e": None if args.only else {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                                               "d2h_bytes_per_step": d2h},
                "gpu_launches": args.steps, "clocks": clk.summary(), "decode": decode,
                "decode_gqa": decode_gqa, "decode_fp8": decode_fp8}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""The multi-GPU path of bench.py on the host: two gloo ranks.

`bench.py --gpus N` runs N independent replicas of the hot path (it has no
exchange step, so there is no collective on the data path); the process
group carries only the timing barrier and the max over ranks, and the
reported value is all ranks' units over the slowest rank's time.  These
tests run those pieces as two processes on CPU."""
import importlib.util
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    b = _bench()
    r, w, local = b.dist_setup(world)
    import torch.distributed as dist
    assert dist.get_backend() == "gloo"
    b.barrier(w)
    t_max = b.max_over_ranks(100.0 + 25.0 * r, w)     # rank 1 is the slower one
    rate = b.job_rate(1000.0, 4, w, t_max)
    b.barrier(w)
    dist.destroy_process_group()
    out.put((r, w, local, t_max, rate))


@pytest.mark.timeout(120)
def test_two_gloo_ranks_time_by_the_slowest_and_sum_the_work():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[:3] for r in res] == [(0, 2, 0), (1, 2, 1)]
    for _, _, _, t_max, rate in res:
        assert t_max == 125.0                          # every rank sees the slowest rank's time
        assert rate == pytest.approx(1000.0 * 4 * 2 / 0.125)  # both ranks' work over that time


def test_single_process_needs_no_process_group():
    b = _bench()
    assert b.dist_setup(1) == (0, 1, 0)
    assert b.max_over_ranks(3.5, 1) == 3.5
    assert b.job_rate(10.0, 2, 1, 1000.0) == 20.0


def test_reference_arm_runs_on_rank_zero_only(capsys):
    b = _bench()

    class Args:
        gpus, steps, warmup = 2, 1, 3

    b.run_reference(Args, 1, 2)                        # rank 1: no work, no output
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores, on
    sampled rows of the headline workload) prints one JSON line with the
    contract's keys and the headline's config."""
    import json
    import subprocess
    import sys as _sys
    out = subprocess.run([_sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--sample-seconds", "0.3"], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "dtype",
                "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    b = _bench()
    assert d["config"] == b.headline_config_of(d["config"]["workload"], d["config"]["flops_per_step"], 1)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1

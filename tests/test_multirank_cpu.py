"""Host logic of the multi-GPU (replica) benchmark path, on CPU with gloo.

With N GPUs every rank runs its own replica of the step; the job time is
the slowest rank's and the value counts every rank's bytes.  These tests run
two gloo ranks on CPU (no GPU, no data-path collective) and check that
reduction and aggregation, and that the CPU reference arm prints on rank 0
only."""

import datetime
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(100.0 + 7.0 * rank, world)
        q.put((rank, slowest, bench.job_gbs(10**9, 5, world, slowest)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_job_time_is_the_slowest_rank_and_value_counts_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [107.0, 107.0]
    expected = 2 * 10**9 * 5 / 0.107 / 1e9
    assert all(abs(r[2] - expected) < 1e-9 * expected for r in res)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert abs(bench.job_gbs(2 * 10**9, 4, 1, 8.0) - 1000.0) < 1e-9


def _run_reference(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "3", "--ref-tokens-per-rank", "2"], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_on_rank_zero_only():
    import bench
    r1 = _run_reference(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference(0)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["n_gpus"] == 2 and line["steps"] == 1 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["unit"] == line["e2e"]["unit"] == "GB/s"
    # the config is the sample this arm ran (2 tokens per rank of the prefill
    # shape), and names the GPU arm's workload it is cut from
    assert line["config"]["workload"].startswith("prefill: T=16 ") and line["config"]["T"] == 16
    assert line["config"]["H"] == 7168 and line["config"]["sample_of"].startswith("prefill: T=32768")
    sample = bench.workload(_default_args()).with_(T=16)
    nb = bench.call_bytes(sample)
    assert line["config"]["step_bytes"] == sum(nb[c] for c in bench.CALLS)
    assert "T=16 " in line["cpu_baseline"]["sample"]
    for key in ("value", "unit", "cores", "kind", "sample", "host_cores", "cpu_model"):
        assert key in line["cpu_baseline"], key
    assert line["cpu_baseline"]["host_cores"] >= 1 and line["cpu_baseline"]["cores"] == 1


def _default_args():
    import argparse
    return argparse.Namespace(workload="prefill", tokens_per_rank=0, dispatch_dtype="default", route=False,
                              max_tokens_per_rank=0)

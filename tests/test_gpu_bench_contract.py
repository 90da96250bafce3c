"""bench.py end to end on the tiny workload: one JSON line with every key the
benchmark contract names, the CUDA path's own kernels counted, the oracle
timed beside it."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_has_the_contract_keys(cuda_device):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny", "--steps", "4",
                        "--warmup", "3", "--cpu-tokens-per-rank", "64"],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "clocks",
                "gpu_launches", "per_call"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"].startswith("tiny: T=64")
    roof = d["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["achieved"] > 0 and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] > 0 and cpu["sample"]
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    # tiny: one-cluster layout + dispatch + combine + both backward passes, per timed step
    assert d["gpu_launches"] == 5 * 4
    for call in ("layout", "dispatch", "combine", "combine_backward", "dispatch_backward"):
        assert d["per_call"][call]["us"] > 0
        # tiny is timed cold per call, beside a same-size copy timed the same way
        copy = d["per_call"][call]["same_size_copy"]
        assert copy["us"] > 0 and copy["GB_s"] > 0
        assert abs(copy["frac_of_copy"] - copy["us"] / d["per_call"][call]["us"]) < 3e-3
    both = d["dispatch_incl_layout"]  # dispatch with its layout
    assert abs(both["us"] - d["per_call"]["layout"]["us"] - d["per_call"]["dispatch"]["us"]) < 0.02
    load = d["load"]  # load skew from the layout's counts: max over mean, at least 1
    for key in ("tokens_per_expert_max_over_mean", "rows_per_rank_max_over_mean", "tokens_per_rank_max_over_mean"):
        assert load[key] >= 1.0


def test_bench_line_for_the_emulated_ranks(cuda_device):
    """--peers: the R ranks' peer calls, every call timed cold (tiny moves far
    less than the L2), the peer kernels named, no traffic figure (the stored
    capture is of the single-GPU kernel)."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny", "--peers", "--steps", "4",
                        "--warmup", "3", "--no-e2e", "--no-cpu-baseline"],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["config"]["parallelism"].startswith("1 GPU, 4 ranks emulated")
    assert d["config"]["per_call_l2"].startswith("cold")
    if d["roofline"]["call"] != "layout":  # the layout has no peer form
        assert "peers_kernel" in d["roofline"]["kernel"]
    assert d["roofline"]["traffic"] is None
    # tiny: the one-cluster layout, then 4 calls x 4 ranks, per timed step
    assert d["gpu_launches"] == (1 + 4 * 4) * 4
    for call in ("layout", "dispatch", "combine", "combine_backward", "dispatch_backward"):
        assert d["per_call"][call]["us"] > 0


def test_bench_line_with_the_fused_dispatch(cuda_device):
    """--fused-dispatch: the layout and the dispatch as one call, same kernels."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny", "--fused-dispatch",
                        "--steps", "4", "--warmup", "3", "--no-e2e", "--no-cpu-baseline"],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["config"]["dispatch_call"].startswith("fused")
    assert set(d["per_call"]) == {"dispatch_with_layout", "combine", "combine_backward", "dispatch_backward"}
    assert d["gpu_launches"] == 5 * 4
    assert d["value"] > 0

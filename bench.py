#!/usr/bin/env python
"""Benchmark of the MoE expert-parallel dispatch / combine hot path on B200.

One step = the whole path over one batch of the workload: routing layout,
dispatch (FP8 with the prefill workload), combine, combine backward and
dispatch backward, all through the C ABI (libep_b200.so).  Inputs are
seeded synthetic draws (combine_ep_get_histogram_b200.workloads) resident in
HBM; every tensor of the prefill workload is larger than the 126 MB L2, so
no flush is needed between steps.

Prints one JSON line (rank 0).  value = effective GB/s of the step over all
ranks (algorithmic bytes read + written by the five calls / device time);
per-call microseconds and GB/s are in "per_call".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle on a bounded sample of the same
workload (rank 0 only).  With N > 1 (torchrun) every rank runs an
independent replica on its own GPU ("replicas only": the virtual-rank path
has no inter-GPU exchange); the step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch/combine µs/call & effective HBM GB/s vs B200 roofline, 1 GPU"
CALLS = ("layout", "dispatch", "combine", "combine_backward", "dispatch_backward")
ROUTE_CALLS = ("route",) + CALLS
# --fused-dispatch: the layout and the dispatch as one call (ep_dispatch_with_layout)
FUSED_CALLS = ("dispatch_with_layout", "combine", "combine_backward", "dispatch_backward")
FALLBACK_HBM_GBS = 6650.0


def call_bytes(w) -> dict:
    """Algorithmic bytes read + written per call."""
    T, H, k, R = w.T, w.H, w.k, w.R
    disp = T * H * 2 + (T * k * (H + 4 * (H // 128)) if w.use_fp8 else T * k * H * 2)
    return {
        "route": T * w.E * 4 + T * k * (8 + 4),
        "layout": T * k * 8 + T * R + 2 * T * k * 4,
        "dispatch": disp,
        "combine": T * k * H * 2 + T * k * 4 + T * H * 2,
        "combine_backward": T * H * 2 + 2 * T * k * H * 2 + 2 * T * k * 4,
        "dispatch_backward": T * k * H * 2 + T * H * 2,
        "dispatch_with_layout": T * k * 8 + T * R + 2 * T * k * 4 + disp,
    }


# DRAM bytes per launch of the dominant kernel (dram__bytes_read.sum +
# dram__bytes_write.sum), captured by ncu on the prefill shape cut to 512
# tokens per rank and scaled to the full launch by the tokens processed (x8;
# the counters grow with the tokens).  An entry only holds for the kernel
# sources and the launch configuration (the host file picks the grids) it was
# taken on: if their hash differs, the bench reports traffic as null.
MEASURED_TRAFFIC = {
    ("prefill", 32768, "combine_backward"): {
        "bytes": 8 * (528.777728e6 + 413.155840e6),
        "sources_sha1": "09e1eb104e5308f5a7f1b26a67b66d821b26af22",
    },
}
KERNEL_SOURCES = ("combine_ep_get_histogram_b200/csrc/common.cuh",
                  "combine_ep_get_histogram_b200/csrc/movement.cuh",
                  "combine_ep_get_histogram_b200/csrc/ep_api.cu")


def code_lines(text: str) -> str:
    """The source's tokens without // comments and without the layout between
    them: whitespace is kept only where it separates two identifier or number
    characters.  A comment edit or a rewrapped line leaves the hash of the
    code unchanged."""
    import re
    code = " ".join(line.split("//", 1)[0] for line in text.splitlines())
    code = re.sub(r"\s+", " ", code)
    return re.sub(r"(?<=\W) | (?=\W)", "", code).strip()


def kernel_sources_sha1(read=None) -> str:
    import hashlib
    h = hashlib.sha1()
    for f in KERNEL_SOURCES:
        if read is None:
            with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
                text = fh.read()
        else:
            text = read(f)
        h.update(code_lines(text).encode())
    return h.hexdigest()


def measured_traffic(w, call: str):
    e = MEASURED_TRAFFIC.get((w.name, w.T, call))
    if e is None or e["sources_sha1"] != kernel_sources_sha1():
        return None
    return e["bytes"]


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (one all-reduce; plumbing only)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(step_bytes: int, steps: int, world: int, total_ms: float) -> float:
    """Whole-job effective GB/s: every rank moves step_bytes per step; the job
    takes the slowest rank's time."""
    return world * step_bytes * steps / (total_ms * 1e-3) / 1e9


def peaks() -> tuple[float, str]:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, kept only inside
    the timed window."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.sel = []
        try:
            self.sel = ["-i", "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)]
        except Exception:
            pass
        self.proc = None
        self.path = None
        self.window = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "50"] + self.sel, stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.out.close()
        import datetime
        sm, smax, reasons, n = [], [], set(), 0
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    continue
                if self.window and not (self.window[0] - 0.05 <= ts <= self.window[1] + 0.05):
                    continue
                n += 1
                try:
                    sm.append(float(parts[1].split()[0]))
                    smax.append(float(parts[2].split()[0]))
                except ValueError:
                    pass
                for name, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": n}


# ------------------------------------------------------------- GPU arm

class CallMarks:
    """Events at the call boundaries of one step.  Warm (no flush): one event
    before the first call and one after each, the calls back to back.  Cold:
    L2 is flushed before each call, outside that call's own pair of events."""

    def __init__(self, marks, flush=None):
        self.marks, self.flush, self.n = marks, flush, 0
        if flush is None:
            self._rec()

    def _rec(self):
        if self.marks is not None:
            self.marks[self.n].record()
        self.n += 1

    def begin(self):
        if self.flush is not None:
            self.flush()
            self._rec()

    def end(self):
        self._rec()


def marks_per_step(ncalls: int, cold: bool) -> int:
    return 2 * ncalls if cold else ncalls + 1


def call_ms(marks, ci: int, cold: bool) -> float:
    """Duration of call ci from one step's marks (CallMarks layout)."""
    a, b = (marks[2 * ci], marks[2 * ci + 1]) if cold else (marks[ci], marks[ci + 1])
    return a.elapsed_time(b)


class Path:
    """Device buffers of one workload and one step through the C ABI."""

    def __init__(self, w, d, dev, max_tokens_per_rank=0, route=False, num_sms=0, fused=False):
        import numpy as np
        import torch
        import combine_ep_get_histogram_b200 as ep
        self.ep, self.w, self.dev = ep, w, dev
        self.shape = ep.make_shape(w.T, w.H, w.k, w.E, w.R, w.use_fp8, num_sms, max_tokens_per_rank)
        P = ep.ep.receive_rows(self.shape)

        def bf16(a):
            return torch.from_numpy(a.view(np.int16))

        self.host = {"topk_idx": torch.from_numpy(d["topk_idx"]), "topk_weights": torch.from_numpy(d["topk_weights"]),
                     "x": bf16(d["x"]), "y": bf16(d["y"]), "g": bf16(d["g"])}
        self.route = route
        self.fused = fused
        if route:
            self.host["scores"] = torch.from_numpy(d["scores"])
        self.inp = {n: t.to(dev) for n, t in self.host.items()}
        self.handle = ep.Handle(self.shape, dev)
        self.ws = ep.workspace(self.shape, dev)
        self.recv_x = torch.empty((P, w.H), dtype=torch.uint8 if w.use_fp8 else torch.int16, device=dev)
        self.recv_scale = torch.empty((P, w.G), dtype=torch.float32, device=dev) if w.use_fp8 else None
        self.recv_weight = torch.empty(P, dtype=torch.float32, device=dev)
        self.out = torch.empty((w.T, w.H), dtype=torch.int16, device=dev)
        self.grad_y = torch.empty((P, w.H), dtype=torch.int16, device=dev)
        self.grad_w = torch.empty((w.T, w.k), dtype=torch.float32, device=dev)
        self.grad_x = torch.empty((w.T, w.H), dtype=torch.int16, device=dev)

    def step(self, marks=None, before_back=None, after_combine=None, flush=None):
        """One pass of the path.  before_back runs (on the host, at enqueue
        time) between dispatch and combine, after_combine right after combine:
        hooks for the end-to-end pipeline's stream waits and events.  marks and
        flush: see CallMarks."""
        ep, i = self.ep, self.inp
        m = CallMarks(marks, flush)
        if self.route:
            m.begin()
            ep.ep_route_group_limited(self.shape, i["scores"], self.w.n_groups, self.w.topk_groups, i["topk_idx"],
                                      i["topk_weights"])
            m.end()
        if self.fused:
            m.begin()
            ep.ep_dispatch_with_layout(self.shape, i["topk_idx"], i["x"], i["topk_weights"], self.handle, self.ws,
                                       self.recv_x, self.recv_scale, self.recv_weight)
            m.end()
        else:
            m.begin()
            ep.ep_get_dispatch_layout(self.shape, i["topk_idx"], self.handle, self.ws)
            m.end()
            m.begin()
            ep.ep_dispatch(self.shape, i["x"], i["topk_weights"], self.handle, self.recv_x, self.recv_scale,
                           self.recv_weight)
            m.end()
        if before_back is not None:
            before_back()
        m.begin()
        ep.ep_combine(self.shape, i["y"], i["topk_weights"], self.handle, self.out)
        if after_combine is not None:
            after_combine()
        m.end()
        m.begin()
        ep.ep_combine_backward(self.shape, i["g"], i["y"], i["topk_weights"], self.handle, self.grad_y,
                               self.grad_w)
        m.end()
        m.begin()
        ep.ep_dispatch_backward(self.shape, self.grad_y, self.handle, self.grad_x)
        m.end()


def launches_per_step(w, peers: bool = False) -> int:
    """Kernels one step launches: layout (one kernel for small problems, else
    count + scan + assign), dispatch, combine and the two backward passes
    (once per rank with the peer calls)."""
    small = (w.T * w.k <= 16384 and w.E <= 256 and w.R <= 64 and w.R * w.E <= 2048
             and -(-w.T // 8) * w.R <= 8192)
    return (1 if small else 3) + 4 * (w.R if peers else 1)


class PeersPath(Path):
    """The step of multi-GPU expert parallelism with its R ranks emulated on
    one GPU: one global layout, then every rank's peer calls for its own
    tokens, each owner rank's receive buffers a separate allocation."""

    def __init__(self, w, d, dev):
        import torch
        super().__init__(w, d, dev)
        ep, multi = self.ep, __import__("combine_ep_get_histogram_b200.multi", fromlist=["multi"])
        ep.ep_get_dispatch_layout(self.shape, self.inp["topk_idx"], self.handle, self.ws)
        torch.cuda.synchronize()
        rows = multi.owner_rows(self.handle.tensors["expert_offset"].cpu().numpy(), w.E, w.R)
        pay = torch.uint8 if w.use_fp8 else torch.int16

        def bufs(cols, dtype):
            return [torch.empty((max(n, 1),) + cols, dtype=dtype, device=dev) for _, n in rows]

        self.rx, self.rw, self.gy = bufs((w.H,), pay), bufs((), torch.float32), bufs((w.H,), torch.int16)
        self.rs = bufs((w.G,), torch.float32) if w.use_fp8 else None
        self.ys = [self.inp["y"][r0:r0 + n] if n else torch.empty((1, w.H), dtype=torch.int16, device=dev)
                   for r0, n in rows]
        Tl = w.T // w.R
        self.ranks = [(r, slice(r * Tl, (r + 1) * Tl)) for r in range(w.R)]

    def step(self, marks=None, before_back=None, after_combine=None, flush=None):
        """One step; every call runs its R ranks on R streams forked from and
        joined back to the current stream, as the ranks of R GPUs would run
        them side by side."""
        import torch
        ep, i, sh, h = self.ep, self.inp, self.shape, self.handle
        cur = torch.cuda.current_stream()
        if not hasattr(self, "rank_streams"):
            self.rank_streams = [torch.cuda.Stream(self.dev) for _ in self.ranks]
        m = CallMarks(marks, flush)

        def fanout(call):
            fork = torch.cuda.Event()
            fork.record(cur)
            for (r, tok), st in zip(self.ranks, self.rank_streams):
                st.wait_event(fork)
                with torch.cuda.stream(st):
                    call(r, tok)
                done = torch.cuda.Event()
                done.record(st)
                cur.wait_event(done)

        m.begin()
        ep.ep_get_dispatch_layout(sh, i["topk_idx"], h, self.ws)
        m.end()
        m.begin()
        fanout(lambda r, tok: ep.ep_dispatch_peers(sh, r, i["topk_idx"], h, i["x"][tok], i["topk_weights"][tok],
                                                   self.rx, self.rs, self.rw))
        m.end()
        if before_back is not None:
            before_back()
        m.begin()
        fanout(lambda r, tok: ep.ep_combine_peers(sh, r, i["topk_idx"], h, self.ys, i["topk_weights"][tok],
                                                  self.out[tok]))
        if after_combine is not None:
            after_combine()
        m.end()
        m.begin()
        fanout(lambda r, tok: ep.ep_combine_backward_peers(sh, r, i["topk_idx"], h, i["g"][tok], self.ys,
                                                           i["topk_weights"][tok], self.gy, self.grad_w[tok]))
        m.end()
        m.begin()
        fanout(lambda r, tok: ep.ep_dispatch_backward_peers(sh, r, i["topk_idx"], h, self.gy, self.grad_x[tok]))
        m.end()


B200_L2_BYTES = 126 * 2**20


def l2_policy(step_bytes: int, l2_bytes: int) -> tuple:
    """(flush, description): no flush when a step moves at least 4x the L2
    size, so that no buffer is still in L2 when the next step reads it;
    otherwise L2 is flushed before every timed step."""
    if step_bytes >= 4 * l2_bytes:
        return False, (f"no flush: a step moves {step_bytes / 1e6:.0f} MB, {step_bytes / l2_bytes:.0f}x the "
                       f"{l2_bytes / 2**20:.0f} MiB L2, so no buffer is still in L2 when the next step reads it")
    return True, (f"L2 flushed before every step ({2 * l2_bytes / 2**20:.0f} MiB written, then "
                  f"{2 * l2_bytes / 2**20:.0f} MiB read, outside the timed region; each step timed on its own)")


MOVEMENT_CALLS = ("dispatch", "dispatch_with_layout", "combine", "combine_backward", "dispatch_backward")


def per_call_policy(nb: dict, l2_bytes: int) -> tuple:
    """(cold, description) for the per-call times: when some movement call
    moves less than 4x the L2 size, it could read what the call before it left
    in L2, so every call is timed on its own after an L2 flush; otherwise the
    calls are timed back to back inside the step."""
    small = min(nb[c] for c in MOVEMENT_CALLS if c in nb)
    if small < 4 * l2_bytes:
        return True, (f"cold: each call timed on its own after an L2 flush outside its events ({2 * l2_bytes / 2**20:.0f} "
                      f"MiB written, then {2 * l2_bytes / 2**20:.0f} MiB read so the flush's dirty lines are written "
                      f"back first; the smallest call moves {small / 1e6:.0f} MB, under 4x the L2)")
    return False, (f"warm: calls back to back in the step (the smallest call moves {small / 1e6:.0f} MB, "
                   f"{small / l2_bytes:.0f}x the L2)")


def bench_config(w, args, world: int, l2_bytes: int = B200_L2_BYTES) -> dict:
    """The JSON line's config: the workload by name and sizes (both arms)."""
    nb = {c: v for c, v in call_bytes(w).items() if c in step_calls(args)}
    step_bytes = sum(nb.values())
    return {"workload": f"{w.name}: T={w.T} ({w.R} virtual ranks x {w.T // w.R} tokens), H={w.H}, "
                        f"E={w.E}, k={w.k}, top-{w.topk_groups} of {w.n_groups} groups, "
                        f"{'FP8' if w.use_fp8 else 'BF16'} dispatch + BF16 combine + both backward passes",
            "T": w.T, "H": w.H, "k": w.k, "E": w.E, "R": w.R, "use_fp8": w.use_fp8,
            "storage": ("e4m3 codes + f32 scales dispatched, bf16 expert rows, outputs and gradients"
                        if w.use_fp8 else "bf16 rows, outputs and gradients"),
            "step_bytes": step_bytes, "l2": l2_policy(step_bytes, l2_bytes)[1],
            "per_call_l2": per_call_policy(nb, l2_bytes)[1],
            "receive_layout": (f"padded [E][R][{args.max_tokens_per_rank}]" if args.max_tokens_per_rank
                               else "dense [T*k]"),
            "parallelism": (f"replicas x{world}" if world > 1 else
                            f"1 GPU, {w.R} ranks emulated through the peer-table calls"
                            if getattr(args, "peers", False) else "1 GPU, virtual ranks"),
            "router_in_step": bool(args.route),
            "dispatch_call": ("fused: ep_dispatch_with_layout" if getattr(args, "fused_dispatch", False)
                              else "separate: ep_get_dispatch_layout, then ep_dispatch")}


def run_ours(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist
    from combine_ep_get_histogram_b200 import workloads as wl

    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    w = workload(args)
    M = args.max_tokens_per_rank
    calls = step_calls(args)
    d = wl.make_inputs(w, parts=("routing", "x", "g") + (() if M else ("y",)) + (("scores",) if args.route else ()))
    if M:  # expert outputs fill the padded receive rows
        d["y"] = wl.normal_bf16(w.E * w.R * M, w.H, w.seed, 2)
    if args.peers and (M or args.route or args.fused_dispatch):
        raise SystemExit("--peers runs the dense layout and separate calls, without routing")
    path = PeersPath(w, d, dev) if args.peers else Path(w, d, dev, M, route=args.route, fused=args.fused_dispatch)
    nb = {c: v for c, v in call_bytes(w).items() if c in calls}
    step_bytes = sum(nb.values())
    nmarks = len(calls) + 1
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size or B200_L2_BYTES
    flush, _ = l2_policy(step_bytes, l2_bytes)
    cold, _ = per_call_policy(nb, l2_bytes)
    # L2 flush: 2x the L2 size written, then another 2x read, so that the
    # flush's own dirty lines reach HBM before the timed work starts (with the
    # write alone, each decode call paid 2-8 us for writing back the flush)
    flush_buf = torch.empty(2 * l2_bytes // 4, dtype=torch.int32, device=dev) if (flush or cold) else None
    flush_rd = torch.ones(2 * l2_bytes // 4, dtype=torch.float32, device=dev) if (flush or cold) else None
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(i: int):
        if flush_buf is not None:
            flush_buf.fill_(i)
            torch.sum(flush_rd, 0, out=flush_sum)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):  # also makes the library's one-time per-device set-up happen here
        path.step()
    barrier()

    # One step is captured as a CUDA graph (the C ABI never allocates or
    # synchronises), so small workloads are not timed against Python's call
    # overhead.  The timed graph holds the step's kernels alone; a second
    # graph of the same step, with events recorded between the calls, gives
    # the per-call breakdown (event nodes between two kernels add their own
    # latency and keep a kernel from starting while the previous one drains).
    per_call_ms = {c: [] for c in calls}
    same_size_copy_us = None
    if args.no_graph:
        run_step = path.step
    else:
        gmarks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nmarks)]
        graph, mark_graph = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            path.step()
        with torch.cuda.graph(mark_graph):
            path.step(gmarks)
        run_step = graph.replay
        for _ in range(args.warmup):
            run_step()
            mark_graph.replay()
        # per-call breakdown: one replay at a time, events read after each
        for i in range(0 if cold else min(args.steps, 20)):
            flush_l2(i)
            mark_graph.replay()
            torch.cuda.synchronize()
            for ci, c in enumerate(calls):
                per_call_ms[c].append(call_ms(gmarks, ci, False))
        barrier()
    if cold:
        # per-call breakdown with L2 flushed before every call (its own step
        # graph, or eager launches); the timed steps below stay as they are
        cmarks = [torch.cuda.Event(enable_timing=True, external=not args.no_graph)
                  for _ in range(marks_per_step(len(calls), True))]

        def cold_flush():
            flush_buf.add_(1)
            torch.sum(flush_rd, 0, out=flush_sum)

        if args.no_graph:
            def run_cold():
                path.step(cmarks, flush=cold_flush)
        else:
            cold_graph = torch.cuda.CUDAGraph()
            torch.cuda.synchronize()
            with torch.cuda.graph(cold_graph):
                path.step(cmarks, flush=cold_flush)
            run_cold = cold_graph.replay
        for _ in range(2):
            run_cold()
        for i in range(min(args.steps, 20)):
            run_cold()
            torch.cuda.synchronize()
            for ci, c in enumerate(calls):
                per_call_ms[c].append(call_ms(cmarks, ci, True))
        # the same method around a device-to-device copy (cudaMemcpyAsync)
        # that moves each call's bytes (half read, half written): what a
        # plain copy of that size reaches when it is timed this way
        half = {c: max(16, nb[c] // 2 // 16 * 16) for c in calls}
        csrc = torch.ones(max(half.values()), dtype=torch.uint8, device=dev)
        cdst = torch.empty_like(csrc)
        kmarks = [torch.cuda.Event(enable_timing=True, external=not args.no_graph) for _ in range(2 * len(calls))]

        def copies_once():
            for ci, c in enumerate(calls):
                cold_flush()
                kmarks[2 * ci].record()
                cdst[:half[c]].copy_(csrc[:half[c]])
                kmarks[2 * ci + 1].record()

        if args.no_graph:
            run_copies = copies_once
        else:
            copy_graph = torch.cuda.CUDAGraph()
            torch.cuda.synchronize()
            with torch.cuda.graph(copy_graph):
                copies_once()
            run_copies = copy_graph.replay
        copy_ms = {c: [] for c in calls}
        for i in range(2 + min(args.steps, 20)):
            run_copies()
            torch.cuda.synchronize()
            if i >= 2:
                for ci, c in enumerate(calls):
                    copy_ms[c].append(kmarks[2 * ci].elapsed_time(kmarks[2 * ci + 1]))
        same_size_copy_us = {c: 1e3 * statistics.median(v) for c, v in copy_ms.items()}
        del csrc, cdst
        barrier()

    # device-timed region: K steps back to back on the launching stream
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(nmarks)] for _ in range(args.steps)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    step_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)] if flush else []
    t0 = time.time()
    e_start.record()
    for s in range(args.steps):
        if flush:  # the flush stays outside the per-step events
            flush_l2(s)
            step_events[s][0].record()
        if args.no_graph:
            path.step(marks[s])
        else:
            run_step()
        if flush:
            step_events[s][1].record()
    e_end.record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    sampler.mark(t0, t1)
    clocks = sampler.stop()
    if args.no_graph and not cold:
        for m in marks:
            for ci, c in enumerate(calls):
                per_call_ms[c].append(call_ms(m, ci, False))
    local_ms = (sum(a.elapsed_time(b) for a, b in step_events) if flush else e_start.elapsed_time(e_end))
    total_ms = max_over_ranks(local_ms, world, dev)
    ms_per_step = total_ms / args.steps

    # End to end through the same C ABI: every step copies its inputs from
    # pinned host memory and reads its results back.  Two device buffer sets
    # alternate, so step i+1's host-to-device copies (one stream) overlap step
    # i's kernels (a second stream) and step i's device-to-host copies (a
    # third stream; PCIe is full duplex).
    e2e = None
    if not args.no_e2e:
        paths = [path, PeersPath(w, d, dev) if args.peers else Path(w, d, dev, M, route=args.route,
                                                                    fused=args.fused_dispatch)]
        pin = {n: t.pin_memory() for n, t in path.host.items()}
        outs = {"out": torch.empty_like(path.out, device="cpu").pin_memory(),
                "grad_x": torch.empty_like(path.grad_x, device="cpu").pin_memory(),
                "grad_w": torch.empty_like(path.grad_w, device="cpu").pin_memory()}
        h2d = sum(t.numel() * t.element_size() for t in pin.values())
        d2h = sum(t.numel() * t.element_size() for t in outs.values())
        back_names = ("g", "y")  # needed from combine on
        front_names = tuple(n for n in pin if n not in back_names)
        s_h2d, s_comp, s_d2h = (torch.cuda.Stream(dev) for _ in range(3))
        comp_done, d2h_done = [None, None], [None, None]

        def e2e_step(i):
            b = i % 2
            p = paths[b]
            ev_front, ev_back, ev_out = (torch.cuda.Event() for _ in range(3))
            with torch.cuda.stream(s_h2d):
                if comp_done[b] is not None:  # step i-2 has finished reading these inputs
                    s_h2d.wait_event(comp_done[b])
                for n in front_names:
                    p.inp[n].copy_(pin[n], non_blocking=True)
                ev_front.record(s_h2d)
                for n in back_names:
                    p.inp[n].copy_(pin[n], non_blocking=True)
                ev_back.record(s_h2d)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_front)
                if d2h_done[b] is not None:  # step i-2's results have left these outputs
                    s_comp.wait_event(d2h_done[b])
                p.step(before_back=lambda: s_comp.wait_event(ev_back), after_combine=lambda: ev_out.record(s_comp))
                comp_done[b] = torch.cuda.Event()
                comp_done[b].record(s_comp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_out)
                outs["out"].copy_(p.out, non_blocking=True)
                s_d2h.wait_event(comp_done[b])
                outs["grad_x"].copy_(p.grad_x, non_blocking=True)
                outs["grad_w"].copy_(p.grad_w, non_blocking=True)
                d2h_done[b] = torch.cuda.Event()
                d2h_done[b].record(s_d2h)

        def join(cur):
            for st in (s_h2d, s_comp, s_d2h):
                ev = torch.cuda.Event()
                ev.record(st)
                cur.wait_event(ev)

        cur = torch.cuda.current_stream()
        for i in range(max(2, min(args.warmup, 4))):
            e2e_step(i)
        join(cur)
        barrier()
        n_e2e = max(2, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for st in (s_h2d, s_comp, s_d2h):
            st.wait_event(e0)
        for i in range(n_e2e):
            e2e_step(i)
        join(cur)
        e1.record(cur)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": round(job_gbs(step_bytes, n_e2e, world, e_ms), 2), "unit": "GB/s",
               "ms_per_step": round(e_ms / n_e2e, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": n_e2e,
               "pipelining": "two device buffer sets; step i+1's host-to-device copies overlap step i's "
                             "kernels and its device-to-host copies (three streams)"}
        del paths[1]

    overlap = measure_overlap(args, w, d, dev, M, ms_per_step) if args.overlap_sms else None
    load = load_skew(path.handle, w)

    if rank != 0:
        return None

    peak, peak_kind = peaks()
    per_call = {}
    for c in calls:
        us = 1e3 * statistics.mean(per_call_ms[c])
        per_call[c] = {"us": round(us, 2), "us_median": round(1e3 * statistics.median(per_call_ms[c]), 2),
                       "bytes": nb[c], "GB_s": round(nb[c] / (us * 1e-6) / 1e9, 1),
                       "frac_of_peak": round(nb[c] / (us * 1e-6) / 1e9 / peak, 3)}
        if same_size_copy_us is not None:
            cu = same_size_copy_us[c]
            per_call[c]["same_size_copy"] = {"us": round(cu, 2), "GB_s": round(nb[c] / (cu * 1e-6) / 1e9, 1),
                                             "frac_of_copy": round(cu / us, 3)}
    dominant = max((c for c in calls), key=lambda c: per_call[c]["us"])
    kernel_of = {"dispatch": "dispatch_tma_kernel<FP8>" if w.use_fp8 else "dispatch_tma_kernel<BF16>",
                 "combine": "gather_reduce_kernel<weighted>", "combine_backward": "combine_backward_kernel",
                 "dispatch_backward": "gather_reduce_kernel<unweighted>", "layout": "layout_*_kernel",
                 "dispatch_with_layout": "layout_*_kernel + dispatch_tma_kernel (early form below 16 tokens per SM)",
                 "route": "route_compact_kernel|route_aligned_kernel|route_group_limited_kernel"}
    if args.peers:
        kernel_of.update({"dispatch": "dispatch_tma_peers_kernel" if 4 <= -(-w.H // 512) <= 16
                          else "dispatch_peers_kernel", "combine": "gather_reduce_peers_kernel<weighted>",
                          "combine_backward": "combine_backward_peers_kernel",
                          "dispatch_backward": "gather_reduce_peers_kernel<unweighted>"})
    ach = per_call[dominant]["GB_s"]
    # the stored capture is of the single-GPU kernel; the peer kernels have none
    traffic = None if args.peers else measured_traffic(w, dominant)
    line = {
        "metric": METRIC,
        "value": round(job_gbs(step_bytes, args.steps, world, total_ms), 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded group-limited routing, N(0,1) activations)",
        "config": bench_config(w, args, world, l2_bytes),
        "per_call": per_call,
        "roofline": {"kernel": kernel_of[dominant], "call": dominant, "bound": "hbm", "achieved": ach,
                     "peak": peak, "unit": "GB/s", "frac": round(ach / peak, 3),
                     "peak_source": f"{peak_kind} hbm_gbs",
                     "bytes_per_launch": nb[dominant], "traffic": traffic,
                     "traffic_source": ("ncu dram__bytes_read.sum + dram__bytes_write.sum at 512 tokens per rank, "
                                        "scaled to the full launch by the tokens processed")},
        "clocks": clocks,
        "gpu_launches": (launches_per_step(w, args.peers) + (1 if args.route else 0)) * args.steps,
        "timing": ("CUDA graph replay of the step (the kernels alone; the per-call times come from a second graph "
                   "with events between the calls)" if not args.no_graph else "eager launches"),
        "e2e": e2e,
    }
    line["load"] = load
    if "layout" in per_call and "dispatch" in per_call:
        # dispatch with and without its layout (the layout is latency-bound and
        # reported on its own above)
        us = per_call["layout"]["us"] + per_call["dispatch"]["us"]
        b = nb["layout"] + nb["dispatch"]
        line["dispatch_incl_layout"] = {"us": round(us, 2), "bytes": b, "GB_s": round(b / (us * 1e-6) / 1e9, 1),
                                        "frac_of_peak": round(b / (us * 1e-6) / 1e9 / peak, 3)}
    if overlap is not None:
        line["overlap"] = overlap
    return line


def load_skew(handle, w) -> dict:
    """Load balance of the step's routing from the layout's counts (read
    after the timed region): the busiest expert's and the busiest rank's
    receive counts over their means.  The pages use max > 2x mean as the sign
    of skew."""
    per_expert = handle.tensors["num_tokens_per_expert"].cpu().numpy().astype(float)
    per_rank = handle.tensors["num_tokens_per_rank"].cpu().numpy().astype(float)
    er = w.E // w.R
    rows_per_rank = per_expert.reshape(w.R, er).sum(axis=1)

    def ratio(v):
        return round(float(v.max() / v.mean()), 3) if v.size and v.mean() > 0 else None

    return {"tokens_per_expert_max_over_mean": ratio(per_expert),
            "rows_per_rank_max_over_mean": ratio(rows_per_rank),
            "tokens_per_rank_max_over_mean": ratio(per_rank)}


def measure_overlap(args, w, d, dev, M, step_ms):
    """The path on a side stream with an SM budget of N beside a
    compute-bound cuBLAS GEMM on the launching stream that leaves N SMs free
    (torch's matmul SM carve-out), against the best serial schedule: the GEMM
    on all SMs, then the path on all SMs.  The GEMM repeats are sized to
    about one full-GPU step of the path."""
    import torch
    budget = Path(w, d, dev, M, route=args.route, num_sms=args.overlap_sms, fused=args.fused_dispatch)
    full = Path(w, d, dev, M, route=args.route, fused=args.fused_dispatch)
    n = 8192
    gen = torch.Generator(device=dev).manual_seed(0)
    a = torch.randn((n, n), device=dev, dtype=torch.bfloat16, generator=gen)
    b = torch.randn((n, n), device=dev, dtype=torch.bfloat16, generator=gen)
    c = torch.empty((n, n), device=dev, dtype=torch.bfloat16)
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream(dev)

    def timed(fn, iters=5):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for _ in range(iters):
            fn()
        e1.record(cur)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters

    one = timed(lambda: torch.matmul(a, b, out=c))
    reps = max(1, round(step_ms / one))

    def gemms(carveout=None):
        torch._C._set_sm_carveout_experimental(carveout)
        try:
            for _ in range(reps):
                torch.matmul(a, b, out=c)
        finally:
            torch._C._set_sm_carveout_experimental(None)

    def serial():
        gemms()
        full.step()

    def overlapped():
        ev = torch.cuda.Event()
        ev.record(cur)
        side.wait_event(ev)
        with torch.cuda.stream(side):
            budget.step()
        gemms(args.overlap_sms)
        done = torch.cuda.Event()
        done.record(side)
        cur.wait_event(done)

    t_gemm, t_gemm_carved = timed(gemms), timed(lambda: gemms(args.overlap_sms))
    t_path, t_path_budget = timed(full.step), timed(budget.step)
    t_serial, t_over = timed(serial), timed(overlapped)
    return {"num_sms": args.overlap_sms, "gemm": f"torch.matmul bf16 {n}x{n}x{n} x {reps}",
            "gemm_ms_all_sms": round(t_gemm, 3), "gemm_ms_carved": round(t_gemm_carved, 3),
            "path_ms_all_sms": round(t_path, 3), "path_ms_at_budget": round(t_path_budget, 3),
            "serial_ms": round(t_serial, 3), "overlapped_ms": round(t_over, 3),
            "saved_frac": round(1.0 - t_over / t_serial, 3),
            "timing": "CUDA events on the launching stream, eager launches, mean of 5"}


def workload(args):
    from combine_ep_get_histogram_b200 import workloads as wl
    w = wl.CONFIGS[args.workload]
    # reshaped workloads (profiling captures of the other kernel variants)
    if getattr(args, "ranks", 0):
        w = w.with_(T=w.T // w.R * args.ranks, R=args.ranks)
    if getattr(args, "hidden", 0):
        w = w.with_(H=args.hidden)
    if getattr(args, "experts", 0):
        w = w.with_(E=args.experts)
    if getattr(args, "groups", 0):
        w = w.with_(routing="group", n_groups=args.groups,
                    topk_groups=getattr(args, "topk_groups", 0) or min(w.topk_groups, args.groups))
    if args.tokens_per_rank:
        w = w.with_(T=w.R * args.tokens_per_rank)
    if args.dispatch_dtype != "default":
        w = w.with_(use_fp8=args.dispatch_dtype == "fp8")
    return w


# -------------------------------------------------------- CPU oracle arm

def step_calls(args) -> tuple:
    calls = FUSED_CALLS if getattr(args, "fused_dispatch", False) else CALLS
    return (("route",) + calls) if args.route else calls


def oracle_pass(w, d, route: bool, M: int):
    """One step of the path on the oracle: routing (if timed), the dense or
    padded layout, dispatch, combine and both backward passes."""
    import oracle
    idx, wts = d["topk_idx"], d["topk_weights"]
    if route:
        idx, wts = oracle.route_group_limited(d["scores"], w.k, w.n_groups, w.topk_groups)
    if M:
        lay, rows = oracle.layout_padded(idx, w.E, w.R, M), w.E * w.R * M
    else:
        lay, rows = oracle.layout(idx, w.E, w.R), w.T * w.k
    slots = lay["slot_of_pair"]
    oracle.dispatch(d["x"], wts, slots, w.use_fp8, P=rows)
    oracle.combine(d["y"], wts, slots)
    gy, _ = oracle.combine_backward(d["g"], d["y"], wts, slots, P=rows)
    oracle.dispatch_backward(gy, slots, w.T, w.k)


def cpu_sample(args, tokens_per_rank: int):
    """The bench's workload (dispatch dtype override, routing and receive
    layout included) cut to tokens_per_rank tokens per virtual rank.  A
    padded layout gets tokens_per_rank rows per (expert, source rank) block."""
    from combine_ep_get_histogram_b200 import workloads as wl
    w = workload(args)
    ws = w.with_(T=w.R * tokens_per_rank)
    M = tokens_per_rank if args.max_tokens_per_rank else 0
    d = wl.make_inputs(ws, parts=("routing", "x", "g") + (() if M else ("y",)) +
                       (("scores",) if args.route else ()))
    if M:
        d["y"] = wl.normal_bf16(ws.E * ws.R * M, ws.H, ws.seed, 2)
    desc = (f"{w.name} shape (H={w.H}, E={w.E}, k={w.k}, R={w.R}) with T={ws.T} "
            f"({tokens_per_rank} tokens per rank) instead of {w.T}"
            + (f", padded blocks of {M} rows" if M else "")
            + f"; one full pass of the step ({', '.join(step_calls(args))})")
    return ws, d, desc, M


def host_cpu() -> dict:
    """The host the CPU legs run on: the cores this process may use and the
    CPU model (the oracle itself is single-threaded)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 0
    model = "unknown"
    try:
        with open("/proc/cpuinfo", encoding="utf-8", errors="replace") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": cores, "cpu_model": model}


def run_cpu_baseline(args) -> dict:
    ws, d, desc, M = cpu_sample(args, args.cpu_tokens_per_rank)
    t = time.perf_counter()
    oracle_pass(ws, d, args.route, M)
    dt = time.perf_counter() - t
    gbs = sum(call_bytes(ws)[c] for c in step_calls(args)) / dt / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": desc,
            "seconds": round(dt, 2), **host_cpu()}


def run_reference(args) -> dict:
    ws, d, desc, M = cpu_sample(args, args.ref_tokens_per_rank)
    for _ in range(args.warmup):
        oracle_pass(ws, d, args.route, M)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(ws, d, args.route, M)
    dt = (time.perf_counter() - t) / args.steps
    gbs = sum(call_bytes(ws)[c] for c in step_calls(args)) / dt / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "device": "host cores (rank 0 only)",
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded)",
        # the configuration this arm actually runs: the sample, and what it is cut from
        "config": {**bench_config(ws, args, 1), "sample_of": bench_config(workload(args), args, 1)["workload"]},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": desc,
                         **host_cpu()},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="prefill")
    ap.add_argument("--route", action="store_true",
                    help="start each step with group-limited routing of [T,E] scores (the step before the path)")
    ap.add_argument("--max-tokens-per-rank", type=int, default=0,
                    help="padded low-latency receive layout with this many rows per (expert, source rank)")
    ap.add_argument("--dispatch-dtype", choices=("default", "bf16", "fp8"), default="default",
                    help="override the workload's dispatch payload (the skewed workload is timed with both)")
    ap.add_argument("--tokens-per-rank", type=int, default=0,
                    help="resize the workload to R x this many tokens (profiling captures)")
    ap.add_argument("--hidden", type=int, default=0, help="reshape: hidden size H (profiling captures)")
    ap.add_argument("--experts", type=int, default=0, help="reshape: number of experts E")
    ap.add_argument("--groups", type=int, default=0, help="reshape: expert groups of the group-limited routing")
    ap.add_argument("--topk-groups", type=int, default=0, help="reshape: groups each token picks")
    ap.add_argument("--ranks", type=int, default=0, help="reshape: virtual ranks R (same tokens per rank)")
    ap.add_argument("--fused-dispatch", action="store_true",
                    help="the layout and the dispatch as one call (ep_dispatch_with_layout)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch each call eagerly instead of replaying a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--peers", action="store_true",
                    help="the step as R ranks emulated on one GPU through the multi-GPU (peer-table) calls")
    ap.add_argument("--overlap-sms", type=int, default=0,
                    help="also time the path with this SM budget on a side stream beside a bf16 GEMM")
    ap.add_argument("--cpu-tokens-per-rank", type=int, default=1536)
    ap.add_argument("--ref-tokens-per-rank", type=int, default=64)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device(f"cuda:{local}"))
    try:
        line = run_ours(args, rank, world, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = run_cpu_baseline(args)
            else:
                line["cpu_baseline"] = None
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

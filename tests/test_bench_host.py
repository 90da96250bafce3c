"""Host-side helpers of bench.py that need no GPU: the code hash that keeps a
measured DRAM-traffic figure tied to the kernel it was taken on (comments
and layout whitespace aside), and the L2
statement made from a step's bytes."""

import os

import bench


def _reader(edit=None):
    def read(f):
        with open(os.path.join(bench.ROOT, f), encoding="utf-8") as fh:
            text = fh.read()
        return edit(f, text) if edit else text
    return read


def test_comment_edits_keep_the_code_hash():
    base = bench.kernel_sources_sha1(_reader())
    assert base == bench.kernel_sources_sha1()
    commented = bench.kernel_sources_sha1(_reader(lambda f, t: t.replace("\n", "  // note\n\n", 3) + "// end\n"))
    assert commented == base


def test_rewrapped_lines_keep_the_code_hash():
    base = bench.kernel_sources_sha1()

    def rewrap(f, t):
        out = []
        for line in t.splitlines():
            code, sep, comment = line.partition("//")
            out.append(code.replace(", ", ",\n      ").replace("    ", "\t") + sep + comment)
        return "\n".join(out)

    assert bench.kernel_sources_sha1(_reader(rewrap)) == base


def test_code_edits_change_the_code_hash():
    base = bench.kernel_sources_sha1()
    edited = bench.kernel_sources_sha1(_reader(lambda f, t: t + "\nconstexpr int kUnused = 1;\n"
                                               if f.endswith("movement.cuh") else t))
    assert edited != base


def test_traffic_is_reported_only_for_the_captured_code():
    from combine_ep_get_histogram_b200 import workloads as wl
    w = wl.CONFIGS["prefill"]
    entry = bench.MEASURED_TRAFFIC[(w.name, w.T, "combine_backward")]
    expect = entry["bytes"] if entry["sources_sha1"] == bench.kernel_sources_sha1() else None
    assert bench.measured_traffic(w, "combine_backward") == expect
    assert bench.measured_traffic(w, "dispatch") is None


def test_l2_statement_follows_the_step_bytes():
    l2 = 126 * 2**20
    flush, text = bench.l2_policy(4 * l2, l2)
    assert not flush and "no flush" in text
    flush, text = bench.l2_policy(4 * l2 - 1, l2)
    assert flush and "flushed" in text


def test_per_call_times_are_cold_when_a_call_fits_a_few_l2s():
    from combine_ep_get_histogram_b200 import workloads as wl
    l2 = 126 * 2**20
    decode = {c: v for c, v in bench.call_bytes(wl.CONFIGS["decode"]).items() if c in bench.MOVEMENT_CALLS}
    prefill = bench.call_bytes(wl.CONFIGS["prefill"])
    cold, text = bench.per_call_policy(decode, l2)
    assert cold and "cold" in text          # decode calls move 75-250 MB
    cold, text = bench.per_call_policy(prefill, l2)
    assert not cold and "warm" in text      # the layout's few MB do not count
    assert bench.marks_per_step(5, True) == 10 and bench.marks_per_step(5, False) == 6


def test_call_marks_bracket_each_call():
    class Ev:
        def __init__(self, log, i):
            self.log, self.i = log, i

        def record(self):
            self.log.append(("mark", self.i))

    for cold in (False, True):
        log = []
        marks = [Ev(log, i) for i in range(bench.marks_per_step(2, cold))]
        m = bench.CallMarks(marks, (lambda: log.append(("flush",))) if cold else None)
        for c in range(2):
            m.begin()
            log.append(("call", c))
            m.end()
        if cold:
            assert log == [("flush",), ("mark", 0), ("call", 0), ("mark", 1),
                           ("flush",), ("mark", 2), ("call", 1), ("mark", 3)]
        else:
            assert log == [("mark", 0), ("call", 0), ("mark", 1), ("call", 1), ("mark", 2)]


def test_load_skew_is_max_over_mean_of_the_layout_counts():
    import torch
    from combine_ep_get_histogram_b200 import workloads as wl

    class FakeHandle:
        tensors = {"num_tokens_per_expert": torch.tensor([6, 2, 2, 2, 1, 1, 1, 1], dtype=torch.int32),
                   "num_tokens_per_rank": torch.tensor([5, 3], dtype=torch.int32)}

    w = wl.Workload("t", T=8, H=128, k=2, E=8, R=2, use_fp8=False, routing="group")
    load = bench.load_skew(FakeHandle(), w)
    assert load["tokens_per_expert_max_over_mean"] == 6 / 2
    assert load["rows_per_rank_max_over_mean"] == round(12 / 8, 3)  # rank rows 12 and 4
    assert load["tokens_per_rank_max_over_mean"] == round(5 / 4, 3)


def test_reshape_options():
    """The profiling reshapes keep every other field of the workload."""
    import argparse
    base = dict(workload="decode", tokens_per_rank=0, dispatch_dtype="default", route=False, max_tokens_per_rank=0,
                hidden=0, experts=0, groups=0, topk_groups=0, ranks=0)
    w0 = bench.workload(argparse.Namespace(**base))
    w = bench.workload(argparse.Namespace(**dict(base, ranks=16)))
    assert (w.R, w.T, w.T // w.R) == (16, 2048, w0.T // w0.R) and w.E == w0.E and w.H == w0.H
    w = bench.workload(argparse.Namespace(**dict(base, hidden=1024, tokens_per_rank=4096)))
    assert (w.H, w.T, w.R) == (1024, 8 * 4096, 8) and w.use_fp8
    w = bench.workload(argparse.Namespace(**dict(base, experts=160, groups=4, topk_groups=2)))
    assert (w.E, w.n_groups, w.topk_groups, w.routing, w.k) == (160, 4, 2, "group", 8)
    w = bench.workload(argparse.Namespace(**dict(base, groups=8, topk_groups=8)))
    assert (w.E, w.n_groups, w.topk_groups) == (256, 8, 8)


def test_fused_dispatch_step_calls_and_bytes():
    import argparse
    from combine_ep_get_histogram_b200 import workloads as wl
    a = argparse.Namespace(route=False, fused_dispatch=True)
    assert bench.step_calls(a) == bench.FUSED_CALLS
    assert bench.step_calls(argparse.Namespace(route=True, fused_dispatch=True))[0] == "route"
    assert bench.step_calls(argparse.Namespace(route=False)) == bench.CALLS
    b = bench.call_bytes(wl.CONFIGS["decode"])
    assert b["dispatch_with_layout"] == b["layout"] + b["dispatch"]

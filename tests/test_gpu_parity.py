"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Bar: layout, slot maps, BF16 payloads, E4M3 payload bytes, fp32 scales and
gate weights bit-exact; combine and dispatch_backward bit-exact (the stated
tolerance is 1 bf16 ulp; both sides run the same fixed-order chain);
grad_y bit-exact; grad_w within 1e-2 relative (or 1e-2 of the rms where the
dot product is near 0).

Every workload is compared element by element, in full: the small ones in
one oracle call, the three large ones (the launch configuration the
benchmark times) token chunk by token chunk, the oracle running the chunks
on a thread pool, so that every receive row, every combined token, every
grad_y row, every grad_w entry and every grad_x token is checked."""

import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import (GpuPath, assert_bits_equal, assert_layout_equal, bf16_host, compare_in_chunks, grad_w_close,
                      to_dev)

pytestmark = pytest.mark.gpu

CHUNK = 1024  # tokens per oracle call in the full-size comparisons


def compact_slots(slots_tk: np.ndarray) -> np.ndarray:
    """Slots of a token subset renumbered 0..n*k-1 (masked pairs stay -1)."""
    n, k = slots_tk.shape
    c = np.arange(n * k, dtype=np.int32).reshape(n, k)
    return np.where(slots_tk >= 0, c, -1).reshape(-1)


def _rows_of(slots_tk: np.ndarray, device):
    valid = slots_tk.reshape(-1) >= 0
    rows = torch.from_numpy(slots_tk.reshape(-1)[valid].astype(np.int64)).to(device)
    return valid, rows


def check_dispatch_all(ref_layout, d, gpu_recv, use_fp8, w):
    """Every receive row (payload, scales, gate weight) against the oracle's
    dispatch of its token chunk."""
    slots_all = ref_layout["slot_of_pair"].reshape(w.T, w.k)
    g_rx, g_rs, g_rw = gpu_recv

    def fetch(t0, t1):
        _, rows = _rows_of(slots_all[t0:t1], g_rx.device)
        return (g_rx.index_select(0, rows).cpu().numpy(),
                g_rs.index_select(0, rows).cpu().numpy() if use_fp8 else None,
                g_rw.index_select(0, rows).cpu().numpy())

    def check(t0, t1, got):
        slots = slots_all[t0:t1]
        valid = slots.reshape(-1) >= 0
        rx, rs, rw = oracle.dispatch(d["x"][t0:t1], d["topk_weights"][t0:t1], compact_slots(slots), use_fp8)
        got_x, got_s, got_w = got
        where = f"tokens [{t0}, {t1})"
        if use_fp8:
            assert_bits_equal(f"recv_x (e4m3), {where}", got_x, rx[valid])
            assert_bits_equal(f"recv_scale, {where}", got_s.view(np.uint32), rs[valid].view(np.uint32))
        else:
            assert_bits_equal(f"recv_x (bf16), {where}", got_x.view(np.uint16), rx[valid])
        assert_bits_equal(f"recv_weight, {where}", got_w.view(np.uint32), rw[valid].view(np.uint32))

    compare_in_chunks(w.T, CHUNK, fetch, check)


def check_gather_all(ref_layout, y_host, wts, gpu_out, w, weighted=True):
    """Every output token of combine (weighted) or dispatch backward against
    the oracle over the token chunk's own rows."""
    slots_all = ref_layout["slot_of_pair"].reshape(w.T, w.k)

    def fetch(t0, t1):
        return bf16_host(gpu_out[t0:t1])

    def check(t0, t1, got):
        slots = slots_all[t0:t1]
        y_sub = y_host[np.where(slots >= 0, slots, 0).reshape(-1)]
        if weighted:
            ref = oracle.combine(y_sub, wts[t0:t1], compact_slots(slots))
        else:
            ref = oracle.dispatch_backward(y_sub, compact_slots(slots), t1 - t0, w.k)
        assert_bits_equal(f"{'combine out' if weighted else 'grad_x'}, tokens [{t0}, {t1})", got, ref)

    compare_in_chunks(w.T, CHUNK, fetch, check)


def check_combine_backward_all(ref_layout, d, y_host, gpu_gy, gpu_gw, w):
    """Every grad_y row bit-exact and every grad_w entry within tolerance;
    the rms that scales the tolerance near 0 is the whole tensor's."""
    slots_all = ref_layout["slot_of_pair"].reshape(w.T, w.k)
    ref_gw = np.empty((w.T, w.k), np.float32)
    got_gw = gpu_gw.cpu().numpy()[: w.T]

    def fetch(t0, t1):
        _, rows = _rows_of(slots_all[t0:t1], gpu_gy.device)
        return bf16_host(gpu_gy.index_select(0, rows))

    def check(t0, t1, got):
        slots = slots_all[t0:t1]
        valid = slots.reshape(-1) >= 0
        y_sub = y_host[np.where(slots >= 0, slots, 0).reshape(-1)]
        rgy, rgw = oracle.combine_backward(d["g"][t0:t1], y_sub, d["topk_weights"][t0:t1], compact_slots(slots))
        assert_bits_equal(f"grad_y, tokens [{t0}, {t1})", got, rgy[valid])
        ref_gw[t0:t1] = rgw

    compare_in_chunks(w.T, CHUNK, fetch, check)
    ok, worst = grad_w_close(got_gw, ref_gw)
    assert ok, worst


# --------------------------------------------------------------- tiny, full

def test_tiny_full(cuda_device):
    w = wl.CONFIGS["tiny"]
    d = wl.make_inputs(w, parts=("routing", "x", "y", "g"))
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    assert_layout_equal(path.layout_host(), ref)
    x = to_dev(d["x"], cuda_device)
    recv = path.dispatch(x)
    rx, _, rw = oracle.dispatch(d["x"], d["topk_weights"], ref["slot_of_pair"], False)
    assert_bits_equal("recv_x", bf16_host(recv[0]), rx)
    assert_bits_equal("recv_weight", recv[2].cpu().numpy().view(np.uint32), rw.view(np.uint32))
    # identity experts: combine the dispatched rows
    out = path.combine(recv[0])
    assert_bits_equal("combine(identity)", bf16_host(out),
                      oracle.combine(rx, d["topk_weights"], ref["slot_of_pair"]))
    # random expert outputs, and both backward passes
    y = to_dev(d["y"], cuda_device)
    assert_bits_equal("combine(y)", bf16_host(path.combine(y)),
                      oracle.combine(d["y"], d["topk_weights"], ref["slot_of_pair"]))
    gy, gw = path.combine_backward(to_dev(d["g"], cuda_device), y)
    rgy, rgw = oracle.combine_backward(d["g"], d["y"], d["topk_weights"], ref["slot_of_pair"])
    assert_bits_equal("grad_y", bf16_host(gy), rgy)
    ok, worst = grad_w_close(gw.cpu().numpy(), rgw)
    assert ok, worst
    gx = path.dispatch_backward(y)
    assert_bits_equal("grad_x", bf16_host(gx), oracle.dispatch_backward(d["y"], ref["slot_of_pair"], w.T, w.k))


def test_tiny_fp8_ragged_chunk(cuda_device):
    """H = 256 is half a warp chunk: FP8 dispatch with idle lanes."""
    w = wl.CONFIGS["tiny"].with_(use_fp8=True, outlier_frac=0.02, outlier_gain=50.0)
    d = wl.make_inputs(w)
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    recv = path.dispatch(to_dev(d["x"], cuda_device))
    rx, rs, rw = oracle.dispatch(d["x"], d["topk_weights"], ref["slot_of_pair"], True)
    assert_bits_equal("recv_x", recv[0].cpu().numpy(), rx)
    assert_bits_equal("recv_scale", recv[1].cpu().numpy().view(np.uint32), rs.view(np.uint32))


# ------------------------------------------------------------- decode, full

def test_decode_full(cuda_device):
    w = wl.CONFIGS["decode"]
    d = wl.make_inputs(w, parts=("routing", "x", "y", "g"))
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    assert_layout_equal(path.layout_host(), ref)
    recv = path.dispatch(to_dev(d["x"], cuda_device))
    rx, rs, rw = oracle.dispatch(d["x"], d["topk_weights"], ref["slot_of_pair"], True)
    assert_bits_equal("recv_x", recv[0].cpu().numpy(), rx)
    assert_bits_equal("recv_scale", recv[1].cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert_bits_equal("recv_weight", recv[2].cpu().numpy().view(np.uint32), rw.view(np.uint32))
    y = to_dev(d["y"], cuda_device)
    assert_bits_equal("combine", bf16_host(path.combine(y)),
                      oracle.combine(d["y"], d["topk_weights"], ref["slot_of_pair"]))
    gy, gw = path.combine_backward(to_dev(d["g"], cuda_device), y)
    rgy, rgw = oracle.combine_backward(d["g"], d["y"], d["topk_weights"], ref["slot_of_pair"])
    assert_bits_equal("grad_y", bf16_host(gy), rgy)
    ok, worst = grad_w_close(gw.cpu().numpy(), rgw)
    assert ok, worst
    assert_bits_equal("grad_x", bf16_host(path.dispatch_backward(y)),
                      oracle.dispatch_backward(d["y"], ref["slot_of_pair"], w.T, w.k))


# ------------------------------------------- large workloads, full-size runs

@pytest.fixture(scope="module")
def prefill_inputs():
    w = wl.CONFIGS["prefill"]
    return w, wl.make_inputs(w, parts=("routing", "x", "y", "g"))


def test_prefill_layout_dispatch_combine(cuda_device, prefill_inputs):
    w, d = prefill_inputs
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    assert_layout_equal(path.layout_host(), ref)
    recv = path.dispatch(to_dev(d["x"], cuda_device))
    check_dispatch_all(ref, d, recv, True, w)
    del recv
    y = to_dev(d["y"], cuda_device)
    out = path.combine(y)
    check_gather_all(ref, d["y"], d["topk_weights"], out, w)
    del y, out
    torch.cuda.empty_cache()


def test_prefill_backward_passes(cuda_device, prefill_inputs):
    """Both backward passes at the prefill shape (H = 7168), in the launch
    configuration the benchmark times: every grad_y row bit-exact, every
    grad_w entry within tolerance, every grad_x token bit-exact."""
    w, d = prefill_inputs
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    y = to_dev(d["y"], cuda_device)
    gy, gw = path.combine_backward(to_dev(d["g"], cuda_device), y)
    check_combine_backward_all(ref, d, d["y"], gy, gw, w)
    gx = path.dispatch_backward(y)  # the expert-output draw serves as grad_recv
    check_gather_all(ref, d["y"], d["topk_weights"], gx, w, weighted=False)
    del y, gy, gw, gx
    torch.cuda.empty_cache()


def test_skewed_bf16_and_fp8(cuda_device):
    w = wl.CONFIGS["skewed"]
    d = wl.make_inputs(w, parts=("routing", "x", "y"))
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    counts = ref["num_tokens_per_expert"]
    assert counts.max() > 0.10 * w.T * w.k  # a hot expert takes > 10 % of the pairs
    x = to_dev(d["x"], cuda_device)
    for use_fp8 in (False, True):
        path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device, use_fp8=use_fp8).layout()
        assert_layout_equal(path.layout_host(), ref)
        recv = path.dispatch(x)
        check_dispatch_all(ref, d, recv, use_fp8, w)
        del recv
    y = to_dev(d["y"], cuda_device)
    check_gather_all(ref, d["y"], d["topk_weights"], path.combine(y), w)
    del y
    torch.cuda.empty_cache()


def test_backward_workload(cuda_device):
    w = wl.CONFIGS["backward"]
    d = wl.make_inputs(w, parts=("routing", "y", "g"))
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    assert_layout_equal(path.layout_host(), ref)
    y = to_dev(d["y"], cuda_device)
    g = to_dev(d["g"], cuda_device)
    gy, gw = path.combine_backward(g, y)
    check_combine_backward_all(ref, d, d["y"], gy, gw, w)
    # grad_x through the dispatch backward (the expert-output draw serves as grad_recv)
    gx = path.dispatch_backward(y)
    check_gather_all(ref, d["y"], d["topk_weights"], gx, w, weighted=False)
    del y, g, gy, gx
    torch.cuda.empty_cache()

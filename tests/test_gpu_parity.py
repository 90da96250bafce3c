"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Bar: layout, slot maps, BF16 payloads, E4M3 payload bytes, fp32 scales and
gate weights bit-exact; combine and dispatch_backward bit-exact (the stated
tolerance is 1 bf16 ulp; both sides run the same fixed-order chain);
grad_y bit-exact; grad_w within 1e-2 relative (or 1e-2 of the rms where the
dot product is near 0).

The two small workloads are compared in full.  The three large ones (the
launch configuration the benchmark times) compare the full layout, then
every output row of a sample of tokens (random tokens plus each virtual
rank's first and last), plus size-independent properties over all rows."""

import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import (GpuPath, assert_bits_equal, assert_layout_equal, bf16_host, grad_w_close,
                      sample_tokens, to_dev)

pytestmark = pytest.mark.gpu


def compact_slots(slots_tk: np.ndarray) -> np.ndarray:
    """Slots of a token subset renumbered 0..n*k-1 (masked pairs stay -1)."""
    n, k = slots_tk.shape
    c = np.arange(n * k, dtype=np.int32).reshape(n, k)
    return np.where(slots_tk >= 0, c, -1).reshape(-1)


def check_dispatch_rows(ref_layout, d, gpu_recv, tokens, use_fp8, w):
    """GPU receive rows of `tokens` against the oracle's dispatch of them."""
    slots = ref_layout["slot_of_pair"].reshape(w.T, w.k)[tokens]
    cs = compact_slots(slots)
    rx, rs, rw = oracle.dispatch(d["x"][tokens], d["topk_weights"][tokens], cs, use_fp8)
    valid = slots.reshape(-1) >= 0
    rows = slots.reshape(-1)[valid]
    g_rx, g_rs, g_rw = gpu_recv
    rows_t = torch.from_numpy(rows.astype(np.int64)).to(g_rx.device)
    got_x = g_rx.index_select(0, rows_t).cpu().numpy()
    if use_fp8:
        assert_bits_equal("recv_x (e4m3)", got_x, rx[valid])
        got_s = g_rs.index_select(0, rows_t).cpu().numpy()
        assert_bits_equal("recv_scale", got_s.view(np.uint32), rs[valid].view(np.uint32))
    else:
        assert_bits_equal("recv_x (bf16)", got_x.view(np.uint16), rx[valid])
    got_w = g_rw.index_select(0, rows_t).cpu().numpy()
    assert_bits_equal("recv_weight", got_w.view(np.uint32), rw[valid].view(np.uint32))


def check_combine_rows(ref_layout, y_host, wts, gpu_out, tokens, w, weighted=True):
    slots = ref_layout["slot_of_pair"].reshape(w.T, w.k)[tokens]
    cs = compact_slots(slots)
    y_sub = y_host[np.where(slots >= 0, slots, 0).reshape(-1)]
    if weighted:
        ref = oracle.combine(y_sub, wts[tokens], cs)
    else:
        ref = oracle.dispatch_backward(y_sub, cs, len(tokens), w.k)
    got = bf16_host(gpu_out[torch.from_numpy(tokens).to(gpu_out.device)])
    assert_bits_equal("combine out" if weighted else "grad_x", got, ref)


def check_properties_all_rows(path, ref_layout, gpu_recv, w):
    """Size-independent checks over every row: each row carries the gate weight
    of its source pair, and all k copies of a token's payload and scales are equal."""
    g_rx, g_rs, g_rw = gpu_recv
    dev = g_rx.device
    src = torch.from_numpy(ref_layout["src_of_slot"].astype(np.int64)).to(dev)
    valid = src >= 0
    assert torch.equal(g_rw[valid], path.wts.reshape(-1)[src[valid]])
    slots = torch.from_numpy(ref_layout["slot_of_pair"].astype(np.int64)).to(dev).reshape(w.T, w.k)
    for t0 in range(0, w.T, 1024):
        s = slots[t0:t0 + 1024]
        rows = g_rx[s.reshape(-1)].reshape(s.shape[0], w.k, -1)
        assert torch.equal(rows, rows[:, :1].expand_as(rows))
        if g_rs is not None:
            sc = g_rs[s.reshape(-1)].reshape(s.shape[0], w.k, -1)
            assert torch.equal(sc, sc[:, :1].expand_as(sc))


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
    tokens = sample_tokens(w.T, w.R, 2048)
    recv = path.dispatch(to_dev(d["x"], cuda_device))
    check_dispatch_rows(ref, d, recv, tokens, True, w)
    check_properties_all_rows(path, ref, recv, w)
    del recv
    y = to_dev(d["y"], cuda_device)
    out = path.combine(y)
    check_combine_rows(ref, d["y"], d["topk_weights"], out, tokens, w)
    del y, out
    torch.cuda.empty_cache()


def test_prefill_backward_passes(cuda_device, prefill_inputs):
    """Both backward passes at the prefill shape (H = 7168), in the launch
    configuration the benchmark times: grad_y bit-exact and grad_w within
    tolerance on sampled tokens, grad_x bit-exact on the same tokens."""
    w, d = prefill_inputs
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    tokens = sample_tokens(w.T, w.R, 1024, seed=7)
    y = to_dev(d["y"], cuda_device)
    gy, gw = path.combine_backward(to_dev(d["g"], cuda_device), y)
    slots = ref["slot_of_pair"].reshape(w.T, w.k)[tokens]
    y_sub = d["y"][np.where(slots >= 0, slots, 0).reshape(-1)]
    rgy, rgw = oracle.combine_backward(d["g"][tokens], y_sub, d["topk_weights"][tokens], compact_slots(slots))
    rows = torch.from_numpy(slots.reshape(-1).astype(np.int64)).to(cuda_device)
    assert_bits_equal("grad_y", bf16_host(gy.index_select(0, rows)), rgy)
    ok, worst = grad_w_close(gw[torch.from_numpy(tokens).to(cuda_device)].cpu().numpy(), rgw)
    assert ok, worst
    gx = path.dispatch_backward(y)  # the expert-output draw serves as grad_recv
    check_combine_rows(ref, d["y"], d["topk_weights"], gx, tokens, w, weighted=False)
    del y, gy, gw, gx
    torch.cuda.empty_cache()


def test_skewed_bf16_and_fp8(cuda_device):
    w = wl.CONFIGS["skewed"]
    d = wl.make_inputs(w, parts=("routing", "x", "y"))
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    counts = ref["num_tokens_per_expert"]
    assert counts.max() > 0.10 * w.T * w.k  # a hot expert takes > 10 % of the pairs
    tokens = sample_tokens(w.T, w.R, 2048)
    x = to_dev(d["x"], cuda_device)
    for use_fp8 in (False, True):
        path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device, use_fp8=use_fp8).layout()
        assert_layout_equal(path.layout_host(), ref)
        recv = path.dispatch(x)
        check_dispatch_rows(ref, d, recv, tokens, use_fp8, w)
        check_properties_all_rows(path, ref, recv, w)
        del recv
    y = to_dev(d["y"], cuda_device)
    check_combine_rows(ref, d["y"], d["topk_weights"], path.combine(y), tokens, w)
    del y
    torch.cuda.empty_cache()


def test_backward_workload(cuda_device):
    w = wl.CONFIGS["backward"]
    d = wl.make_inputs(w, parts=("routing", "y", "g"))
    ref = oracle.layout(d["topk_idx"], w.E, w.R)
    path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
    assert_layout_equal(path.layout_host(), ref)
    tokens = sample_tokens(w.T, w.R, 2048)
    y = to_dev(d["y"], cuda_device)
    g = to_dev(d["g"], cuda_device)
    gy, gw = path.combine_backward(g, y)
    slots = ref["slot_of_pair"].reshape(w.T, w.k)[tokens]
    cs = compact_slots(slots)
    y_sub = d["y"][np.where(slots >= 0, slots, 0).reshape(-1)]
    rgy, rgw = oracle.combine_backward(d["g"][tokens], y_sub, d["topk_weights"][tokens], cs)
    rows = torch.from_numpy(slots.reshape(-1).astype(np.int64)).to(cuda_device)
    assert_bits_equal("grad_y", bf16_host(gy.index_select(0, rows)), rgy)
    ok, worst = grad_w_close(gw[torch.from_numpy(tokens).to(cuda_device)].cpu().numpy(), rgw)
    assert ok, worst
    # grad_x through the dispatch backward (the expert-output draw serves as grad_recv)
    gx = path.dispatch_backward(y)
    check_combine_rows(ref, d["y"], d["topk_weights"], gx, tokens, w, weighted=False)
    del y, g, gy, gx
    torch.cuda.empty_cache()

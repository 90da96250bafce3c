"""The padded low-latency receive layout ([E][R][M] rows) against the oracle.

Layout (slots, counts, offsets, is_token_in_rank, the row -> pair map with
-1 in unfilled rows) bit-exact; dispatch, combine and both backward passes
through the padded slots compared like the dense ones."""

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
import oracle
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import GpuPath, assert_bits_equal, assert_layout_equal, bf16_host, grad_w_close, to_dev

pytestmark = pytest.mark.gpu


def routing(T, k, E, seed, masked=0.0, duplicates=False):
    rng = np.random.default_rng(seed)
    if duplicates:
        idx = rng.integers(0, E, size=(T, k))
    else:
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    if masked:
        idx = np.where(rng.random((T, k)) < masked, -1, idx)
    return np.ascontiguousarray(idx.astype(np.int64))


def run_padded(device, T, H, k, E, R, M, use_fp8, idx, seed=0, full_path=True):
    w = wl.Workload("padded", T=T, H=H, k=k, E=E, R=R, use_fp8=use_fp8, routing="group")
    rows = E * R * M
    wts = np.random.default_rng(seed).uniform(0.01, 1.0, size=(T, k)).astype(np.float32)
    ref = oracle.layout_padded(idx, E, R, M)
    path = GpuPath(w, idx, wts, device, use_fp8=use_fp8, max_tokens_per_rank=M).layout()
    assert path.rows == rows
    assert_layout_equal(path.layout_host(), ref)
    status = ep.ep_get_error(path.handle)
    expect = (ep.ep.EP_ERR_BAD_INDEX if ref["status"] & oracle.BAD_INDEX else
              ep.ep.EP_ERR_CAPACITY if ref["status"] & oracle.CAPACITY else ep.ep.EP_OK)
    assert status == expect
    if not full_path:
        return path, ref
    slots = ref["slot_of_pair"]
    used = np.sort(slots[slots >= 0])
    x = wl.normal_bf16(T, H, seed, 1)
    recv = path.dispatch(to_dev(x, device))
    rx, rs, rw = oracle.dispatch(x, wts, slots, use_fp8, P=rows)
    t_used = torch.from_numpy(used.astype(np.int64)).to(device)
    got = recv[0].index_select(0, t_used).cpu().numpy()
    if use_fp8:
        assert_bits_equal("recv_x", got, rx[used])
        assert_bits_equal("recv_scale", recv[1].index_select(0, t_used).cpu().numpy().view(np.uint32),
                          rs[used].view(np.uint32))
    else:
        assert_bits_equal("recv_x", got.view(np.uint16), rx[used])
    assert_bits_equal("recv_weight", recv[2].index_select(0, t_used).cpu().numpy().view(np.uint32),
                      rw[used].view(np.uint32))
    y = wl.normal_bf16(rows, H, seed, 2)
    g = wl.normal_bf16(T, H, seed, 3, 0.01)
    yd = to_dev(y, device)
    assert_bits_equal("combine", bf16_host(path.combine(yd))[:T], oracle.combine(y, wts, slots))
    gy, gw = path.combine_backward(to_dev(g, device), yd)
    rgy, rgw = oracle.combine_backward(g, y, wts, slots, P=rows)
    assert_bits_equal("grad_y", bf16_host(gy.index_select(0, t_used)), rgy[used])
    ok, worst = grad_w_close(gw.cpu().numpy()[:T], rgw)
    assert ok, worst
    assert_bits_equal("grad_x", bf16_host(path.dispatch_backward(yd))[:T], oracle.dispatch_backward(y, slots, T, k))
    return path, ref


@pytest.mark.parametrize("M", [64, 96])
@pytest.mark.parametrize("use_fp8", [True, False])
def test_padded_low_latency_shape(cuda_device, M, use_fp8):
    """8 ranks x 64 tokens, top-8 of 64 experts, H = 2048 (TMA dispatch)."""
    T, H, k, E, R = 512, 2048, 8, 64, 8
    run_padded(cuda_device, T, H, k, E, R, M, use_fp8, routing(T, k, E, seed=M))


@pytest.mark.parametrize("R", [1, 3, 16, 32])
def test_padded_rank_counts(cuda_device, R):
    """Up to 8 ranks the layout is one cluster of R CTAs that sums the totals
    through distributed shared memory (R = 1 and an odd R = 3 included);
    past 8 the totals are atomics into zeroed arrays."""
    T, H, k, E = 384, 256, 4, 96
    run_padded(cuda_device, T, H, k, E, R, T // R + 2, R % 2 == 1, routing(T, k, E, seed=R, masked=0.1))


def test_padded_max_ranks(cuda_device):
    """R = 256 ranks (the maximum), one expert per rank, 2 tokens per rank."""
    T, H, k, E, R = 512, 256, 4, 256, 256
    run_padded(cuda_device, T, H, k, E, R, T // R + 2, False, routing(T, k, E, seed=11, masked=0.1))


def test_padded_capacity_overflow_masked_and_bad(cuda_device):
    T, H, k, E, R = 64, 256, 4, 8, 4
    idx = routing(T, k, E, seed=3, masked=0.2, duplicates=True)
    idx[0] = 2  # one token sends all k pairs to expert 2: its rank's block overflows M = T/R
    run_padded(cuda_device, T, H, k, E, R, T // R, True, idx)
    bad = idx.copy()
    bad[5, 1] = E + 3
    path, ref = run_padded(cuda_device, T, H, k, E, R, T // R + 4, False, bad)
    assert ref["status"] & oracle.BAD_INDEX


def test_padded_empty(cuda_device):
    T, H, k, E, R, M = 0, 128, 8, 16, 4, 4
    run_padded(cuda_device, T, H, k, E, R, M, True, np.zeros((0, k), np.int64), full_path=False)


def test_padded_limits(cuda_device):
    """(T/R)*k = 8192 pairs per source rank, k = 32, E = 512."""
    T, H, k, E, R = 2048, 128, 32, 512, 8
    run_padded(cuda_device, T, H, k, E, R, T // R, True, routing(T, k, E, seed=9))


def test_padded_decode_workload_layout(cuda_device):
    w = wl.CONFIGS["decode"]
    idx, _, _ = wl.routing(w)
    run_padded(cuda_device, w.T, w.H, w.k, w.E, w.R, w.T // w.R, True, idx, full_path=False)

"""Edge cases of the CUDA path against the oracle, compared in full:
masked (-1) and duplicate pairs, out-of-range ids, the empty input, k = 1 and
the k / E maxima, one rank and one expert per rank, ragged hidden sizes and
layout tiles, every pair on one expert, a one-SM grid, large batches on the
whole GPU and under an SM budget, FP8 rounding ties,
zeros and subnormal codes, and run-to-run determinism."""

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
import oracle
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import GpuPath, assert_bits_equal, assert_layout_equal, bf16_host, grad_w_close, to_dev

pytestmark = pytest.mark.gpu


def weights(T, k, seed=0):
    rng = np.random.default_rng(seed)
    return rng.uniform(0.01, 1.0, size=(T, k)).astype(np.float32)


def run_and_compare(device, T, H, k, E, R, use_fp8, idx, x=None, num_sms=0, seed=0):
    w = wl.Workload("edge", T=T, H=H, k=k, E=E, R=R, use_fp8=use_fp8, routing="group")
    wts = weights(T, k, seed)
    if x is None:
        x = wl.normal_bf16(T, H, seed, 1)
    y = wl.normal_bf16(T * k, H, seed, 2)
    g = wl.normal_bf16(T, H, seed, 3, 0.01)
    ref = oracle.layout(idx, E, R)
    path = GpuPath(w, idx, wts, device, use_fp8=use_fp8, num_sms=num_sms).layout()
    assert_layout_equal(path.layout_host(), ref)
    recv = path.dispatch(to_dev(x, device))
    rx, rs, rw = oracle.dispatch(x, wts, ref["slot_of_pair"], use_fp8)
    n = int(ref["expert_offset"][-1])  # rows that hold a pair
    got_x = recv[0].cpu().numpy()[:n]
    if use_fp8:
        assert_bits_equal("recv_x", got_x, rx[:n])
        assert_bits_equal("recv_scale", recv[1].cpu().numpy()[:n].view(np.uint32), rs[:n].view(np.uint32))
    else:
        assert_bits_equal("recv_x", got_x.view(np.uint16), rx[:n])
    assert_bits_equal("recv_weight", recv[2].cpu().numpy()[:n].view(np.uint32), rw[:n].view(np.uint32))
    yd = to_dev(y, device)
    assert_bits_equal("combine", bf16_host(path.combine(yd))[:T],
                      oracle.combine(y, wts, ref["slot_of_pair"]))
    gy, gw = path.combine_backward(to_dev(g, device), yd)
    rgy, rgw = oracle.combine_backward(g, y, wts, ref["slot_of_pair"])
    assert_bits_equal("grad_y", bf16_host(gy)[:n], rgy[:n])
    ok, worst = grad_w_close(gw.cpu().numpy()[:T], rgw)
    assert ok, worst
    assert_bits_equal("grad_x", bf16_host(path.dispatch_backward(yd))[:T],
                      oracle.dispatch_backward(y, ref["slot_of_pair"], T, k))
    return path, ref


def random_idx(T, k, E, seed=0, masked=0.0, distinct=True):
    rng = np.random.default_rng(seed)
    if distinct:
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    else:
        idx = rng.integers(0, E, size=(T, k))
    if masked:
        idx = np.where(rng.random((T, k)) < masked, -1, idx)
    return np.ascontiguousarray(idx.astype(np.int64))


# T*k <= 16384 (with E <= 256, R <= 64) takes the one-CTA layout kernel, larger
# problems the three-kernel tiled one: the cases below run both.
@pytest.mark.parametrize("T", [96, 4096])
@pytest.mark.parametrize("use_fp8", [False, True])
def test_masked_and_duplicate_pairs(cuda_device, use_fp8, T):
    k, E, R = 6, 24, 4
    idx = random_idx(T, k, E, seed=1, masked=0.25, distinct=False)
    idx[5] = -1  # a token with no pair
    idx[7] = 3   # one expert k times
    run_and_compare(cuda_device, T, 256, k, E, R, use_fp8, idx)


@pytest.mark.parametrize("T", [32, 8192])
def test_bad_index_flagged_and_masked(cuda_device, T):
    k, E, R = 4, 16, 2
    idx = random_idx(T, k, E, seed=2)
    idx[3, 1] = E
    idx[9, 0] = -7
    idx[T - 1, 3] = 1 << 40
    path, ref = run_and_compare(cuda_device, T, 128, k, E, R, False, idx)
    assert oracle.layout(idx, E, R)["status"] == oracle.BAD_INDEX
    assert ep.ep_get_error(path.handle) == ep.ep.EP_ERR_BAD_INDEX
    assert ep.ep_get_error(path.handle) == ep.ep.EP_OK  # cleared by the read
    good = GpuPath(path.w, random_idx(T, k, E, seed=3), weights(T, k), cuda_device).layout()
    assert ep.ep_get_error(good.handle) == ep.ep.EP_OK


def test_empty_input(cuda_device):
    w = wl.Workload("empty", T=0, H=256, k=8, E=64, R=8, use_fp8=True, routing="group")
    idx = np.zeros((0, 8), np.int64)
    path = GpuPath(w, idx, np.zeros((0, 8), np.float32), cuda_device)
    path.handle.tensors["expert_offset"].fill_(-5)
    path.layout()
    got = path.layout_host()
    assert np.all(got["expert_offset"] == 0) and np.all(got["num_tokens_per_expert"] == 0)
    assert np.all(got["num_tokens_per_rank"] == 0) and np.all(got["count_src_rank_expert"] == 0)
    empty = torch.empty((1, 256), dtype=torch.int16, device=cuda_device)
    assert ep.ep_dispatch(path.shape, empty, path.wts, path.handle, torch.empty((1, 256), dtype=torch.uint8,
                          device=cuda_device), torch.empty((1, 2), device=cuda_device), None) == 0
    assert ep.ep_combine(path.shape, empty, path.wts, path.handle, empty) == 0
    assert ep.ep_get_error(path.handle) == 0


@pytest.mark.parametrize("T,H,k,E,R,use_fp8", [
    (64, 128, 1, 8, 2, True),          # k = 1
    (256, 128, 32, 1024, 8, True),     # k and E at their maxima (32-token tiles)
    (48, 136, 3, 9, 1, False),         # one rank, odd k, H % 16 == 8
    (128, 256, 4, 64, 64, False),      # one expert per rank
    (16, 8, 2, 4, 2, False),           # smallest H
    (64, 7176, 8, 32, 4, False),       # wide H with a ragged last chunk
    (32, 640, 8, 32, 4, True),         # FP8: one full chunk + one group
    (2400, 384, 8, 64, 8, True),       # 300 tokens per rank: ragged layout tiles
    (2048, 2048, 8, 256, 8, False),    # largest one-CTA layout (16384 pairs), TMA BF16 dispatch
    (2056, 2048, 8, 256, 8, True),     # just past it: tiled layout
    (512, 8192, 8, 64, 8, True),       # widest TMA dispatch (16 warps)
    (256, 8704, 4, 64, 8, False),      # past the TMA width: warp dispatch
    (300, 1024, 3, 16, 4, False),      # k = 3 with H % 512 = 0: a gather batch with unused row slots
    (256, 1536, 12, 48, 8, True),      # k = 12: a gather batch of 8 rows and one of 4
    (99, 256, 4, 48, 3, False),        # one-CTA layout tiles that straddle two source ranks
    (1024, 512, 8, 128, 16, True),     # every one-CTA layout tile holds two source ranks
    (512, 256, 8, 256, 256, False),    # R at its maximum, one expert per rank, 2 tokens per rank
    (256 * 40, 128, 4, 1024, 256, True),  # R and E at their maxima, tiled layout
])
def test_shapes(cuda_device, T, H, k, E, R, use_fp8):
    run_and_compare(cuda_device, T, H, k, E, R, use_fp8, random_idx(T, k, E, seed=T + k))


@pytest.mark.parametrize("num_sms", [0, 100])
@pytest.mark.parametrize("H,use_fp8", [(2176, True), (2560, False)])
def test_large_batch_whole_gpu_and_budget(cuda_device, H, use_fp8, num_sms):
    """4096 tokens, past 16 per SM: on the whole GPU (num_sms = 0) dispatch and
    combine backward launch oversubscribed grids, under an SM budget persistent
    ones; H = 2176 adds a ragged last chunk.  Both against the oracle in full."""
    T, k, E, R = 4096, 8, 64, 8
    run_and_compare(cuda_device, T, H, k, E, R, use_fp8, random_idx(T, k, E, seed=11), num_sms=num_sms)


def test_all_pairs_on_few_experts(cuda_device):
    T, k, E, R = 1024, 8, 256, 8
    idx = np.tile(np.arange(k, dtype=np.int64), (T, 1))  # every token -> experts 0..7 (rank 0)
    path, ref = run_and_compare(cuda_device, T, 128, k, E, R, True, idx)
    assert ref["num_tokens_per_rank"][0] == T and np.all(ref["num_tokens_per_rank"][1:] == 0)


def test_one_sm_grid(cuda_device):
    T, k, E, R = 512, 8, 64, 8
    run_and_compare(cuda_device, T, 1024, k, E, R, True, random_idx(T, k, E, seed=5), num_sms=1)


def test_fp8_ties_zeros_and_subnormals(cuda_device):
    """Rows built so that x / scale hits E4M3 rounding ties, subnormal codes,
    signed zeros, and very small and very large magnitudes."""
    T, H, k, E, R = 8, 256, 2, 4, 2
    vals = np.zeros((T, H), np.float32)
    ties = [448.0, 1.0625, 1.1875, 232.0, 0.0009765625, 0.0146484375, -0.00146484375, -0.000244140625,
            3.0, 0.001953125, -448.0, 13.0, 26.0, 52.0, 104.0, 208.0]
    vals[0, :len(ties)] = ties                   # scale exactly 1
    vals[1, :128] = 0.0                          # all-zero group: scale 1
    vals[1, 128:] = np.linspace(-3, 3, 128)
    vals[2] = np.float32(2.0 ** -120) * np.linspace(-1, 1, H)   # tiny group
    vals[3] = np.float32(1e30) * np.linspace(-1, 1, H)          # huge group
    rng = np.random.default_rng(0)
    vals[4:] = rng.standard_normal((4, H)) * np.exp2(rng.integers(-40, 40, size=(4, 1)))
    x = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    x[1, 5] = 0x8000  # -0
    idx = random_idx(T, k, E, seed=6)
    run_and_compare(cuda_device, T, H, k, E, R, True, idx, x=x)


def test_deterministic(cuda_device):
    w = wl.CONFIGS["decode"]
    d = wl.make_inputs(w, parts=("routing", "x", "y", "g"))
    outs = []
    for _ in range(2):
        path = GpuPath(w, d["topk_idx"], d["topk_weights"], cuda_device).layout()
        recv = path.dispatch(to_dev(d["x"], cuda_device))
        y = to_dev(d["y"], cuda_device)
        gy, gw = path.combine_backward(to_dev(d["g"], cuda_device), y)
        outs.append([path.layout_host()["slot_of_pair"], recv[0].cpu(), recv[1].cpu(),
                     path.combine(y).cpu(), gy.cpu(), gw.cpu(), path.dispatch_backward(y).cpu()])
    for a, b in zip(*outs):
        if isinstance(a, np.ndarray):
            assert np.array_equal(a, b)
        else:
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@pytest.mark.parametrize("T,H,use_fp8,num_sms", [
    (1024, 7040, True, 0),    # ragged last chunk (13.75 chunks)
    (1024, 6656, True, 0),    # 13 chunks
    (1024, 7168, False, 0),   # BF16 rows
    (40, 7168, True, 4),      # SM budget: several tokens per CTA, the next one prefetched into registers
    (60, 6656, False, 4),     # several tokens per CTA, the row stages reused
])
def test_small_batch_bulk_store_dispatch(cuda_device, T, H, use_fp8, num_sms):
    """Small batches with 1536 < H <= 8192: the bulk-store dispatch on a
    persistent grid, whole GPU or under an SM budget, against the oracle in
    full."""
    k, E, R = 8, 64, 4
    run_and_compare(cuda_device, T, H, k, E, R, use_fp8, random_idx(T, k, E, seed=T + H), num_sms=num_sms)


@pytest.mark.parametrize("T,H,k,masked,num_sms", [
    (96, 512, 6, 0.25, 0),     # masked and duplicate pairs, k < 8
    (1024, 1024, 1, 0.0, 0),   # k = 1
    (500, 2048, 8, 0.1, 3),    # SM budget: each warp strides over many units
    (4, 512, 8, 0.0, 0),       # fewer units than warps
])
def test_small_batch_gathers(cuda_device, T, H, k, masked, num_sms):
    """Small batches with k <= 8 and H a multiple of 512 (the persistent grid,
    few units per warp or fewer units than warps): combine and dispatch
    backward against the oracle in full."""
    E, R = 32, 4
    idx = random_idx(T, k, E, seed=T + k, masked=masked, distinct=masked == 0.0)
    run_and_compare(cuda_device, T, H, k, E, R, False, idx, num_sms=num_sms)


def test_portable_cluster_layout():
    """The one-launch layout with the portable 8-CTA cluster (EP_LAYOUT_CLUSTER=8;
    a B200 otherwise takes the 16-CTA one): the shape tests again, in a
    process of their own."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, EP_LAYOUT_CLUSTER="8")
    here = os.path.dirname(os.path.abspath(__file__))
    files = [os.path.join(here, f) for f in ("test_gpu_edge.py", "test_gpu_fused.py")]
    pick = "test_shapes or test_masked_and_duplicate or test_fused_matches"
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        "-k", pick] + files, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]

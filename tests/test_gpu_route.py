"""Group-limited top-k routing on the GPU against the oracle, through the
three kernels: groups on lane boundaries with the chosen groups' experts
moved onto all lanes (the compact kernel, whenever that leaves fewer per
lane) or not (the aligned kernel), and groups off lane boundaries (the
general kernel).

The selections compare input scores only, so topk_idx must match exactly
(ties included: many scores are quantised to force them); the weights are
an fp32 softmax on the GPU against float64 in the oracle (2e-6 relative)."""

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
import oracle
from gpu_util import assert_layout_equal

pytestmark = pytest.mark.gpu


def scores_for(T, E, seed, ties=True):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((T, E)).astype(np.float32)
    if ties:
        s[: T // 2] = np.round(s[: T // 2] * 4) / 4  # exact ties in half the tokens
    return s


def route_gpu(device, s, k, ng, tg, R=1):
    T, E = s.shape
    shape = ep.make_shape(T, 128, k, E, R)
    idx = torch.full((max(T, 1), k), -9, dtype=torch.int64, device=device)
    w = torch.full((max(T, 1), k), -9.0, dtype=torch.float32, device=device)
    ep.ep_route_group_limited(shape, torch.from_numpy(s).to(device), ng, tg, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy()[:T], w.cpu().numpy()[:T]


@pytest.mark.parametrize("T,E,k,ng,tg", [
    # groups on lane boundaries; (experts per lane, candidates per lane) of
    # the compact kernel in brackets, "aligned" where it would not help
    (1024, 256, 8, 8, 4),      # decode shape: top-4 of 8 groups, top-8 experts (8, 4)
    (32768, 256, 8, 8, 4),     # prefill shape (8, 4)
    (300, 48, 6, 3, 2),        # E not a multiple of 32, 16 experts per group (2, 1)
    (200, 64, 5, 1, 1),        # one group: plain top-k (aligned)
    (77, 256, 3, 32, 1),       # one group of 8 chosen out of 32 (8, 1)
    (512, 1024, 32, 32, 16),   # E and k at their maxima, 32 groups (32, 16)
    (100, 16, 16, 4, 4),       # every expert chosen (aligned)
    (333, 512, 8, 16, 4),      # 16 experts per lane (16, 4)
    (250, 128, 8, 8, 4),       # the backward shape's 128 experts (4, 2)
    (129, 128, 8, 8, 3),       # 48 candidates: lanes 24 to 31 hold none (4, 2)
    # groups off lane boundaries: 12 experts per group over lanes of 4, 40
    # over lanes of 8, E not a multiple of the experts per lane
    (257, 96, 8, 8, 4),
    (150, 160, 8, 4, 2),
    (200, 33, 4, 3, 2),
    (257, 96, 12, 8, 4),
    (150, 160, 10, 4, 2),
    (64, 300, 9, 3, 2),
])
def test_route_matches_oracle(cuda_device, T, E, k, ng, tg):
    s = scores_for(T, E, seed=T + E + k)
    idx, w = route_gpu(cuda_device, s, k, ng, tg)
    ridx, rw = oracle.route_group_limited(s, k, ng, tg)
    assert np.array_equal(idx, ridx)
    assert np.allclose(w, rw, rtol=2e-6, atol=0)


def test_route_then_layout(cuda_device):
    """Routing feeds the layout: the whole front of the path on the GPU
    against oracle routing followed by the oracle layout."""
    T, E, k, ng, tg, R = 2048, 256, 8, 8, 4, 8
    s = scores_for(T, E, seed=5, ties=False)
    shape = ep.make_shape(T, 128, k, E, R)
    idx = torch.empty((T, k), dtype=torch.int64, device=cuda_device)
    w = torch.empty((T, k), dtype=torch.float32, device=cuda_device)
    ep.ep_route_group_limited(shape, torch.from_numpy(s).to(cuda_device), ng, tg, idx, w)
    h = ep.Handle(shape, cuda_device)
    ep.ep_get_dispatch_layout(shape, idx, h, ep.workspace(shape, cuda_device))
    torch.cuda.synchronize()
    ridx, _ = oracle.route_group_limited(s, k, ng, tg)
    ref = oracle.layout(ridx, E, R)
    got = {n: h.tensors[n].cpu().numpy()[: ep.handle_sizes(shape)[n]] for n in ref if n != "status"}
    assert_layout_equal(got, {n: v for n, v in ref.items() if n != "status"})


def test_route_empty(cuda_device):
    idx, w = route_gpu(cuda_device, np.zeros((0, 64), np.float32), 4, 4, 2)
    assert idx.shape == (0, 4)


_DEBUG_SCRIPT = r'''
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
import combine_ep_get_histogram_b200 as ep
import oracle
from test_gpu_route import scores_for
dev = torch.device("cuda:0")
for (T, E, k, ng, tg) in ((1024, 256, 8, 8, 4), (200, 64, 5, 1, 1), (257, 96, 8, 8, 4)):  # the three kernels
    s = scores_for(T, E, seed=3)
    sd = torch.from_numpy(s).to(dev)
    idx = torch.empty((T, k), dtype=torch.int64, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    torch.cuda._sleep(100_000_000)  # keeps the stream busy for tens of milliseconds
    ep.ep_route_group_limited(ep.make_shape(T, 128, k, E, 1), sd, ng, tg, idx, w)
    # with EP_DEBUG=1 the call synchronised the stream before it returned
    assert torch.cuda.current_stream().query(), "EP_DEBUG=1 did not synchronise the router call"
    ridx, rw = oracle.route_group_limited(s, k, ng, tg)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=0)
print("debug ok")
'''


def test_route_under_ep_debug(cuda_device):
    """EP_DEBUG=1 checks every call, the router's three kernels included: the
    call returns only after its stream has drained (and reports any error the
    kernel raised), and the results still match the oracle."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, EP_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", _DEBUG_SCRIPT, root], capture_output=True, text=True, timeout=300,
                       env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "debug ok" in r.stdout

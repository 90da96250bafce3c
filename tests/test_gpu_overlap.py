"""SM budget and overlap with compute.

The caller decides how many SMs the dispatch / combine kernels may fill, so
that its own compute can run beside them
("deepep-expert-parallel-communication-library", section 二 SM 资源控制; the
DeepEP guide's async / compute-stream options, "DeepEP：MoE 专家并行 EP 通信
kernel 编译与使用指南",
section 五).  Here the whole path runs on a side stream with a small
``num_sms`` while a cuBLAS GEMM runs on the launching stream, the two ordered
only by events.  Every output must be bit-identical to a plain run of the
path on all SMs, and the combined output must equal the oracle's."""

import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_histogram_b200 import workloads as wl
from gpu_util import StepBuffers, assert_bits_equal, bf16_host

pytestmark = pytest.mark.gpu

# prefill shape (H=7168, E=256, k=8, 8 ranks, FP8 dispatch) at 256 tokens per rank
W = wl.CONFIGS["prefill"].with_(T=8 * 256)


@pytest.fixture(scope="module")
def plain(cuda_device):
    d = wl.make_inputs(W, parts=("routing", "x", "y", "g"))
    ref = StepBuffers(W, cuda_device)
    ref.load(d)
    ref.run()
    out = ref.outputs()
    lay = oracle.layout(d["topk_idx"], W.E, W.R)
    assert_bits_equal("combine", bf16_host(ref.out), oracle.combine(d["y"], d["topk_weights"], lay["slot_of_pair"]))
    return d, out


@pytest.mark.parametrize("num_sms", [1, 8, 37])
def test_budgeted_path_on_a_side_stream_beside_a_gemm(cuda_device, plain, num_sms):
    d, expected = plain
    path = StepBuffers(W, cuda_device, num_sms=num_sms)
    path.load(d)
    gen = torch.Generator(device=cuda_device).manual_seed(0)
    a = torch.randn((4096, 4096), device=cuda_device, dtype=torch.bfloat16, generator=gen)
    b = torch.randn((4096, 4096), device=cuda_device, dtype=torch.bfloat16, generator=gen)
    c_ref = torch.matmul(a, b)
    c = torch.empty_like(c_ref)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream(cuda_device)
    torch.cuda.synchronize()

    ready = torch.cuda.Event()
    ready.record(main)
    side.wait_event(ready)
    with torch.cuda.stream(side):
        path.run()
    for _ in range(4):  # enqueued after the path, so the two overlap on the device
        torch.matmul(a, b, out=c)
    done = torch.cuda.Event()
    done.record(side)
    main.wait_event(done)
    torch.cuda.synchronize()

    got = path.outputs()
    for i, (x, y) in enumerate(zip(got, expected)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), i
    torch.testing.assert_close(c.float(), c_ref.float(), rtol=1e-2, atol=1e-1)


def test_budget_beyond_the_device_means_all_sms(cuda_device, plain):
    d, expected = plain
    path = StepBuffers(W, cuda_device, num_sms=100000)
    path.load(d)
    path.run()
    for i, (x, y) in enumerate(zip(path.outputs(), expected)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), i

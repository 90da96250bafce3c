"""The scratch-free layout entry point (ep_get_dispatch_layout_noalloc).

It serves callers that cannot allocate device memory: code running while a
CUDA graph is captured, code inside another framework's allocator hooks, and
hosts with a fixed device-memory budget.  Instead of a caller workspace it
uses one fixed 1 MiB array inside the library.  These tests check that two
calls in a row, with different routings (so the second call starts from the
first call's leftover scratch), give exactly the handle that the workspace
entry point gives, and that shapes needing more scratch are refused before
anything is enqueued.  This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
from combine_ep_get_histogram_b200 import ep as binding
from combine_ep_get_histogram_b200 import workloads as wl

LAYOUT_FIELDS = ("num_tokens_per_expert", "expert_offset", "num_tokens_per_rank", "count_src_rank_expert",
                 "src_rank_expert_offset", "is_token_in_rank", "slot_of_pair", "src_of_slot", "error_word")


def test_noalloc_refuses_shapes_beyond_its_scratch():
    lib = ep.library()
    cap = lib.ep_noalloc_scratch_bytes()
    assert cap == 1 << 20
    s = ep.make_shape(T=8 * 1_000_000, H=128, k=8, E=1024, R=8)
    assert ep.workspace_size(s) > cap
    h = binding.ep_handle_t(*([4096] * 9))  # never dereferenced: the size check comes first
    st = lib.ep_get_dispatch_layout_noalloc(ctypes.byref(s), 4096, ctypes.byref(h), None)
    assert st == binding.EP_ERR_SCRATCH_TOO_SMALL
    assert "scratch" in binding.status_string(st)


@pytest.mark.gpu
def test_noalloc_layout_matches_workspace_layout_twice(cuda_device):
    for name in ("prefill", "skewed"):  # two calls in a row, different routings and sizes
        w = wl.CONFIGS[name]
        idx_np, _, _ = wl.routing(w)
        idx = torch.from_numpy(idx_np).to(cuda_device)
        shape = ep.make_shape(w.T, w.H, w.k, w.E, w.R, w.use_fp8)
        assert ep.workspace_size(shape) <= ep.library().ep_noalloc_scratch_bytes()
        ref = ep.Handle(shape, cuda_device)
        ep.ep_get_dispatch_layout(shape, idx, ref, ep.workspace(shape, cuda_device))
        got = ep.Handle(shape, cuda_device)
        for f in LAYOUT_FIELDS:
            got.tensors[f].fill_(-3 if got.tensors[f].dtype != torch.uint8 else 7)
        got.tensors["error_word"].zero_()
        ep.ep_get_dispatch_layout_noalloc(shape, idx, got)
        torch.cuda.synchronize()
        for f in LAYOUT_FIELDS:
            a, b = got.tensors[f].cpu().numpy(), ref.tensors[f].cpu().numpy()
            assert np.array_equal(a, b), (name, f)
        assert ep.ep_get_error(got) == binding.EP_OK

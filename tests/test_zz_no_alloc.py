"""The scratch-free layout entry point (ep_get_dispatch_layout_noalloc).

It serves callers that may not allocate device memory: code inside another
framework's allocator or memory-pool hooks, and hosts whose device memory is
fixed at start-up.  Instead of a caller workspace it uses one fixed 1 MiB
array inside the library.  These tests check that two calls in a row, with
different routings (so the second call starts from the first call's leftover
scratch), give exactly the handle that the workspace entry point gives, and
that bad arguments and shapes needing more scratch are refused before
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
    # aligned, non-null host-side stand-ins: they pass the argument checks and
    # are never dereferenced, because the size check refuses the shape next
    h = binding.ep_handle_t(*([4096] * 9))
    st = lib.ep_get_dispatch_layout_noalloc(ctypes.byref(s), 4096, ctypes.byref(h), None)
    assert st == binding.EP_ERR_SCRATCH_TOO_SMALL
    assert "scratch" in binding.status_string(st)


def test_noalloc_checks_arguments_before_the_scratch_size():
    """Same argument errors as ep_get_dispatch_layout, whatever the size."""
    lib = ep.library()
    big = ep.make_shape(T=8 * 1_000_000, H=128, k=8, E=1024, R=8)
    h = binding.ep_handle_t(*([4096] * 9))
    assert lib.ep_get_dispatch_layout_noalloc(ctypes.byref(big), 4096, None, None) == binding.EP_ERR_INVALID_ARG
    assert lib.ep_get_dispatch_layout_noalloc(ctypes.byref(big), None, ctypes.byref(h), None) == \
        binding.EP_ERR_INVALID_ARG
    assert lib.ep_get_dispatch_layout_noalloc(ctypes.byref(big), 4100, ctypes.byref(h), None) == \
        binding.EP_ERR_INVALID_ARG  # topk_idx not 8-byte aligned
    bad = binding.ep_handle_t(*([4096] * 8 + [0]))  # no error word
    assert lib.ep_get_dispatch_layout_noalloc(ctypes.byref(big), 4096, ctypes.byref(bad), None) == \
        binding.EP_ERR_INVALID_ARG
    odd = ep.make_shape(T=63, H=256, k=4, E=16, R=4)  # T % R != 0
    assert lib.ep_get_dispatch_layout_noalloc(ctypes.byref(odd), 4096, ctypes.byref(h), None) == \
        binding.EP_ERR_INVALID_ARG


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


# Run in a fresh process: the primary context, then a second context created
# with the driver API on the same device, then the primary context again.
# Each context has its own address for the library's scratch array, so a
# call in the second context must not reuse the first context's address.
_CONTEXTS_SCRIPT = r'''
import ctypes, sys
import numpy as np
sys.path.insert(0, sys.argv[1])
from cuda.bindings import driver as cu
import combine_ep_get_histogram_b200 as ep
from combine_ep_get_histogram_b200 import ep as binding
from combine_ep_get_histogram_b200 import workloads as wl

def ok(r):
    err = r[0] if isinstance(r, tuple) else r
    assert err == cu.CUresult.CUDA_SUCCESS, err
    return r[1] if isinstance(r, tuple) and len(r) == 2 else r

lib = ep.library()
ok(cu.cuInit(0))
dev = ok(cu.cuDeviceGet(0))

def run(label, w):
    idx_np, _, _ = wl.routing(w)
    shape = ep.make_shape(w.T, w.H, w.k, w.E, w.R, w.use_fp8)
    sizes = ep.handle_sizes(shape)
    elem = {n: (1 if n == "is_token_in_rank" else 4) for n in sizes}
    bufs = []
    def alloc(nbytes):
        p = int(ok(cu.cuMemAlloc(max(nbytes, 256))))
        bufs.append(p)
        return p
    idx = alloc(idx_np.nbytes)
    ok(cu.cuMemcpyHtoD(idx, idx_np.ctypes.data, idx_np.nbytes))
    handles = []
    for fill in (0x11, 0x7d):  # the no-alloc handle starts from garbage
        ptrs = []
        for n in binding.HANDLE_FIELDS:
            p = alloc(sizes[n] * elem[n])
            ok(cu.cuMemsetD8(p, 0 if n == "error_word" else fill, sizes[n] * elem[n]))
            ptrs.append(p)
        handles.append(binding.ep_handle_t(*ptrs))
    ws_bytes = ep.workspace_size(shape)
    ws = alloc(ws_bytes)
    assert lib.ep_get_dispatch_layout(ctypes.byref(shape), idx, ctypes.byref(handles[0]), ws, ws_bytes, None) == 0
    assert lib.ep_get_dispatch_layout_noalloc(ctypes.byref(shape), idx, ctypes.byref(handles[1]), None) == 0
    ok(cu.cuCtxSynchronize())
    for i, n in enumerate(binding.HANDLE_FIELDS):
        nb = sizes[n] * elem[n]
        a, b = np.empty(nb, np.uint8), np.empty(nb, np.uint8)
        ok(cu.cuMemcpyDtoH(a.ctypes.data, getattr(handles[0], n), nb))
        ok(cu.cuMemcpyDtoH(b.ctypes.data, getattr(handles[1], n), nb))
        assert np.array_equal(a, b), (label, n)
    assert lib.ep_get_error(ctypes.byref(handles[1]), None) == 0
    for p in bufs:
        ok(cu.cuMemFree(p))
    print(label, "ok")

primary = ok(cu.cuDevicePrimaryCtxRetain(dev))
ok(cu.cuCtxSetCurrent(primary))
run("primary", wl.CONFIGS["decode"])
second = ok(cu.cuCtxCreate(0, dev))  # becomes current
run("second", wl.CONFIGS["prefill"])
run("second again", wl.CONFIGS["decode"])
ok(cu.cuCtxSetCurrent(primary))
run("primary again", wl.CONFIGS["skewed"])
ok(cu.cuCtxDestroy(second))
ok(cu.cuDevicePrimaryCtxRelease(dev))
print("contexts ok")
'''


@pytest.mark.gpu
def test_noalloc_in_a_second_context(cuda_device):
    """The scratch address is looked up per CUDA context: calls in a context
    created with the driver API, and back in the primary context, give the
    workspace entry point's handle."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _CONTEXTS_SCRIPT, root], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "contexts ok" in r.stdout

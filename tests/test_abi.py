"""The C ABI library loads, exports every entry point include/ep.h declares,
and rejects bad arguments on the host before any CUDA call (no GPU needed)."""

import ctypes
import os
import re

import pytest

import combine_ep_get_histogram_b200 as ep
from combine_ep_get_histogram_b200 import ep as binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ep.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("ep_get_dispatch_layout", "ep_dispatch", "ep_combine", "ep_combine_backward",
              "ep_dispatch_backward", "ep_get_error", "ep_workspace_size", "ep_handle_sizes"):
        assert n in names
    assert set(names) == set(binding.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings():
    for st in range(7):
        assert binding.status_string(st).startswith("EP_")


def test_handle_sizes_and_workspace():
    s = ep.make_shape(T=64, H=256, k=4, E=16, R=4)
    sizes = ep.handle_sizes(s)
    assert sizes == {"num_tokens_per_expert": 16, "expert_offset": 17, "num_tokens_per_rank": 4,
                     "count_src_rank_expert": 64, "src_rank_expert_offset": 64,
                     "is_token_in_rank": 256, "slot_of_pair": 256, "src_of_slot": 256,
                     "error_word": 1}
    ws = ep.workspace_size(s)
    assert ws > 0 and ws % 256 == 0
    big = ep.make_shape(T=32768, H=7168, k=8, E=256, R=8, use_fp8=True)
    # (E + R) columns x (8 ranks x 32 tiles of 128 tokens), plus the totals
    assert ep.workspace_size(big) == (264 * 256 * 4 + 255) // 256 * 256 + (264 * 4 + 255) // 256 * 256


BAD_SHAPES = [
    dict(T=63, H=256, k=4, E=16, R=4),      # T % R
    dict(T=64, H=256, k=4, E=18, R=4),      # E % R
    dict(T=64, H=256, k=0, E=16, R=4),      # k < 1
    dict(T=64, H=256, k=33, E=64, R=4),     # k > 32
    dict(T=64, H=256, k=4, E=2048, R=4),    # E > 1024
    dict(T=64, H=250, k=4, E=16, R=4),      # H % 8
    dict(T=64, H=320, k=4, E=16, R=4, use_fp8=True),  # H % 128 with FP8
    dict(T=64, H=256, k=4, E=4, R=8),       # R > E
    dict(T=512, H=256, k=4, E=512, R=512),  # R > 256
    dict(T=1 << 28, H=256, k=8, E=16, R=4),  # T * k >= 2^31
    dict(T=-4, H=256, k=4, E=16, R=4),
    dict(T=64, H=256, k=4, E=16, R=4, num_sms=-1),
]


@pytest.mark.parametrize("kw", BAD_SHAPES)
def test_bad_shapes_rejected_on_host(kw):
    s = ep.make_shape(**kw)
    lib = ep.library()
    assert lib.ep_workspace_size(ctypes.byref(s)) == 0
    h = binding.ep_handle_t(*([4096] * 9))
    fake = 1 << 20  # never dereferenced: validation fails first
    assert lib.ep_get_dispatch_layout(ctypes.byref(s), fake, ctypes.byref(h), fake, 1 << 20, None) == 1
    assert lib.ep_dispatch(ctypes.byref(s), fake, fake, ctypes.byref(h), fake, fake, None, None) == 1
    assert lib.ep_dispatch_with_layout(ctypes.byref(s), fake, fake, fake, ctypes.byref(h), fake, 1 << 20, fake, fake,
                                       None, None) == 1
    assert lib.ep_combine(ctypes.byref(s), fake, fake, ctypes.byref(h), fake, None) == 1
    assert lib.ep_combine_backward(ctypes.byref(s), fake, fake, fake, ctypes.byref(h), fake, fake, None) == 1
    assert lib.ep_dispatch_backward(ctypes.byref(s), fake, ctypes.byref(h), fake, None) == 1


def test_use_fp8_must_be_zero_or_one():
    s = binding.ep_shape_t(64, 256, 4, 16, 4, 2, 0, 0)  # make_shape would coerce it to 1
    assert ep.library().ep_workspace_size(ctypes.byref(s)) == 0


def test_bad_pointers_rejected_on_host():
    s = ep.make_shape(T=64, H=256, k=4, E=16, R=4, use_fp8=True)
    lib = ep.library()
    good = 1 << 20
    h = binding.ep_handle_t(*([good] * 9))
    sref, href = ctypes.byref(s), ctypes.byref(h)
    ws = ep.workspace_size(s)
    # layout: null index, misaligned index, small / misaligned workspace, null handle array
    assert lib.ep_get_dispatch_layout(sref, None, href, good, ws, None) == 1
    assert lib.ep_get_dispatch_layout(sref, good + 4, href, good, ws, None) == 1
    assert lib.ep_get_dispatch_layout(sref, good, href, good, ws - 1, None) == 1
    assert lib.ep_get_dispatch_layout(sref, good, href, good + 16, ws, None) == 1
    h2 = binding.ep_handle_t(*([good] * 6 + [0] + [good] * 2))
    assert lib.ep_get_dispatch_layout(sref, good, ctypes.byref(h2), good, ws, None) == 1
    assert lib.ep_get_dispatch_layout(sref, good, None, good, ws, None) == 1
    # dispatch: rows must be 16-byte aligned, FP8 needs recv_scale
    assert lib.ep_dispatch(sref, good + 8, good, href, good, good, None, None) == 1
    assert lib.ep_dispatch(sref, good, good, href, good + 2, good, None, None) == 1
    assert lib.ep_dispatch(sref, good, good, href, good, None, None, None) == 1
    assert lib.ep_dispatch(sref, good, good + 2, href, good, good, None, None) == 1
    # layout + dispatch in one call: every check of both before anything runs
    fused = lib.ep_dispatch_with_layout
    assert fused(sref, None, good, good, href, good, ws, good, good, None, None) == 1
    assert fused(sref, good, good + 8, good, href, good, ws, good, good, None, None) == 1
    assert fused(sref, good, good, good, href, good, ws - 1, good, good, None, None) == 1
    assert fused(sref, good, good, good, href, good, ws, good, None, None, None) == 1
    assert fused(sref, good, good, good, ctypes.byref(h2), good, ws, good, good, None, None) == 1
    assert lib.ep_combine(sref, good + 8, good, href, good, None) == 1
    assert lib.ep_combine(sref, good, good, href, None, None) == 1
    assert lib.ep_combine_backward(sref, good, good, good, href, good, None, None) == 1
    assert lib.ep_dispatch_backward(sref, good, href, good + 4, None) == 1
    assert lib.ep_get_error(None, None) == 1


def test_peer_calls_reject_bad_arguments_on_host():
    """The multi-GPU calls check rank, shape and every owner's buffer before
    any device work (no GPU needed to see the rejections)."""
    s = ep.make_shape(T=64, H=256, k=4, E=16, R=4, use_fp8=True)
    lib = ep.library()
    good = 1 << 20
    h = binding.ep_handle_t(*([good] * 9))
    sref, href = ctypes.byref(s), ctypes.byref(h)
    rows = binding.peer_rows([good] * 4)
    one_short = binding.peer_rows([good] * 3)            # owner 3 missing
    odd = binding.peer_rows([good, good + 8, good, good])  # owner 1 not 16-byte aligned
    rr = ctypes.byref(rows)
    # rank out of range, null / misaligned topk_idx, null weights
    assert lib.ep_dispatch_peers(sref, 4, good, href, good, good, rr, rr, None, None) == 1
    assert lib.ep_dispatch_peers(sref, -1, good, href, good, good, rr, rr, None, None) == 1
    assert lib.ep_dispatch_peers(sref, 0, None, href, good, good, rr, rr, None, None) == 1
    assert lib.ep_dispatch_peers(sref, 0, good + 4, href, good, good, rr, rr, None, None) == 1
    assert lib.ep_dispatch_peers(sref, 0, good, href, good, None, rr, rr, None, None) == 1
    # every owner's buffer present and aligned; FP8 needs the scale table
    assert lib.ep_dispatch_peers(sref, 0, good, href, good, good, ctypes.byref(one_short), rr, None, None) == 1
    assert lib.ep_dispatch_peers(sref, 0, good, href, good, good, ctypes.byref(odd), rr, None, None) == 1
    assert lib.ep_dispatch_peers(sref, 0, good, href, good, good, rr, None, None, None) == 1
    assert lib.ep_combine_peers(sref, 0, good, href, None, good, good, None) == 1
    assert lib.ep_combine_peers(sref, 0, good, href, ctypes.byref(odd), good, good, None) == 1
    assert lib.ep_combine_backward_peers(sref, 0, good, href, good, rr, good, None, good, None) == 1
    assert lib.ep_dispatch_backward_peers(sref, 0, good, href, rr, good + 2, None) == 1
    # more ranks than the peer table holds; the padded layout has no peer form
    big = ep.make_shape(T=128, H=256, k=4, E=128, R=128)
    assert lib.ep_combine_peers(ctypes.byref(big), 0, good, href, rr, good, good, None) == 1
    padded = ep.make_shape(T=64, H=256, k=4, E=16, R=4, max_tokens_per_rank=16)
    assert lib.ep_combine_peers(ctypes.byref(padded), 0, good, href, rr, good, good, None) == 1


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_LIB", None)
    with pytest.raises(RuntimeError, match="not built"):
        binding.library()


@pytest.mark.parametrize("ng,tg,k", [(0, 1, 2), (3, 2, 2), (8, 9, 2), (8, 2, 17), (64, 4, 2)])
def test_route_bad_arguments_rejected_on_host(ng, tg, k):
    s = ep.make_shape(T=64, H=128, k=k, E=64, R=4)
    fake = 1 << 20
    assert ep.library().ep_route_group_limited(ctypes.byref(s), fake, ng, tg, fake, fake, None) == 1


def test_ipc_calls_reject_bad_arguments_on_host():
    """The CUDA-IPC helpers check their pointers before any CUDA call."""
    lib = ep.library()
    rec = binding.ep_ipc_buffer_t()
    base, ptr = ctypes.c_void_p(), ctypes.c_void_p()
    assert ctypes.sizeof(rec) == 80
    assert lib.ep_ipc_export(None, ctypes.byref(rec)) == binding.EP_ERR_INVALID_ARG
    assert lib.ep_ipc_export(4096, None) == binding.EP_ERR_INVALID_ARG
    assert lib.ep_ipc_open(None, ctypes.byref(base), ctypes.byref(ptr)) == binding.EP_ERR_INVALID_ARG
    assert lib.ep_ipc_open(ctypes.byref(rec), None, ctypes.byref(ptr)) == binding.EP_ERR_INVALID_ARG
    assert lib.ep_ipc_open(ctypes.byref(rec), ctypes.byref(base), None) == binding.EP_ERR_INVALID_ARG
    assert lib.ep_ipc_close(None) == binding.EP_ERR_INVALID_ARG

"""ctypes binding of libep_b200.so (C ABI in include/ep.h).

Argument marshalling only: every entry point forwards device pointers and
sizes to the CUDA library, whose kernels do all the work.  There is no
fallback: if the library is missing or the device is not an sm_100 GPU the
calls raise.

The functions keep the C names (``ep_get_dispatch_layout``, ``ep_dispatch``,
``ep_combine``, ``ep_combine_backward``, ``ep_dispatch_backward``,
``ep_get_error``) and accept torch tensors (or raw integer device pointers).
``Handle`` owns the device arrays of a dispatch handle; ``workspace`` sizes
the layout scratch.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libep_b200.so")

EP_OK, EP_ERR_INVALID_ARG, EP_ERR_BAD_INDEX, EP_ERR_CUDA, EP_ERR_UNSUPPORTED = 0, 1, 2, 3, 4
EP_ERR_SCRATCH_TOO_SMALL = 5
EP_ERR_CAPACITY = 6

HANDLE_FIELDS = ("num_tokens_per_expert", "expert_offset", "num_tokens_per_rank",
                 "count_src_rank_expert", "src_rank_expert_offset", "is_token_in_rank",
                 "slot_of_pair", "src_of_slot", "error_word")

EXPORTED = ("ep_handle_sizes", "ep_workspace_size", "ep_get_dispatch_layout", "ep_dispatch",
            "ep_dispatch_with_layout",
            "ep_combine", "ep_combine_backward", "ep_dispatch_backward", "ep_get_error",
            "ep_status_string", "ep_last_cuda_error", "ep_get_dispatch_layout_noalloc",
            "ep_noalloc_scratch_bytes", "ep_route_group_limited", "ep_dispatch_peers", "ep_combine_peers",
            "ep_combine_backward_peers", "ep_dispatch_backward_peers", "ep_ipc_export", "ep_ipc_open",
            "ep_ipc_close")

EP_MAX_PEERS = 64


class ep_shape_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "H", "k", "E", "R", "use_fp8", "num_sms",
                                              "max_tokens_per_rank")]


class ep_handle_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in HANDLE_FIELDS]


class ep_peer_rows_t(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_void_p * EP_MAX_PEERS)]


class ep_ipc_buffer_t(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64), ("bytes", ctypes.c_uint64)]


class EPError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {status_string(status)}"
        if status == EP_ERR_CUDA:
            msg += f" ({_lib().ep_last_cuda_error().decode()})"
        super().__init__(msg)
        self.status = status


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m combine_ep_get_histogram_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64)
        shp, hp = ctypes.POINTER(ep_shape_t), ctypes.POINTER(ep_handle_t)
        pp = ctypes.POINTER(ep_peer_rows_t)
        sig = {
            "ep_handle_sizes": (ctypes.c_int, [shp, i64p]),
            "ep_workspace_size": (ctypes.c_size_t, [shp]),
            "ep_get_dispatch_layout": (ctypes.c_int, [shp, vp, hp, vp, ctypes.c_size_t, vp]),
            "ep_dispatch": (ctypes.c_int, [shp, vp, vp, hp, vp, vp, vp, vp]),
            "ep_dispatch_with_layout": (ctypes.c_int, [shp, vp, vp, vp, hp, vp, ctypes.c_size_t, vp, vp, vp, vp]),
            "ep_combine": (ctypes.c_int, [shp, vp, vp, hp, vp, vp]),
            "ep_combine_backward": (ctypes.c_int, [shp, vp, vp, vp, hp, vp, vp, vp]),
            "ep_dispatch_backward": (ctypes.c_int, [shp, vp, hp, vp, vp]),
            "ep_get_error": (ctypes.c_int, [hp, vp]),
            "ep_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "ep_last_cuda_error": (ctypes.c_char_p, []),
            "ep_get_dispatch_layout_noalloc": (ctypes.c_int, [shp, vp, hp, vp]),
            "ep_noalloc_scratch_bytes": (ctypes.c_size_t, []),
            "ep_route_group_limited": (ctypes.c_int, [shp, vp, ctypes.c_int, ctypes.c_int, vp, vp, vp]),
            "ep_dispatch_peers": (ctypes.c_int, [shp, ctypes.c_int32, vp, hp, vp, vp, pp, pp, pp, vp]),
            "ep_combine_peers": (ctypes.c_int, [shp, ctypes.c_int32, vp, hp, pp, vp, vp, vp]),
            "ep_combine_backward_peers": (ctypes.c_int, [shp, ctypes.c_int32, vp, hp, vp, pp, vp, pp, vp, vp]),
            "ep_dispatch_backward_peers": (ctypes.c_int, [shp, ctypes.c_int32, vp, hp, pp, vp, vp]),
            "ep_ipc_export": (ctypes.c_int, [vp, ctypes.POINTER(ep_ipc_buffer_t)]),
            "ep_ipc_open": (ctypes.c_int, [ctypes.POINTER(ep_ipc_buffer_t), ctypes.POINTER(vp), ctypes.POINTER(vp)]),
            "ep_ipc_close": (ctypes.c_int, [vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _LIB = L
    return _LIB


def library():
    """The loaded ctypes library (raises if it is not built)."""
    return _lib()


def status_string(status: int) -> str:
    return _lib().ep_status_string(status).decode()


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> int:
    if status != EP_OK:
        raise EPError(status, where)
    return status


def make_shape(T: int, H: int, k: int, E: int, R: int, use_fp8: bool = False, num_sms: int = 0,
               max_tokens_per_rank: int = 0) -> ep_shape_t:
    """max_tokens_per_rank = 0: dense receive layout (T*k rows); M > 0: padded
    low-latency layout (E*R*M rows, see include/ep.h)."""
    return ep_shape_t(T, H, k, E, R, int(bool(use_fp8)), num_sms, max_tokens_per_rank)


def receive_rows(shape: ep_shape_t) -> int:
    M = shape.max_tokens_per_rank
    return shape.E * shape.R * M if M > 0 else shape.T * shape.k


def handle_sizes(shape: ep_shape_t) -> dict:
    counts = (ctypes.c_int64 * 9)()
    _check(_lib().ep_handle_sizes(ctypes.byref(shape), counts), "ep_handle_sizes")
    return dict(zip(HANDLE_FIELDS, list(counts)))


def workspace_size(shape: ep_shape_t) -> int:
    return int(_lib().ep_workspace_size(ctypes.byref(shape)))


class Handle:
    """Device arrays of a dispatch handle (torch tensors) and their C view."""

    DTYPES = {"is_token_in_rank": "uint8"}

    def __init__(self, shape: ep_shape_t, device):
        import torch
        self.shape = shape
        self.tensors = {}
        for name, n in handle_sizes(shape).items():
            dt = torch.uint8 if name == "is_token_in_rank" else torch.int32
            # zero-filled: error_word must start at 0
            self.tensors[name] = torch.zeros(max(n, 1), dtype=dt, device=device)
        self.c = ep_handle_t(*(t.data_ptr() for t in self.tensors.values()))

    def __getattr__(self, name):
        t = self.__dict__.get("tensors")
        if t is not None and name in t:
            return t[name]
        raise AttributeError(name)


def workspace(shape: ep_shape_t, device):
    import torch
    return torch.empty(max(workspace_size(shape), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------ entry points

def ep_get_dispatch_layout(shape: ep_shape_t, topk_idx, handle: Handle, ws, stream=None, check=True) -> int:
    nbytes = ws.numel() if hasattr(ws, "numel") else workspace_size(shape)
    st = _lib().ep_get_dispatch_layout(ctypes.byref(shape), _ptr(topk_idx), ctypes.byref(handle.c),
                                       _ptr(ws), nbytes, _stream(stream))
    return _check(st, "ep_get_dispatch_layout") if check else st


def ep_get_dispatch_layout_noalloc(shape: ep_shape_t, topk_idx, handle: Handle, stream=None,
                                   check=True) -> int:
    """The layout with the library's fixed scratch array instead of a caller
    workspace, for callers that cannot allocate device memory (see ep.h)."""
    st = _lib().ep_get_dispatch_layout_noalloc(ctypes.byref(shape), _ptr(topk_idx), ctypes.byref(handle.c),
                                               _stream(stream))
    return _check(st, "ep_get_dispatch_layout_noalloc") if check else st


def ep_dispatch(shape: ep_shape_t, x, topk_weights, handle: Handle, recv_x, recv_scale=None,
                recv_weight=None, stream=None, check=True) -> int:
    st = _lib().ep_dispatch(ctypes.byref(shape), _ptr(x), _ptr(topk_weights), ctypes.byref(handle.c),
                            _ptr(recv_x), _ptr(recv_scale), _ptr(recv_weight), _stream(stream))
    return _check(st, "ep_dispatch") if check else st


def ep_dispatch_with_layout(shape: ep_shape_t, topk_idx, x, topk_weights, handle: Handle, ws, recv_x,
                            recv_scale=None, recv_weight=None, stream=None, check=True) -> int:
    """ep_get_dispatch_layout and ep_dispatch in one call (see ep.h)."""
    nbytes = ws.numel() if hasattr(ws, "numel") else workspace_size(shape)
    st = _lib().ep_dispatch_with_layout(ctypes.byref(shape), _ptr(topk_idx), _ptr(x), _ptr(topk_weights),
                                        ctypes.byref(handle.c), _ptr(ws), nbytes, _ptr(recv_x), _ptr(recv_scale),
                                        _ptr(recv_weight), _stream(stream))
    return _check(st, "ep_dispatch_with_layout") if check else st


def ep_combine(shape: ep_shape_t, y, topk_weights, handle: Handle, out, stream=None, check=True) -> int:
    st = _lib().ep_combine(ctypes.byref(shape), _ptr(y), _ptr(topk_weights), ctypes.byref(handle.c),
                           _ptr(out), _stream(stream))
    return _check(st, "ep_combine") if check else st


def ep_combine_backward(shape: ep_shape_t, grad_out, y, topk_weights, handle: Handle, grad_y, grad_w,
                        stream=None, check=True) -> int:
    st = _lib().ep_combine_backward(ctypes.byref(shape), _ptr(grad_out), _ptr(y), _ptr(topk_weights),
                                    ctypes.byref(handle.c), _ptr(grad_y), _ptr(grad_w), _stream(stream))
    return _check(st, "ep_combine_backward") if check else st


def ep_dispatch_backward(shape: ep_shape_t, grad_recv, handle: Handle, grad_x, stream=None, check=True) -> int:
    st = _lib().ep_dispatch_backward(ctypes.byref(shape), _ptr(grad_recv), ctypes.byref(handle.c),
                                     _ptr(grad_x), _stream(stream))
    return _check(st, "ep_dispatch_backward") if check else st


def ep_route_group_limited(shape: ep_shape_t, scores, n_groups: int, topk_groups: int, topk_idx, topk_weights,
                           stream=None, check=True) -> int:
    st = _lib().ep_route_group_limited(ctypes.byref(shape), _ptr(scores), n_groups, topk_groups, _ptr(topk_idx),
                                       _ptr(topk_weights), _stream(stream))
    return _check(st, "ep_route_group_limited") if check else st


def ep_get_error(handle: Handle, stream=None) -> int:
    """Synchronises the stream; returns EP_OK or EP_ERR_BAD_INDEX (and clears it)."""
    return _lib().ep_get_error(ctypes.byref(handle.c), _stream(stream))


# ---------------------------------------------------- multi-GPU (one rank per GPU)

def peer_rows(buffers) -> ep_peer_rows_t | None:
    """Peer table for the *_peers calls: buffers[o] is owner rank o's buffer
    (a tensor or a raw device pointer, possibly another GPU's memory), or
    None for no table."""
    if buffers is None:
        return None
    if len(buffers) > EP_MAX_PEERS:
        raise ValueError(f"at most {EP_MAX_PEERS} ranks")
    t = ep_peer_rows_t()
    for o, b in enumerate(buffers):
        t.rows[o] = _ptr(b)
    return t


def _byref(t):
    return None if t is None else ctypes.byref(t)


def ep_dispatch_peers(shape: ep_shape_t, rank: int, topk_idx, handle: Handle, x, topk_weights, recv_x,
                      recv_scale=None, recv_weight=None, stream=None, check=True) -> int:
    """This rank's tokens into their owners' receive buffers (recv_*: one
    buffer per owner rank)."""
    st = _lib().ep_dispatch_peers(ctypes.byref(shape), rank, _ptr(topk_idx), ctypes.byref(handle.c), _ptr(x),
                                  _ptr(topk_weights), _byref(peer_rows(recv_x)), _byref(peer_rows(recv_scale)),
                                  _byref(peer_rows(recv_weight)), _stream(stream))
    return _check(st, "ep_dispatch_peers") if check else st


def ep_combine_peers(shape: ep_shape_t, rank: int, topk_idx, handle: Handle, y, topk_weights, out, stream=None,
                     check=True) -> int:
    """This rank's tokens, combined from the owners' expert outputs (y: one buffer per owner rank)."""
    st = _lib().ep_combine_peers(ctypes.byref(shape), rank, _ptr(topk_idx), ctypes.byref(handle.c),
                                 _byref(peer_rows(y)), _ptr(topk_weights), _ptr(out), _stream(stream))
    return _check(st, "ep_combine_peers") if check else st


def ep_combine_backward_peers(shape: ep_shape_t, rank: int, topk_idx, handle: Handle, grad_out, y, topk_weights,
                              grad_y, grad_w, stream=None, check=True) -> int:
    st = _lib().ep_combine_backward_peers(ctypes.byref(shape), rank, _ptr(topk_idx), ctypes.byref(handle.c),
                                          _ptr(grad_out), _byref(peer_rows(y)), _ptr(topk_weights),
                                          _byref(peer_rows(grad_y)), _ptr(grad_w), _stream(stream))
    return _check(st, "ep_combine_backward_peers") if check else st


def ep_dispatch_backward_peers(shape: ep_shape_t, rank: int, topk_idx, handle: Handle, grad_recv, grad_x,
                               stream=None, check=True) -> int:
    st = _lib().ep_dispatch_backward_peers(ctypes.byref(shape), rank, _ptr(topk_idx), ctypes.byref(handle.c),
                                           _byref(peer_rows(grad_recv)), _ptr(grad_x), _stream(stream))
    return _check(st, "ep_dispatch_backward_peers") if check else st


# ------------------------------------------- peer buffers between processes (CUDA IPC)

def ep_ipc_export(buf) -> bytes:
    """The record (ep_ipc_buffer_t, 80 bytes) another process opens to reach
    this device buffer (a tensor or a raw pointer inside a cudaMalloc
    allocation)."""
    rec = ep_ipc_buffer_t()
    _check(_lib().ep_ipc_export(_ptr(buf), ctypes.byref(rec)), "ep_ipc_export")
    return bytes(rec)


def ep_ipc_open(record: bytes) -> tuple[int, int]:
    """Maps another process's exported buffer: (mapped_base for
    ep_ipc_close, the buffer's device address)."""
    rec = ep_ipc_buffer_t.from_buffer_copy(record)
    base, ptr = ctypes.c_void_p(), ctypes.c_void_p()
    _check(_lib().ep_ipc_open(ctypes.byref(rec), ctypes.byref(base), ctypes.byref(ptr)), "ep_ipc_open")
    return int(base.value), int(ptr.value)


def ep_ipc_close(mapped_base: int) -> int:
    return _check(_lib().ep_ipc_close(mapped_base), "ep_ipc_close")


def ipc_record_bytes(record: bytes) -> int:
    """Bytes from the exported buffer's start to the end of its allocation."""
    return int(ep_ipc_buffer_t.from_buffer_copy(record).bytes)

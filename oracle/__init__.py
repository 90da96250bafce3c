"""CPU oracle for MoE expert-parallel dispatch / combine (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this package.  It loads the plain C
oracle (``ep_oracle.c``) and shares no code with the CUDA library: it imports
nothing from ``combine_ep_get_histogram_b200``.

bf16 tensors travel as uint16 numpy arrays of their bit patterns, e4m3 as
uint8 codes.  See ``ep_oracle.c`` for the definitions each function follows
and the readings taken where the pages are silent.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

OK, BAD_INDEX, INVALID, CAPACITY = 0, 1, 2, 4

_lib = None


def lib():
    global _lib
    if _lib is None:
        # EP_ORACLE_LIB names another build of ep_oracle.c; the mutation tests
        # use it to check that the pins reject a deliberately wrong oracle.
        path = os.environ.get("EP_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        L.epo_e4m3_value.restype = ctypes.c_double
        L.epo_e4m3_value.argtypes = [ctypes.c_uint8]
        L.epo_e4m3_encode.restype = ctypes.c_uint8
        L.epo_e4m3_encode.argtypes = [ctypes.c_float]
        L.epo_bf16_from_f32.restype = ctypes.c_uint16
        L.epo_bf16_from_f32.argtypes = [ctypes.c_float]
        for name in ("epo_e4m3_encode_array", "epo_e4m3_value_array", "epo_bf16_from_f32_array"):
            f = getattr(L, name)
            f.restype = None
            f.argtypes = [p, i64, p]
        L.epo_layout.restype = ctypes.c_int
        L.epo_layout.argtypes = [i64, i64, i64, i64] + [p] * 9
        L.epo_layout_padded.restype = ctypes.c_int
        L.epo_layout_padded.argtypes = [i64, i64, i64, i64, i64] + [p] * 9
        L.epo_route_group_limited.restype = ctypes.c_int
        L.epo_route_group_limited.argtypes = [i64, i64, i64, i64, i64, p, p, p]
        L.epo_dispatch_bf16.restype = None
        L.epo_dispatch_bf16.argtypes = [i64, i64, i64] + [p] * 5
        L.epo_dispatch_fp8.restype = None
        L.epo_dispatch_fp8.argtypes = [i64, i64, i64] + [p] * 6
        L.epo_combine.restype = None
        L.epo_combine.argtypes = [i64, i64, i64] + [p] * 4
        L.epo_combine_backward.restype = None
        L.epo_combine_backward.argtypes = [i64, i64, i64] + [p] * 6
        L.epo_dispatch_backward.restype = None
        L.epo_dispatch_backward.argtypes = [i64, i64, i64] + [p] * 3
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ formats

def e4m3_encode(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().epo_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_value(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    lib().epo_e4m3_value_array(_ptr(c), c.size, _ptr(out))
    return out


def bf16_from_f32(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().epo_bf16_from_f32_array(_ptr(v), v.size, _ptr(out))
    return out


def f32_from_bf16(b) -> np.ndarray:
    return (_c(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------- layout

def layout(topk_idx: np.ndarray, E: int, R: int) -> dict:
    """Routing layout of topk_idx [T,k] int64 over E experts and R virtual ranks.

    Returns the arrays of the handle plus ``status`` (OK or BAD_INDEX)."""
    idx = _c(topk_idx, np.int64)
    T, k = idx.shape
    d = {
        "num_tokens_per_expert": np.zeros(E, np.int32),
        "expert_offset": np.zeros(E + 1, np.int32),
        "num_tokens_per_rank": np.zeros(R, np.int32),
        "count_src_rank_expert": np.zeros(R * E, np.int32),
        "src_rank_expert_offset": np.zeros(R * E, np.int32),
        "is_token_in_rank": np.zeros(T * R, np.uint8),
        "slot_of_pair": np.zeros(T * k, np.int32),
        "src_of_slot": np.zeros(T * k, np.int32),
    }
    st = lib().epo_layout(T, k, E, R, _ptr(idx),
                          *(_ptr(d[n]) for n in ("num_tokens_per_expert", "expert_offset",
                                                 "num_tokens_per_rank", "count_src_rank_expert",
                                                 "src_rank_expert_offset", "is_token_in_rank",
                                                 "slot_of_pair", "src_of_slot")))
    if st == INVALID:
        raise ValueError("oracle layout: invalid shape")
    d["status"] = st
    return d


def layout_padded(topk_idx: np.ndarray, E: int, R: int, M: int) -> dict:
    """Padded (low-latency) layout: receive rows [E][R][M]; returns the handle
    arrays ("src_of_slot" has E*R*M entries) plus ``status`` (bit flags
    BAD_INDEX | CAPACITY, or OK)."""
    idx = _c(topk_idx, np.int64)
    T, k = idx.shape
    d = {
        "num_tokens_per_expert": np.zeros(E, np.int32),
        "expert_offset": np.zeros(E + 1, np.int32),
        "num_tokens_per_rank": np.zeros(R, np.int32),
        "count_src_rank_expert": np.zeros(R * E, np.int32),
        "src_rank_expert_offset": np.zeros(R * E, np.int32),
        "is_token_in_rank": np.zeros(T * R, np.uint8),
        "slot_of_pair": np.zeros(T * k, np.int32),
        "src_of_slot": np.zeros(E * R * M, np.int32),
    }
    st = lib().epo_layout_padded(T, k, E, R, M, _ptr(idx),
                                 *(_ptr(d[n]) for n in ("num_tokens_per_expert", "expert_offset",
                                                        "num_tokens_per_rank", "count_src_rank_expert",
                                                        "src_rank_expert_offset", "is_token_in_rank",
                                                        "slot_of_pair", "src_of_slot")))
    if st == INVALID:
        raise ValueError("oracle padded layout: invalid shape")
    d["status"] = st
    return d


def route_group_limited(scores: np.ndarray, k: int, n_groups: int, topk_groups: int):
    """scores [T,E] float32 -> (topk_idx [T,k] int64, topk_weights [T,k] float32)."""
    sc = _c(scores, np.float32)
    T, E = sc.shape
    idx = np.zeros((T, k), np.int64)
    w = np.zeros((T, k), np.float32)
    if lib().epo_route_group_limited(T, E, k, n_groups, topk_groups, _ptr(sc), _ptr(idx), _ptr(w)) == INVALID:
        raise ValueError("oracle routing: invalid arguments")
    return idx, w


# ------------------------------------------------------------ data movement

def dispatch(x: np.ndarray, topk_weights: np.ndarray, slot_of_pair: np.ndarray,
             use_fp8: bool, P: int | None = None, recv=None):
    """x [T,H] bf16 bits; slot_of_pair [T*k]; returns (recv_x, recv_scale or None,
    recv_weight).  Rows the layout gives no pair stay zero.  ``recv`` may pass
    preallocated (recv_x, recv_scale, recv_weight) to fill."""
    x = _c(x, np.uint16)
    T, H = x.shape
    w = _c(topk_weights, np.float32).reshape(T, -1)
    k = w.shape[1]
    slots = _c(slot_of_pair, np.int32).reshape(-1)
    assert slots.size == T * k
    P = T * k if P is None else P
    if use_fp8:
        assert H % 128 == 0
        if recv is None:
            recv = (np.zeros((P, H), np.uint8), np.zeros((P, H // 128), np.float32),
                    np.zeros(P, np.float32))
        rx, rs, rw = recv
        lib().epo_dispatch_fp8(T, H, k, _ptr(x), _ptr(w), _ptr(slots), _ptr(rx), _ptr(rs), _ptr(rw))
        return rx, rs, rw
    if recv is None:
        recv = (np.zeros((P, H), np.uint16), None, np.zeros(P, np.float32))
    rx, _, rw = recv
    lib().epo_dispatch_bf16(T, H, k, _ptr(x), _ptr(w), _ptr(slots), _ptr(rx), _ptr(rw))
    return rx, None, rw


def combine(y: np.ndarray, topk_weights: np.ndarray, slot_of_pair: np.ndarray) -> np.ndarray:
    """y [P,H] bf16 bits; topk_weights [T,k]; returns out [T,H] bf16 bits."""
    y = _c(y, np.uint16)
    H = y.shape[1]
    w = _c(topk_weights, np.float32)
    T, k = w.shape
    slots = _c(slot_of_pair, np.int32).reshape(-1)
    assert slots.size == T * k
    out = np.zeros((T, H), np.uint16)
    lib().epo_combine(T, H, k, _ptr(y), _ptr(w), _ptr(slots), _ptr(out))
    return out


def combine_backward(grad_out: np.ndarray, y: np.ndarray, topk_weights: np.ndarray,
                     slot_of_pair: np.ndarray, P: int | None = None, grad_y=None):
    """Returns (grad_y [P,H] bf16 bits, grad_w [T,k] float32)."""
    g = _c(grad_out, np.uint16)
    y = _c(y, np.uint16)
    T, H = g.shape
    w = _c(topk_weights, np.float32).reshape(T, -1)
    k = w.shape[1]
    slots = _c(slot_of_pair, np.int32).reshape(-1)
    P = T * k if P is None else P
    gy = np.zeros((P, H), np.uint16) if grad_y is None else grad_y
    gw = np.zeros((T, k), np.float32)
    lib().epo_combine_backward(T, H, k, _ptr(g), _ptr(y), _ptr(w), _ptr(slots), _ptr(gy), _ptr(gw))
    return gy, gw


def dispatch_backward(grad_recv: np.ndarray, slot_of_pair: np.ndarray, T: int, k: int) -> np.ndarray:
    """grad_recv [P,H] bf16 bits; returns grad_x [T,H] bf16 bits."""
    gr = _c(grad_recv, np.uint16)
    H = gr.shape[1]
    slots = _c(slot_of_pair, np.int32).reshape(-1)
    assert slots.size == T * k
    gx = np.zeros((T, H), np.uint16)
    lib().epo_dispatch_backward(T, H, k, _ptr(gr), _ptr(slots), _ptr(gx))
    return gx

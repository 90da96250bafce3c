"""Helpers for the GPU parity tests: run the CUDA path through the C ABI on
numpy inputs, and compare with the CPU oracle."""

from __future__ import annotations

import numpy as np
import torch

import combine_ep_get_histogram_b200 as ep

LAYOUT_FIELDS = ("num_tokens_per_expert", "expert_offset", "num_tokens_per_rank",
                 "count_src_rank_expert", "src_rank_expert_offset", "is_token_in_rank",
                 "slot_of_pair", "src_of_slot")


def to_dev(a: np.ndarray, device) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


class GpuPath:
    """One workload on the GPU: the handle, the layout and the buffers."""

    def __init__(self, w, topk_idx: np.ndarray, topk_weights: np.ndarray, device,
                 use_fp8: bool | None = None, num_sms: int = 0, max_tokens_per_rank: int = 0):
        self.w = w
        self.device = device
        self.use_fp8 = w.use_fp8 if use_fp8 is None else use_fp8
        self.shape = ep.make_shape(w.T, w.H, w.k, w.E, w.R, self.use_fp8, num_sms, max_tokens_per_rank)
        self.rows = ep.ep.receive_rows(self.shape)
        self.handle = ep.Handle(self.shape, device)
        self.ws = ep.workspace(self.shape, device)
        self.idx = to_dev(topk_idx, device)
        self.wts = to_dev(topk_weights.astype(np.float32), device)

    def layout(self):
        ep.ep_get_dispatch_layout(self.shape, self.idx, self.handle, self.ws)
        return self

    def layout_host(self) -> dict:
        torch.cuda.synchronize()
        return {n: self.handle.tensors[n].cpu().numpy()[: self._count(n)] for n in LAYOUT_FIELDS}

    def _count(self, n):
        return ep.handle_sizes(self.shape)[n]

    def dispatch(self, x_dev, fill=0):
        w = self.w
        P = self.rows
        if self.use_fp8:
            recv_x = torch.full((max(P, 1), w.H), fill, dtype=torch.uint8, device=self.device)
            recv_scale = torch.full((max(P, 1), w.H // 128), float(fill), dtype=torch.float32,
                                    device=self.device)
        else:
            recv_x = torch.full((max(P, 1), w.H), fill, dtype=torch.int16, device=self.device)
            recv_scale = None
        recv_weight = torch.full((max(P, 1),), float(fill), dtype=torch.float32, device=self.device)
        ep.ep_dispatch(self.shape, x_dev, self.wts, self.handle, recv_x, recv_scale, recv_weight)
        return recv_x, recv_scale, recv_weight

    def combine(self, y_dev):
        out = torch.empty((max(self.w.T, 1), self.w.H), dtype=torch.int16, device=self.device)
        ep.ep_combine(self.shape, y_dev, self.wts, self.handle, out)
        return out

    def combine_backward(self, g_dev, y_dev):
        w = self.w
        grad_y = torch.zeros((max(self.rows, 1), w.H), dtype=torch.int16, device=self.device)
        grad_w = torch.full((max(w.T, 1), w.k), -7.0, dtype=torch.float32, device=self.device)
        ep.ep_combine_backward(self.shape, g_dev, y_dev, self.wts, self.handle, grad_y, grad_w)
        return grad_y, grad_w

    def dispatch_backward(self, grad_recv_dev):
        grad_x = torch.empty((max(self.w.T, 1), self.w.H), dtype=torch.int16, device=self.device)
        ep.ep_dispatch_backward(self.shape, grad_recv_dev, self.handle, grad_x)
        return grad_x


def assert_layout_equal(got: dict, ref: dict):
    for n in LAYOUT_FIELDS:
        a = np.asarray(got[n]).astype(np.int64)
        b = np.asarray(ref[n]).astype(np.int64)
        assert a.shape == b.shape, n
        if not np.array_equal(a, b):
            bad = np.nonzero(a != b)[0]
            raise AssertionError(f"{n}: {bad.size} mismatches, first at {bad[:5]}: "
                                 f"gpu {a[bad[:5]]} oracle {b[bad[:5]]}")


def assert_bits_equal(name, got: np.ndarray, ref: np.ndarray):
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    if not np.array_equal(got, ref):
        bad = np.argwhere(got != ref)
        raise AssertionError(f"{name}: {len(bad)} of {got.size} differ, first {bad[:5].tolist()}: "
                             f"gpu {got[tuple(bad[:5].T)]} oracle {ref[tuple(bad[:5].T)]}")


def bf16_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place (ordered-integer metric)."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, 0x8000 - (x & 0x7FFF), 0x8000 + x)
    return np.abs(ordered(a) - ordered(b))


def grad_w_close(got: np.ndarray, ref: np.ndarray, rel=1e-2):
    """|got - ref| <= rel * |ref|, or <= rel * rms(ref) where ref is near 0."""
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2))) if ref.size else 0.0
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    ok = (err <= rel * np.abs(ref)) | (err <= rel * rms)
    return bool(np.all(ok)), float(np.max(err / np.maximum(np.abs(ref), rms)) if ref.size else 0.0)


def oracle_threads() -> int:
    """Host threads for the chunked oracle comparisons (the oracle's C calls
    release the GIL, so chunks run in parallel)."""
    import os
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(32, n))


def compare_in_chunks(T: int, chunk: int, fetch, check, threads: int | None = None):
    """Every token in [0, T) in chunks of `chunk`: fetch(t0, t1) reads the GPU
    outputs of the chunk on the calling thread, check(t0, t1, fetched) runs the
    oracle on the chunk and compares, on a thread pool.  At most two chunks per
    thread are held at once, so host memory stays bounded at any T."""
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or oracle_threads()
    with ThreadPoolExecutor(threads) as ex:
        pending = []
        for t0 in range(0, T, chunk):
            t1 = min(T, t0 + chunk)
            pending.append(ex.submit(check, t0, t1, fetch(t0, t1)))
            if len(pending) >= 2 * threads:
                pending.pop(0).result()
        for f in pending:
            f.result()


class StepBuffers:
    """Every buffer of one pass of the whole path (layout, dispatch, combine,
    combine backward, dispatch backward) for one shape, run on the current
    stream; inputs are loaded from numpy draws."""

    def __init__(self, w, device, max_tokens_per_rank=0, num_sms=0):
        self.w = w
        self.shape = ep.make_shape(w.T, w.H, w.k, w.E, w.R, w.use_fp8, num_sms, max_tokens_per_rank)
        P = ep.ep.receive_rows(self.shape)
        self.h = ep.Handle(self.shape, device)
        self.ws = ep.workspace(self.shape, device)
        self.idx = torch.empty((w.T, w.k), dtype=torch.int64, device=device)
        self.wts = torch.empty((w.T, w.k), dtype=torch.float32, device=device)
        self.x = torch.empty((w.T, w.H), dtype=torch.int16, device=device)
        self.y = torch.empty((P, w.H), dtype=torch.int16, device=device)
        self.g = torch.empty((w.T, w.H), dtype=torch.int16, device=device)
        self.rx = torch.empty((P, w.H), dtype=torch.uint8 if w.use_fp8 else torch.int16, device=device)
        self.rs = torch.empty((P, w.G), dtype=torch.float32, device=device) if w.use_fp8 else None
        self.rw = torch.empty(P, dtype=torch.float32, device=device)
        self.out = torch.empty((w.T, w.H), dtype=torch.int16, device=device)
        self.gy = torch.empty((P, w.H), dtype=torch.int16, device=device)
        self.gw = torch.empty((w.T, w.k), dtype=torch.float32, device=device)
        self.gx = torch.empty((w.T, w.H), dtype=torch.int16, device=device)

    def load(self, d):
        self.idx.copy_(torch.from_numpy(d["topk_idx"]))
        self.wts.copy_(torch.from_numpy(d["topk_weights"]))
        for n in ("x", "y", "g"):
            getattr(self, n).copy_(to_dev(d[n], "cpu"))

    def run(self):
        ep.ep_get_dispatch_layout(self.shape, self.idx, self.h, self.ws)
        ep.ep_dispatch(self.shape, self.x, self.wts, self.h, self.rx, self.rs, self.rw)
        ep.ep_combine(self.shape, self.y, self.wts, self.h, self.out)
        ep.ep_combine_backward(self.shape, self.g, self.y, self.wts, self.h, self.gy, self.gw)
        ep.ep_dispatch_backward(self.shape, self.gy, self.h, self.gx)

    def outputs(self):
        """Handle arrays, and the receive rows that hold a pair (padded
        layouts leave the other rows unwritten)."""
        torch.cuda.synchronize()
        if self.shape.max_tokens_per_rank:
            rows = torch.nonzero(self.h.src_of_slot >= 0).squeeze(1)
        else:
            rows = torch.arange(int(self.h.expert_offset[-1].item()), device=self.rx.device)
        res = [self.h.tensors[f].clone() for f in ("slot_of_pair", "src_of_slot", "expert_offset",
                                                    "num_tokens_per_rank", "is_token_in_rank")]
        res += [self.rx[rows].clone(), self.rw[rows].clone(), self.out.clone(), self.gy[rows].clone(),
                self.gw.clone(), self.gx.clone()]
        if self.rs is not None:
            res.append(self.rs[rows].clone())
        return res

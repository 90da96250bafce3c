"""Seeded synthetic inputs for MoE expert-parallel dispatch / combine.

This module only draws inputs. It holds none of the arithmetic of the layout,
dispatch, combine or backward operations, and it imports neither the CUDA
binding nor the CPU oracle, so both can be fed from it.

The workload shapes follow the pages' own benchmark setups: 4096 tokens per
rank, hidden 7168, top-4 groups and top-8 experts, FP8 dispatch and BF16
combine for the "normal" (training / prefill) kernels, and 128 tokens per rank,
hidden 7168, top-8 for the low-latency decode kernels
("deepep-expert-parallel-communication-library" (blog.hotdry.top), section 一
两种内核设计; "DeepSeek 开源周第二弹" (czhn.yksolo.com), sections 具有 NVLink
和 RDMA 转发的普通内核 and 具有纯 RDMA 的低延迟内核).  Group-limited gating
(experts split into groups; a token first picks groups, then experts inside
them) is the routing those pages describe
("deepep-expert-parallel-communication-library", section 三 NVLink-RDMA
跨域转发).  No public dataset is used by the pages; these synthetic draws stand
in for real router traces.

Draw recipe (seed 0 unless stated):
  * stream 0, one sequential ``numpy.random.default_rng([seed, 0])``:
    routing draws, then gate logits, then the outlier channel choice;
  * stream 4: router scores [T, E], one float32 N(0, 1) draw;
  * streams 1 (x), 2 (expert outputs y) and 3 (grad_out g): row chunks of
    ``max(1, 2**22 // H)`` rows, chunk c drawn from
    ``default_rng([seed, stream, c])`` as float32 N(0, 1), multiplied by the
    stream's sigma (and per-channel outlier factor) in float32, then rounded
    to bf16 (round to nearest even).  Chunks are independent streams, so the
    values do not depend on how many threads fill them.
  * group-limited routing: the chosen groups are the first ``topk_groups``
    entries of a uniformly random permutation of the groups; the experts are
    the first k entries of a uniformly random permutation of the union of the
    chosen groups' experts.  The top-k order is that sampling order.
  * Zipf routing: popularity of the expert at position i (1-based) of a seeded
    random permutation is proportional to i**-s; k distinct experts are drawn
    by the Gumbel-top-k method, which has the same distribution as k
    successive draws renormalised over the experts not yet drawn
    (W. Kool, H. van Hoof, M. Welling, "Stochastic Beams and Where to Find
    Them", ICML 2019).  The top-k order is the draw order.
  * gate weights: softmax over the k slots of N(0, 1) logits, in float64,
    stored as float32.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = ["Workload", "CONFIGS", "routing", "normal_bf16", "make_inputs",
           "bf16_bits_to_f32", "chunk_rows"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens over all virtual ranks
    H: int            # hidden size
    k: int            # experts per token (top-k)
    E: int            # experts
    R: int            # virtual ranks
    use_fp8: bool     # FP8 dispatch payload
    routing: str      # "group" or "zipf"
    n_groups: int = 1
    topk_groups: int = 1
    zipf_s: float = 0.0
    outlier_frac: float = 0.0   # fraction of channels scaled by outlier_gain
    outlier_gain: float = 1.0
    g_sigma: float = 1.0        # std of grad_out
    seed: int = 0

    @property
    def P(self) -> int:
        return self.T * self.k

    @property
    def G(self) -> int:
        return self.H // 128

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny correctness case, decode (8 ranks x 128 tokens),
# prefill / training (8 ranks x 4096 tokens, 1 % outlier channels), a skewed
# Zipf(1.2) routing case and the backward shape.
CONFIGS = {
    "tiny": Workload("tiny", T=64, H=256, k=4, E=16, R=4, use_fp8=False,
                     routing="group", n_groups=4, topk_groups=2),
    "decode": Workload("decode", T=1024, H=7168, k=8, E=256, R=8, use_fp8=True,
                       routing="group", n_groups=8, topk_groups=4),
    "prefill": Workload("prefill", T=32768, H=7168, k=8, E=256, R=8, use_fp8=True,
                        routing="group", n_groups=8, topk_groups=4,
                        outlier_frac=0.01, outlier_gain=50.0),
    "skewed": Workload("skewed", T=16384, H=7168, k=8, E=256, R=8, use_fp8=False,
                       routing="zipf", zipf_s=1.2),
    "backward": Workload("backward", T=32768, H=4096, k=8, E=128, R=8, use_fp8=False,
                         routing="group", n_groups=8, topk_groups=4, g_sigma=1e-2),
}


def routing(w: Workload):
    """Returns (topk_idx int64 [T,k], topk_weights float32 [T,k], outlier
    channel indices int64) drawn from stream 0."""
    rng = np.random.default_rng([w.seed, 0])
    T, k, E = w.T, w.k, w.E
    if w.routing == "group":
        per_group = E // w.n_groups
        u = rng.random((T, w.n_groups))
        groups = np.argsort(u, axis=1, kind="stable")[:, : w.topk_groups]
        cand = (groups[:, :, None] * per_group + np.arange(per_group)[None, None, :])
        cand = cand.reshape(T, w.topk_groups * per_group)
        v = rng.random(cand.shape)
        pick = np.argsort(v, axis=1, kind="stable")[:, :k]
        idx = np.take_along_axis(cand, pick, axis=1)
    elif w.routing == "zipf":
        perm = rng.permutation(E)
        ranks = np.arange(1, E + 1, dtype=np.float64)
        pop = np.empty(E, dtype=np.float64)
        pop[perm] = ranks ** (-w.zipf_s)
        pop /= pop.sum()
        keys = np.log(pop)[None, :] + rng.gumbel(size=(T, E))
        idx = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    else:
        raise ValueError(f"unknown routing {w.routing!r}")
    logits = rng.standard_normal((T, k))
    logits -= logits.max(axis=1, keepdims=True)
    ex = np.exp(logits)
    weights = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    n_out = int(round(w.outlier_frac * w.H))
    outliers = (np.sort(rng.choice(w.H, size=n_out, replace=False))
                if n_out else np.zeros(0, dtype=np.int64))
    return np.ascontiguousarray(idx.astype(np.int64)), np.ascontiguousarray(weights), outliers


def chunk_rows(H: int) -> int:
    return max(1, (1 << 22) // H)


def _f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(f).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def normal_bf16(rows: int, H: int, seed: int, stream: int, sigma: float = 1.0,
                channel_gain: np.ndarray | None = None,
                threads: int | None = None) -> np.ndarray:
    """bf16 bit patterns (uint16 [rows, H]) of sigma * N(0,1) (times a
    per-channel gain), drawn in independent row chunks."""
    out = np.empty((rows, H), dtype=np.uint16)
    if rows == 0:
        return out
    cr = chunk_rows(H)
    nchunks = (rows + cr - 1) // cr
    sig = np.float32(sigma)
    gain = None if channel_gain is None else channel_gain.astype(np.float32)

    def fill(c: int) -> None:
        lo = c * cr
        hi = min(rows, lo + cr)
        buf = np.empty((hi - lo, H), dtype=np.float32)
        np.random.default_rng([seed, stream, c]).standard_normal(out=buf, dtype=np.float32)
        if sig != np.float32(1.0):
            np.multiply(buf, sig, out=buf)
        if gain is not None:
            np.multiply(buf, gain[None, :], out=buf)
        out[lo:hi] = _f32_to_bf16_bits(buf)

    nt = threads or min(32, os.cpu_count() or 1)
    if nchunks == 1 or nt == 1:
        for c in range(nchunks):
            fill(c)
    else:
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widens bf16 bit patterns to float32 (exact)."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def make_inputs(w: Workload, parts=("routing", "x")) -> dict:
    """Draws the requested parts of a workload's inputs.

    parts: any of "routing" (topk_idx, topk_weights), "x" ([T,H] tokens),
    "y" ([T*k,H] expert outputs), "g" ([T,H] grad of the combined output),
    "scores" ([T,E] float32 N(0,1) router scores, stream 4).
    """
    d: dict = {"workload": w}
    idx, wts, outliers = routing(w)
    d["outliers"] = outliers
    if "routing" in parts:
        d["topk_idx"] = idx
        d["topk_weights"] = wts
    if "x" in parts:
        gain = None
        if len(outliers):
            gain = np.ones(w.H, dtype=np.float32)
            gain[outliers] = np.float32(w.outlier_gain)
        d["x"] = normal_bf16(w.T, w.H, w.seed, 1, 1.0, gain)
    if "y" in parts:
        d["y"] = normal_bf16(w.P, w.H, w.seed, 2, 1.0)
    if "g" in parts:
        d["g"] = normal_bf16(w.T, w.H, w.seed, 3, w.g_sigma)
    if "scores" in parts:
        sc = np.empty((w.T, w.E), dtype=np.float32)
        np.random.default_rng([w.seed, 4]).standard_normal(out=sc, dtype=np.float32)
        d["scores"] = sc
    return d

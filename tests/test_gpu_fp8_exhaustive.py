"""Exhaustive FP8 quantisation parity: every pair (x, amax) of finite bf16
values with |x| <= amax goes through the dispatch kernel and is compared
byte for byte with the oracle.

Each 128-channel group holds amax in its first channel and 127 consecutive
bf16 bit patterns from [0, amax] after it; odd channels are negated.  That is
532,701,119 non-negative (x, amax) pairs (and their negatives) in about 4.2 M
groups, laid out as tokens of H = 7168 dispatched to one expert."""

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import combine_ep_get_histogram_b200 as ep
import oracle
from gpu_util import assert_bits_equal

pytestmark = pytest.mark.gpu

H = 7168
GROUPS_PER_TOKEN = H // 128


def all_pairs_tokens():
    amax = np.arange(1, 0x7F80, dtype=np.int64)           # positive finite bf16 bit patterns
    per_a = (amax + 1 + 126) // 127                        # groups needed for x in [0, amax]
    a_of_group = np.repeat(amax, per_a).astype(np.int32)
    first = np.cumsum(per_a) - per_a
    gi = (np.arange(a_of_group.size) - np.repeat(first, per_a)).astype(np.int32)
    G = a_of_group.size
    T = (G + GROUPS_PER_TOKEN - 1) // GROUPS_PER_TOKEN
    out = np.zeros((T * GROUPS_PER_TOKEN, 128), dtype=np.uint16)
    lane = np.arange(127, dtype=np.int32)[None, :]
    sign = np.where(lane % 2 == 1, 0x8000, 0).astype(np.int32)
    step = 1 << 18
    for g0 in range(0, G, step):
        g1 = min(G, g0 + step)
        a = a_of_group[g0:g1, None]
        xs = gi[g0:g1, None] * 127 + lane
        xs = np.where(xs <= a, xs, 0)
        out[g0:g1, 0] = a[:, 0]
        out[g0:g1, 1:] = (xs | sign).astype(np.uint16)
    return out.reshape(T, H), int((amax + 1).sum())


def test_fp8_quantisation_every_bf16_pair(cuda_device):
    x, npairs = all_pairs_tokens()
    assert npairs == 532_701_119
    T = x.shape[0]
    shape = ep.make_shape(T, H, 1, 1, 1, use_fp8=True)
    h = ep.Handle(shape, cuda_device)
    idx = torch.zeros((T, 1), dtype=torch.int64, device=cuda_device)
    wts = torch.ones((T, 1), dtype=torch.float32, device=cuda_device)
    ep.ep_get_dispatch_layout(shape, idx, h, ep.workspace(shape, cuda_device))
    xd = torch.from_numpy(x.view(np.int16)).to(cuda_device)
    rx = torch.empty((T, H), dtype=torch.uint8, device=cuda_device)
    rs = torch.empty((T, H // 128), dtype=torch.float32, device=cuda_device)
    ep.ep_dispatch(shape, xd, wts, h, rx, rs, None)
    got_x, got_s = rx.cpu().numpy(), rs.cpu().numpy()
    del xd, rx, rs
    torch.cuda.empty_cache()

    slots = np.arange(T, dtype=np.int32)
    ref_x = np.empty((T, H), np.uint8)
    ref_s = np.empty((T, H // 128), np.float32)
    chunk = 2048

    def run(t0):
        t1 = min(T, t0 + chunk)
        rx_, rs_, _ = oracle.dispatch(x[t0:t1], np.ones((t1 - t0, 1), np.float32),
                                      np.arange(t1 - t0, dtype=np.int32), True)
        ref_x[t0:t1] = rx_
        ref_s[t0:t1] = rs_

    with ThreadPoolExecutor(16) as ex:
        list(ex.map(run, range(0, T, chunk)))
    assert_bits_equal("e4m3 codes", got_x, ref_x)
    assert_bits_equal("scales", got_s.view(np.uint32), ref_s.view(np.uint32))
    assert slots.size == T

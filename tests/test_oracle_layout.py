"""Pins of the oracle's routing layout (per-expert / per-rank histograms,
offsets, is_token_in_rank and the stable slot assignment): brute-force
enumeration of tiny routing tables against a sort-based restatement, library
cross-checks (numpy stable argsort, torch.bincount) and invariants on the
five synthetic workloads."""

import itertools

import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_histogram_b200 import workloads as wl


def sort_based_layout(idx, E, R):
    """The layout as a sort: a pair's slot is its position after a stable sort
    of all valid pairs by expert id (the pairs are in (t, j) order before)."""
    T, k = idx.shape
    Tr, Er = T // R, E // R
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < E)
    order = np.argsort(np.where(valid, flat, E), kind="stable")
    nvalid = int(valid.sum())
    slot = np.full(T * k, -1, np.int64)
    slot[order[:nvalid]] = np.arange(nvalid)
    src = np.full(T * k, -1, np.int64)
    src[:nvalid] = order[:nvalid]
    counts = np.bincount(flat[valid], minlength=E)
    offs = np.concatenate([[0], np.cumsum(counts)])
    in_rank = np.zeros((T, R), np.uint8)
    tok = np.repeat(np.arange(T), k)
    in_rank[tok[valid], flat[valid] // Er] = 1
    # first slot of (source rank r, expert e): valid pairs with expert < e, plus
    # pairs of expert e whose token lies below rank r's first token
    sre = np.zeros((R, E), np.int64)
    cnt_sre = np.zeros((R, E), np.int64)
    np.add.at(cnt_sre, (tok[valid] // Tr, flat[valid]), 1)
    for r in range(R):
        below = valid & (tok < r * Tr)
        sre[r] = offs[:-1] + np.bincount(flat[below], minlength=E)
    return dict(slot_of_pair=slot, src_of_slot=src, num_tokens_per_expert=counts,
                expert_offset=offs, is_token_in_rank=in_rank.reshape(-1),
                num_tokens_per_rank=in_rank.sum(0), src_rank_expert_offset=sre.reshape(-1),
                count_src_rank_expert=cnt_sre.reshape(-1))


def assert_layout_equal(got, ref):
    for name, v in ref.items():
        assert np.array_equal(np.asarray(got[name], np.int64), np.asarray(v, np.int64)), name


@pytest.mark.parametrize("T,k,E,R", [(1, 1, 2, 1), (2, 2, 2, 2), (2, 2, 3, 1), (3, 2, 3, 1),
                                     (2, 3, 2, 2), (4, 1, 4, 2)])
def test_brute_force_all_tables(T, k, E, R):
    """Every routing table with entries in [-1, E) (duplicates included)."""
    n = 0
    for entries in itertools.product(range(-1, E), repeat=T * k):
        idx = np.array(entries, np.int64).reshape(T, k)
        got = oracle.layout(idx, E, R)
        assert got["status"] == oracle.OK
        assert_layout_equal(got, sort_based_layout(idx, E, R))
        n += 1
    assert n == (E + 1) ** (T * k)


def test_random_tables_against_sort_and_bincount():
    rng = np.random.default_rng(11)
    for trial in range(200):
        R = int(rng.integers(1, 5))
        Er = int(rng.integers(1, 6))
        E = R * Er
        T = R * int(rng.integers(0, 9))
        k = int(rng.integers(1, 6))
        idx = rng.integers(-1, E, size=(T, k)).astype(np.int64)
        got = oracle.layout(idx, E, R)
        assert_layout_equal(got, sort_based_layout(idx, E, R))
        flat = torch.from_numpy(idx.reshape(-1))
        ref_counts = torch.bincount(flat[flat >= 0], minlength=E).numpy()
        assert np.array_equal(got["num_tokens_per_expert"], ref_counts)


def test_bad_index_is_reported_and_masked():
    idx = np.array([[0, 5], [-2, 1], [3, -1]], np.int64)  # E = 4: 5 and -2 are bad
    got = oracle.layout(idx, 4, 1)
    assert got["status"] == oracle.BAD_INDEX
    masked = np.where((idx >= 0) & (idx < 4), idx, -1)
    assert_layout_equal(got, sort_based_layout(masked, 4, 1))
    assert list(got["slot_of_pair"]) == [0, -1, -1, 1, 2, -1]


def test_invalid_shapes_rejected():
    with pytest.raises(ValueError):
        oracle.layout(np.zeros((3, 2), np.int64), 4, 2)  # T % R != 0
    with pytest.raises(ValueError):
        oracle.layout(np.zeros((4, 2), np.int64), 6, 4)  # E % R != 0


def test_empty_input():
    got = oracle.layout(np.zeros((0, 8), np.int64), 16, 4)
    assert got["status"] == oracle.OK
    assert np.all(got["expert_offset"] == 0) and np.all(got["num_tokens_per_rank"] == 0)


@pytest.mark.parametrize("name", list(wl.CONFIGS))
def test_workload_invariants(name):
    w = wl.CONFIGS[name]
    idx, _, _ = wl.routing(w)
    got = oracle.layout(idx, w.E, w.R)
    assert got["status"] == oracle.OK
    P = w.T * w.k
    counts = got["num_tokens_per_expert"]
    assert counts.sum() == P  # every pair counted once
    slots = got["slot_of_pair"]
    assert np.array_equal(np.sort(slots), np.arange(P))  # slots are a permutation
    src = got["src_of_slot"]
    assert np.array_equal(src[slots], np.arange(P))  # inverse maps
    flat = idx.reshape(-1)
    offs = got["expert_offset"]
    assert np.all(slots >= offs[flat]) and np.all(slots < offs[flat + 1])  # contiguous blocks
    # inside each expert block the source pair index increases
    e_of_slot = flat[src]
    same = e_of_slot[1:] == e_of_slot[:-1]
    assert np.all(src[1:][same] > src[:-1][same])
    itr = got["is_token_in_rank"].reshape(w.T, w.R)
    direct = np.zeros((w.T, w.R), np.uint8)
    direct[np.repeat(np.arange(w.T), w.k), flat // (w.E // w.R)] = 1
    assert np.array_equal(itr, direct)
    assert np.array_equal(got["num_tokens_per_rank"], itr.sum(0))
    # rank partitions of the receive buffer tile [0, P)
    Er = w.E // w.R
    bounds = offs[np.arange(0, w.E + 1, Er)]
    assert bounds[0] == 0 and bounds[-1] == P and np.all(np.diff(bounds) >= 0)
    assert_layout_equal(got, sort_based_layout(idx, w.E, w.R))


# ----------------------------------------------------- padded (low-latency) layout

def sort_based_padded(idx, E, R, M):
    """Padded rows as a sort: valid pairs stably sorted by block key e*R + r
    (pairs are in (t, j) order before); a pair's position in its block is its
    sorted index minus the block's first index."""
    T, k = idx.shape
    Tr = T // R
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < E)
    tok = np.repeat(np.arange(T), k)
    key = np.where(valid, flat * R + tok // max(Tr, 1), E * R)
    order = np.argsort(key, kind="stable")
    skey = key[order]
    first = np.searchsorted(skey, skey, side="left")
    pos = np.arange(order.size) - first
    slot = np.full(T * k, -1, np.int64)
    ok = (skey < E * R) & (pos < M)
    slot[order[ok]] = skey[ok] * M + pos[ok]
    rows = np.full(E * R * M, -1, np.int64)
    rows[slot[slot >= 0]] = np.nonzero(slot >= 0)[0]
    overflow = bool(np.any((skey < E * R) & (pos >= M)))
    return slot, rows, overflow


@pytest.mark.parametrize("T,k,E,R", [(2, 2, 2, 1), (2, 2, 2, 2), (3, 2, 3, 1), (4, 1, 4, 2)])
def test_padded_brute_force_all_tables(T, k, E, R):
    Tr = T // R
    for M in (Tr, Tr + 1):
        for entries in itertools.product(range(-1, E), repeat=T * k):
            idx = np.array(entries, np.int64).reshape(T, k)
            got = oracle.layout_padded(idx, E, R, M)
            slot, rows, overflow = sort_based_padded(idx, E, R, M)
            assert np.array_equal(got["slot_of_pair"], slot)
            assert np.array_equal(got["src_of_slot"], rows)
            assert bool(got["status"] & oracle.CAPACITY) == overflow
            dense = oracle.layout(idx, E, R)
            for n in ("num_tokens_per_expert", "num_tokens_per_rank", "count_src_rank_expert",
                      "is_token_in_rank"):
                assert np.array_equal(got[n], dense[n]), n
            assert np.array_equal(got["expert_offset"], np.arange(E + 1) * R * M)


def test_padded_random_tables_and_capacity():
    rng = np.random.default_rng(21)
    for trial in range(100):
        R = int(rng.integers(1, 5))
        E = R * int(rng.integers(1, 5))
        T = R * int(rng.integers(1, 7))
        k = int(rng.integers(1, 5))
        M = T // R + int(rng.integers(0, 3))
        idx = rng.integers(-1, E, size=(T, k)).astype(np.int64)  # duplicates allowed
        got = oracle.layout_padded(idx, E, R, M)
        slot, rows, overflow = sort_based_padded(idx, E, R, M)
        assert np.array_equal(got["slot_of_pair"], slot)
        assert np.array_equal(got["src_of_slot"], rows)
        assert bool(got["status"] & oracle.CAPACITY) == overflow
    with pytest.raises(ValueError):
        oracle.layout_padded(np.zeros((8, 2), np.int64), 4, 2, 3)  # M < T/R


def test_padded_decode_workload_invariants():
    w = wl.CONFIGS["decode"]
    idx, _, _ = wl.routing(w)
    M = w.T // w.R
    got = oracle.layout_padded(idx, w.E, w.R, M)
    assert got["status"] == oracle.OK  # distinct experts per token: never over capacity
    slots = got["slot_of_pair"]
    flat = idx.reshape(-1)
    r_of_pair = np.repeat(np.arange(w.T), w.k) // M
    block = slots // M
    assert np.array_equal(block, flat * w.R + r_of_pair)  # each pair in its (expert, source rank) block
    assert np.array_equal(got["src_of_slot"][slots], np.arange(w.T * w.k))
    pos = slots % M
    cnt = got["count_src_rank_expert"].reshape(w.R, w.E)
    assert np.all(pos < cnt[r_of_pair, flat])  # rows packed from the block start
    # same rank-relative positions as the dense layout
    dense = oracle.layout(idx, w.E, w.R)
    rel_dense = dense["slot_of_pair"] - dense["src_rank_expert_offset"].reshape(w.R, w.E)[r_of_pair, flat]
    assert np.array_equal(pos, rel_dense)

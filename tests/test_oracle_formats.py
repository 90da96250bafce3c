"""Pins of the oracle's number formats (E4M3 and bf16) against the format
definitions, brute force and PyTorch's own casts (run, not read)."""

import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_e4m3_table():
    """Value of every E4M3 code according to PyTorch's float8_e4m3fn."""
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()


def test_e4m3_decode_matches_torch_table():
    ours = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    ref = torch_e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])


def test_e4m3_encode_roundtrips_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = torch_e4m3_table()[codes].astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_e4m3_midpoints_round_to_even_and_neighbours_round_to_nearest():
    table = torch_e4m3_table()
    pos = [c for c in range(0x7F)]  # 0x00 .. 0x7E, increasing values
    for c in pos[:-1]:
        lo, hi = table[c], table[c + 1]
        mid = np.float32((lo + hi) / 2)  # <= 5 significant bits: exact in float32
        assert float(mid) == (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode([mid])[0] == even, hex(c)
        below = np.nextafter(mid, np.float32(-np.inf), dtype=np.float32)
        above = np.nextafter(mid, np.float32(np.inf), dtype=np.float32)
        assert oracle.e4m3_encode([below])[0] == c
        assert oracle.e4m3_encode([above])[0] == c + 1
        # negative side mirrors with the sign bit
        assert oracle.e4m3_encode([-mid])[0] == (even | 0x80)


def test_e4m3_saturates():
    big = np.array([448.0, 448.5, 463.99, 464.0, 480.0, 1e6, 3e38], dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)


def test_e4m3_golden_cases():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_encode_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            v, code = line.split()[:2]
            rows.append((np.float32(float(v)), int(code, 16)))
    vals = np.array([r[0] for r in rows], dtype=np.float32)
    assert len(rows) >= 20
    assert list(oracle.e4m3_encode(vals)) == [r[1] for r in rows]


def test_e4m3_brute_force_nearest_code():
    """encode(v) is the finite code nearest to v, ties to the even code."""
    rng = np.random.default_rng(7)
    table = torch_e4m3_table()
    finite = np.array([c for c in range(256) if not np.isnan(table[c])])
    fv = table[finite]
    mags = np.exp2(rng.uniform(-12, 9, 4000))
    v = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    v = v[np.abs(v) <= 448]
    got = oracle.e4m3_encode(v)
    for x, g in zip(v.astype(np.float64), got):
        d = np.abs(fv - x)
        best = finite[d == d.min()]
        # same value can have two codes only for +-0
        if len(best) > 1:
            best = best[[np.signbit(table[b]) == np.signbit(x) for b in best]]
        if len(best) > 1:
            best = [b for b in best if (b & 1) == 0]
        assert g == best[0], (x, hex(g), [hex(b) for b in best])


def test_e4m3_matches_torch_cast_in_range():
    rng = np.random.default_rng(3)
    v = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 100,
        rng.uniform(-448, 448, 100000).astype(np.float32),
        (rng.standard_normal(100000) * 1e-3).astype(np.float32),
    ])
    v = np.clip(v, -448, 448).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_bf16_matches_torch_cast():
    rng = np.random.default_rng(5)
    parts = [
        rng.standard_normal(300000).astype(np.float32),
        (rng.standard_normal(100000) * np.exp2(rng.uniform(-140, 120, 100000))).astype(np.float32),
        # exact ties: low 16 bits = 0x8000, both parities of bit 16
        (rng.integers(0, 2**31, 20000, dtype=np.uint32) & 0xFFFF0000 | 0x8000).view(np.float32),
        # float32 subnormals and values near the bf16 overflow threshold
        (rng.integers(1, 2**23, 20000, dtype=np.uint32)).view(np.float32),
        np.array([3.3895314e38, 3.39e38, 3.4028235e38, -3.4028235e38, 0.0, -0.0], dtype=np.float32),
    ]
    v = np.concatenate(parts)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_from_f32(v), ref)


@pytest.mark.parametrize("v,bits", [(1.0, 0x3F80), (-2.0, 0xC000), (1.00390625, 0x3F80),
                                    (1.01171875, 0x3F82), (-0.0, 0x8000)])
def test_bf16_hand_cases(v, bits):
    # 1 + 2^-8 is halfway between 1.0 and 1 + 2^-7: even -> 1.0;
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: even -> 1 + 2^-6 (0x3F82)
    assert oracle.bf16_from_f32([v])[0] == bits

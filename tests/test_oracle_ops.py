"""Pins of the oracle's data-movement operations: dispatch (BF16 and FP8),
combine, combine backward and dispatch backward.

Each is checked against something other than the oracle's own code:
hand-derived worked examples (tests/golden), the E4M3 error bound, exact
arithmetic (float64 partial results checked exact with fractions, then one
float32 rounding by numpy and the bf16 rounding by PyTorch), PyTorch autograd
in float64, and special cases (k = 1, unit weights, masked pairs)."""

import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_histogram_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(b):
    return oracle.f32_from_bf16(b)


def torch_bf16_bits(v):
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def to_bf16_bits(v):
    """bf16 bit patterns of float values (PyTorch's rounding)."""
    return torch_bf16_bits(np.asarray(v, np.float32))


@pytest.fixture(scope="module")
def tiny():
    w = wl.CONFIGS["tiny"]
    d = wl.make_inputs(w, parts=("routing", "x", "y", "g"))
    d["layout"] = oracle.layout(d["topk_idx"], w.E, w.R)
    return d


# ------------------------------------------------------------------ dispatch

def test_dispatch_bf16_copies_rows(tiny):
    w = tiny["workload"]
    slots = tiny["layout"]["slot_of_pair"].reshape(w.T, w.k)
    rx, rs, rw = oracle.dispatch(tiny["x"], tiny["topk_weights"], slots, use_fp8=False)
    assert rs is None
    for t in range(w.T):
        for j in range(w.k):
            assert np.array_equal(rx[slots[t, j]], tiny["x"][t])
            assert rw[slots[t, j]] == tiny["topk_weights"][t, j]


def fp8_token(values, H=128):
    row = np.zeros(H, np.float32)
    row[: len(values)] = values
    bits = to_bf16_bits(row)
    assert np.array_equal(f32(bits), row), "test values must be exact in bf16"
    return bits


def golden_e4m3():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_encode_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                v, code = line.split()[:2]
                rows.append((float(v), int(code, 16)))
    return rows


def dispatch_one(tok_bits):
    H = tok_bits.size
    rx, rs, rw = oracle.dispatch(tok_bits.reshape(1, H), np.ones((1, 1), np.float32),
                                 np.zeros(1, np.int32), use_fp8=True)
    return rx[0], rs[0]


def test_fp8_worked_example_scale_one():
    """amax = 448 gives scale = 1 exactly, so every code is the hand-derived
    E4M3 encoding of the value itself (golden cases that are exact in bf16)."""
    cases = [(v, c) for v, c in golden_e4m3() if abs(v) <= 448 and
             float(np.float32(v)) == float(f32(to_bf16_bits([v]))[0])]
    assert len(cases) >= 15
    vals = [448.0] + [v for v, _ in cases]
    codes, scale = dispatch_one(fp8_token(vals))
    assert scale[0] == np.float32(1.0)
    assert codes[0] == 0x7E
    assert list(codes[1:len(vals)]) == [c for _, c in cases]


def test_fp8_worked_example_divides_by_scale():
    """amax = 224 gives scale = 0.5: codes encode 2x (1.0 -> 0x38, 116 -> 232 -> tie -> 0x76);
    multiplying by the scale instead would give 0.25 -> 0x30."""
    codes, scale = dispatch_one(fp8_token([224.0, 0.5, 116.0, -0.5]))
    assert scale[0] == np.float32(0.5)
    assert list(codes[:4]) == [0x7E, 0x38, 0x76, 0xB8]
    assert np.all(codes[4:128] == 0x00)


def test_fp8_zero_group_and_signs():
    row = np.zeros(256, np.float32)
    row[128] = 3.0
    bits = to_bf16_bits(row)
    bits[5] = 0x8000  # -0 in the all-zero first group
    codes, scale = dispatch_one(bits)
    assert scale[0] == np.float32(1.0)  # amax 0 -> scale 1
    assert np.all(np.delete(codes[:128], 5) == 0) and codes[5] == 0x80
    assert codes[128] == 0x7E


def test_fp8_scale_correctly_rounded_and_error_bound(tiny):
    w = tiny["workload"]
    rng = np.random.default_rng(2)
    x = tiny["x"].copy()
    # widen the dynamic range: per-group gains from 2^-30 to 2^20, plus zeros
    gains = np.exp2(rng.integers(-30, 21, size=(w.T, w.H // 128))).astype(np.float32)
    xf = f32(x).reshape(w.T, w.H // 128, 128) * gains[:, :, None]
    xf[0, 0] = 0.0
    x = to_bf16_bits(xf.reshape(w.T, w.H))
    slots = tiny["layout"]["slot_of_pair"].reshape(w.T, w.k)
    rx, rs, rw = oracle.dispatch(x, tiny["topk_weights"], slots, use_fp8=True)
    xv = f32(x).astype(np.float64).reshape(w.T, w.H // 128, 128)
    table = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    for t in range(w.T):
        for j in range(w.k):
            s = slots[t, j]
            codes = rx[s].reshape(-1, 128)
            for g in range(w.H // 128):
                amax = np.abs(xv[t, g]).max()
                scale = rs[s, g]
                if amax == 0:
                    assert scale == 1.0 and np.all((codes[g] & 0x7F) == 0)
                    continue
                # scale is amax / 448 correctly rounded to float32
                exact = Fraction(float(amax)) / 448
                err = abs(Fraction(float(scale)) - exact)
                up = np.nextafter(np.float32(scale), np.float32(np.inf))
                assert err <= (Fraction(float(up)) - Fraction(float(scale))) / 2
                # the largest element lands on +-448
                i = int(np.argmax(np.abs(xv[t, g])))
                assert codes[g][i] & 0x7F == 0x7E
                # element-wise E4M3 error bound: half an ulp (2^-4 relative for
                # normals, 2^-10 absolute below 2^-6), in units of the scale
                deq = table[codes[g]] * float(scale)
                bound = 2.0 ** -4 * np.abs(xv[t, g]) * (1 + 2.0 ** -20) + 2.0 ** -10 * float(scale)
                assert np.all(np.abs(deq - xv[t, g]) <= bound)
                assert np.all(np.signbit(table[codes[g]]) == np.signbit(xv[t, g]))


def test_fp8_roundtrip_through_combine(tiny):
    """Identity experts on dequantised FP8 payloads, gate weights summing to 1:
    the float64 combine returns x within the E4M3 error bound."""
    w = tiny["workload"]
    slots = tiny["layout"]["slot_of_pair"].reshape(w.T, w.k)
    rx, rs, _ = oracle.dispatch(tiny["x"], tiny["topk_weights"], slots, use_fp8=True)
    table = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    deq = table[rx].reshape(-1, w.H // 128, 128) * rs[:, :, None].astype(np.float64)
    deq = deq.reshape(-1, w.H)
    wt = tiny["topk_weights"].astype(np.float64)
    out = (wt[:, :, None] * deq[slots]).sum(1)
    x = f32(tiny["x"]).astype(np.float64)
    scale_max = np.repeat(rs[slots[:, 0]], 128, axis=1).astype(np.float64)
    bound = 2.0 ** -4 * np.abs(x) * 1.001 + 2.0 ** -10 * scale_max + 1e-6 * np.abs(x)
    assert np.all(np.abs(out - x) <= bound)


# ------------------------------------------------------------------- combine

def read_chain_cases():
    rows = []
    with open(os.path.join(GOLDEN, "combine_chain_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, ws, ys, out = line.split()[:4]
            wv = np.array([int(h, 16) for h in ws.split(",")], np.uint32).view(np.float32)
            yv = np.array([int(h, 16) for h in ys.split(",")], np.uint16)
            assert len(wv) == len(yv) == int(k)
            rows.append((wv, yv, int(out, 16)))
    return rows


def test_combine_golden_chains():
    rows = read_chain_cases()
    assert len(rows) >= 5
    for wv, yv, expect in rows:
        k = len(wv)
        y = yv.reshape(k, 1)  # one channel, pair j sits in slot j
        out = oracle.combine(y, wv.reshape(1, k), np.arange(k, dtype=np.int32))
        assert out[0, 0] == expect, (wv, yv, hex(out[0, 0]), hex(expect))


def exact_chain(wv, yv, slots, add_only=False):
    """fp32 chain evaluated as exact float64 steps (checked exact) with one
    numpy float32 rounding per step; bf16 rounding by PyTorch."""
    T, k = slots.shape
    H = yv.shape[1]
    acc = np.zeros((T, H), np.float32)
    for j in range(k):
        s = slots[:, j]
        ok = s >= 0
        term = f32(yv[np.where(ok, s, 0)]).astype(np.float64)
        if not add_only:
            term = term * wv[:, j].astype(np.float64)[:, None]
        exact = acc.astype(np.float64) + term
        # float64 holds the exact value when no bits were lost: check a sample
        for (a, b, c) in list(zip(acc.ravel()[:64], term.ravel()[:64], exact.ravel()[:64])):
            assert Fraction(float(a)) + Fraction(float(b)) == Fraction(float(c))
        acc = np.where(ok[:, None], exact.astype(np.float32), acc)
    return torch_bf16_bits(acc)


def test_combine_matches_exact_chain(tiny):
    w = tiny["workload"]
    slots = tiny["layout"]["slot_of_pair"].reshape(w.T, w.k)
    out = oracle.combine(tiny["y"], tiny["topk_weights"], slots)
    assert np.array_equal(out, exact_chain(tiny["topk_weights"], tiny["y"], slots))


def test_combine_k1_unit_weight_is_a_gather():
    rng = np.random.default_rng(4)
    y = to_bf16_bits(rng.standard_normal((10, 64)).astype(np.float32))
    slots = rng.permutation(10).astype(np.int32)
    out = oracle.combine(y, np.ones((10, 1), np.float32), slots)
    assert np.array_equal(out, y[slots])


def test_combine_identity_experts_return_x(tiny):
    """BF16 dispatch, identity experts, softmax weights (sum 1 up to float32
    rounding): combine returns x within one bf16 ulp."""
    w = tiny["workload"]
    slots = tiny["layout"]["slot_of_pair"].reshape(w.T, w.k)
    rx, _, _ = oracle.dispatch(tiny["x"], tiny["topk_weights"], slots, use_fp8=False)
    out = oracle.combine(rx, tiny["topk_weights"], slots)
    a = f32(out).astype(np.float64)
    x = f32(tiny["x"]).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(x), 1e-30))) - 7)
    assert np.all(np.abs(a - x) <= ulp)


def test_combine_masked_pairs_are_skipped():
    y = to_bf16_bits(np.array([[1.0, 2.0], [3.0, 4.0]], np.float32))
    wv = np.array([[0.5, 0.25], [1.0, 1.0]], np.float32)
    slots = np.array([1, -1, -1, -1], np.int32)  # token 1 has no valid pair
    out = oracle.combine(y, wv, slots)
    assert list(f32(out[0])) == [1.5, 2.0]
    assert list(out[1]) == [0, 0]


# ------------------------------------------------------------------ backward

def test_combine_backward_against_autograd(tiny):
    w = tiny["workload"]
    slots = tiny["layout"]["slot_of_pair"].reshape(w.T, w.k)
    gy, gw = oracle.combine_backward(tiny["g"], tiny["y"], tiny["topk_weights"], slots)
    # grad_y: one float32 product (PyTorch), then PyTorch's bf16 rounding
    prod = (torch.from_numpy(tiny["topk_weights"])[:, :, None] *
            torch.from_numpy(f32(tiny["g"]))[:, None, :]).numpy()
    ref_gy = torch_bf16_bits(prod)
    assert np.array_equal(gy[slots], ref_gy)
    # grad_w from float64 autograd of out = sum_j w_j * y[slot_j], loss = <out, g>
    wt = torch.tensor(tiny["topk_weights"], dtype=torch.float64, requires_grad=True)
    yy = torch.from_numpy(f32(tiny["y"]).astype(np.float64))[torch.from_numpy(slots.astype(np.int64))]
    out = (wt[:, :, None] * yy).sum(1)
    (out * torch.from_numpy(f32(tiny["g"]).astype(np.float64))).sum().backward()
    ref = wt.grad.numpy()
    assert np.allclose(gw, ref, rtol=1e-6, atol=1e-12 * np.abs(ref).max())


def test_combine_backward_power_of_two_weights_scale_exactly():
    rng = np.random.default_rng(8)
    T, k, H = 6, 3, 64
    g = to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    y = to_bf16_bits(rng.standard_normal((T * k, H)).astype(np.float32))
    wv = np.exp2(rng.integers(-3, 3, size=(T, k))).astype(np.float32)
    slots = rng.permutation(T * k).astype(np.int32)
    slots[4] = -1
    gy, gw = oracle.combine_backward(g, y, wv, slots)
    for t in range(T):
        for j in range(k):
            s = slots[t * k + j]
            if s < 0:
                assert gw[t, j] == 0.0
                continue
            assert np.array_equal(f32(gy[s]), f32(g[t]) * wv[t, j])  # exact scaling


def test_dispatch_backward_exact_and_adjoint(tiny):
    w = tiny["workload"]
    slots = tiny["layout"]["slot_of_pair"].reshape(w.T, w.k)
    rng = np.random.default_rng(9)
    # small integers: every partial sum is exact
    gr_int = rng.integers(-50, 50, size=(w.P, w.H))
    gr = to_bf16_bits(gr_int.astype(np.float32))
    gx = oracle.dispatch_backward(gr, slots, w.T, w.k)
    assert np.array_equal(f32(gx), gr_int[slots].sum(1).astype(np.float32))
    # random values: exact chain, and the adjoint of the BF16 dispatch gather
    gx = oracle.dispatch_backward(tiny["y"], slots, w.T, w.k)
    assert np.array_equal(gx, exact_chain(np.ones((w.T, w.k), np.float32), tiny["y"], slots,
                                          add_only=True))
    xv = torch.zeros((w.T, w.H), dtype=torch.float64, requires_grad=True)
    token_of_slot = torch.from_numpy((tiny["layout"]["src_of_slot"] // w.k).astype(np.int64))
    recv = xv[token_of_slot]
    (recv * torch.from_numpy(f32(tiny["y"]).astype(np.float64))).sum().backward()
    ref = xv.grad.numpy()
    got = f32(gx).astype(np.float64)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)

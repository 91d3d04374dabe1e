"""Pins of the oracle's fp8 metadata (an optional, lower-precision copy of the
page metadata that the scoring can read instead of the exact bf16 min/max).

What fixes it, independently of the oracle's own code:
  * the E4M3 grid built from its definition (k * 2^-9 for k < 8, then
    m * 2^(E-3) for m in 8..15 and E in -6..8, up to 448), and PyTorch's own
    float8_e4m3fn reading of every byte pattern (a library routine);
  * outward rounding as brute force over that grid;
  * the row exponent by its defining inequalities;
  * the Quest bound: fp8 score >= exact score >= max over tokens of q.k, with
    equality when every key already lies on the (scaled) grid.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decoding_b200 import workloads as wl
from test_oracle import PS, case_np, f64, token_keys


def grid():
    """Every non-negative finite E4M3 value, from the format's definition."""
    vals = {k * 2.0 ** -9 for k in range(8)}
    for E in range(-6, 9):
        for m in range(8, 16):
            v = m * 2.0 ** (E - 3)
            if v <= 448.0:
                vals.add(v)
    return sorted(vals)


GRID = grid()
FULL = sorted({-v for v in GRID} | set(GRID))


def test_grid_matches_torch_float8():
    """Our decoding of every byte equals PyTorch's float8_e4m3fn reading."""
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    for x in range(256):
        if x in (0x7F, 0xFF):                   # NaN patterns never occur here
            assert math.isnan(ref[x])
            continue
        assert oracle.fp8_decode(x) == ref[x], hex(x)
    assert len(GRID) == 127 and GRID[-1] == 448.0   # 0, 7 subnormals, 119 normals


def test_encode_decode_round_trip_on_the_grid():
    seen = set()
    for v in FULL:
        x = oracle.fp8_encode(v)
        assert x not in (0x7F, 0xFF)
        assert oracle.fp8_decode(x) == v
        seen.add(x)
    assert len(seen) == len(FULL)               # one pattern per value; zero is 0x00
    assert oracle.fp8_encode(0.0) == 0 and oracle.fp8_encode(-0.0) == 0


def test_outward_rounding_is_the_nearest_grid_value_outside():
    rng = np.random.default_rng(7)
    ys = list(rng.uniform(-448, 448, 3000)) + list(rng.uniform(-0.05, 0.05, 2000))
    ys += FULL + [(a + b) / 2 for a, b in zip(FULL, FULL[1:])]
    ys += [2.0 ** -12, -(2.0 ** -12), 1e-300, -1e-300]
    arr = np.array(FULL)
    for y in ys:
        lo = oracle.fp8_round(y, up=False)
        hi = oracle.fp8_round(y, up=True)
        assert lo == arr[arr <= y].max(), y
        assert hi == arr[arr >= y].min(), y


@pytest.mark.parametrize("a", [0.0, 1.0, 448.0, 448.0000001, 449.0, 2.0 ** -20, 3.5, 1e30,
                               224.0, 224.5, 1.75, 1.7500001, 7.0 * 2 ** 100])
def test_row_exponent_is_the_smallest_that_fits(a):
    e = oracle.fp8_row_exponent(a)
    if a == 0.0:
        assert e == 0
        return
    assert a * 2.0 ** -e <= 448.0
    assert a * 2.0 ** -(e - 1) > 448.0


def test_row_exponent_random():
    rng = np.random.default_rng(3)
    for a in np.exp(rng.uniform(-40, 40, 500)):
        e = oracle.fp8_row_exponent(float(a))
        assert a * 2.0 ** -e <= 448.0 < a * 2.0 ** -(e - 1)


def test_meta_fp8_box_contains_the_exact_box_tightly():
    d, c, a = case_np(B=2, Hq=4, Hkv=2, D=32, lens=(200, 71), seed=5)
    m = oracle.meta(d, a["k"], a["pt"], a["sl"])
    m8 = oracle.meta_fp8(d, m, a["pt"], a["sl"])
    arr = np.array(FULL)
    for b in range(d.B):
        for p in range(-(-int(a["sl"][b]) // PS)):
            phys = a["pt"][b, p]
            for g in range(d.Hkv):
                row = m8[phys, g]
                e = int(np.frombuffer(row[2 * d.D:2 * d.D + 4].tobytes(), np.int32)[0])
                assert not row[2 * d.D + 4:].any()
                mn, mx = f64(m[phys, g, 0]), f64(m[phys, g, 1])
                amax = max(np.abs(mn).max(), np.abs(mx).max())
                assert e == oracle.fp8_row_exponent(float(amax))
                lo = np.array([oracle.fp8_decode(x) for x in row[:d.D]]) * 2.0 ** e
                hi = np.array([oracle.fp8_decode(x) for x in row[d.D:2 * d.D]]) * 2.0 ** e
                assert (lo <= mn).all() and (hi >= mx).all()
                # tight: no grid value lies strictly between the rounded and exact ones
                for i in range(d.D):
                    ys, yh = mn[i] * 2.0 ** -e, mx[i] * 2.0 ** -e
                    assert not ((arr > lo[i] * 2.0 ** -e) & (arr <= ys)).any()
                    assert not ((arr < hi[i] * 2.0 ** -e) & (arr >= yh)).any()


def test_fp8_scores_bound_the_exact_scores_and_the_logits():
    d, c, a = case_np(B=2, Hq=8, Hkv=2, D=32, lens=(300, 150), seed=9)
    m = oracle.meta(d, a["k"], a["pt"], a["sl"])
    m8 = oracle.meta_fp8(d, m, a["pt"], a["sl"])
    s8 = oracle.scores_fp8(d, a["q"], m8, a["pt"], a["sl"], 16, 32)
    s = oracle.scores(d, a["q"], a["k"], a["pt"], a["sl"], 16, 32)
    cand = ~np.isnan(s)
    assert np.array_equal(cand, ~np.isnan(s8))
    assert (s8[cand] >= s[cand] - 1e-12 * np.abs(s[cand])).all()
    assert (s8[cand] > s[cand]).any()           # the rounding does loosen some bounds
    G = d.Hq // d.Hkv
    for b in range(d.B):
        for g in range(d.Hkv):
            keys = token_keys(d, a, b, g)
            for p in np.where(cand[b, g])[0]:
                blk = keys[p * PS:(p + 1) * PS]
                true_max = max((blk @ f64(a["q"][b, g * G + j])).max() for j in range(G))
                assert s8[b, g, p] >= true_max - 1e-12 * abs(true_max)


def test_fp8_scores_equal_exact_scores_for_grid_keys():
    """Keys that are E4M3 normal values with a row maximum of 448 * 2^-3 (so
    e = -3 and scaling keeps them on the grid): the box survives unchanged
    and both scores agree exactly."""
    d, c, a = case_np(B=1, Hq=4, Hkv=1, D=16, lens=(64,), seed=2, poison=False)
    rng = np.random.default_rng(4)
    normals = np.array([v for v in FULL if abs(v) >= 2.0 ** -6 and abs(v) <= 56.0])
    k = rng.choice(normals, size=a["k"].shape)
    k.reshape(-1)[0] = 56.0                     # row maxima: 56 = 448 * 2^-3
    k[..., 0] = 56.0
    kb = torch.tensor(k, dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(kb.double(), torch.tensor(k))      # exact in bf16 too
    kk = wl.bits(kb)
    m = oracle.meta(d, kk, a["pt"], a["sl"])
    m8 = oracle.meta_fp8(d, m, a["pt"], a["sl"])
    s = oracle.scores(d, a["q"], kk, a["pt"], a["sl"], 0, 0)
    s8 = oracle.scores_fp8(d, a["q"], m8, a["pt"], a["sl"], 0, 0)
    cand = ~np.isnan(s)
    np.testing.assert_array_equal(s8[cand], s[cand])

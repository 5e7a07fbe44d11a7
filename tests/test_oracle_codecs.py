"""Pins for the oracle's E2M1 and UE4M3 codecs (CPU only).

The oracle's codecs are checked against (a) values computed here from the
formats' bit-field definitions, (b) an exact-rational brute-force nearest
search, (c) the round-to-nearest-even tie table in tests/golden, and (d)
PyTorch's float8_e4m3fn cast for in-range scale values.
"""
from fractions import Fraction
import os

import numpy as np
import pytest
import torch

import oracle


def e2m1_value_from_bits(code: int) -> float:
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def e4m3_value_from_bits(code: int) -> float:
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 0:
        return m / 8 * 2.0 ** (1 - 7)
    return (1 + m / 8) * 2.0 ** (e - 7)


def brute_nearest_even(x: float, codes_values):
    """Exact nearest by rational distance; ties -> even code; input |x| > max
    saturates.  codes_values: list of (code, value) non-negative, ascending."""
    a = Fraction(abs(x))
    best = None
    for code, v in codes_values:
        d = abs(a - Fraction(v))
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    return best[1]


E2M1_POS = [(c, e2m1_value_from_bits(c)) for c in range(8)]
E4M3_POS = [(c, e4m3_value_from_bits(c)) for c in range(127)]


def test_e2m1_decode_matches_format_definition():
    got = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    want = np.array([e2m1_value_from_bits(c) for c in range(16)], dtype=np.float32)
    assert np.array_equal(got, want)
    assert sorted(set(np.abs(want).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_ue4m3_decode_matches_format_definition():
    codes = np.arange(127, dtype=np.uint8)
    got = oracle.ue4m3_decode(codes)
    want = np.array([e4m3_value_from_bits(c) for c in range(127)], dtype=np.float32)
    assert np.array_equal(got, want)
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e2m1_tie_table(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "e2m1_rne_ties.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            x, v, c = line.split()
            rows.append((float(x), float(v), int(c)))
    xs = np.array([r[0] for r in rows], dtype=np.float32)
    codes = oracle.e2m1_encode(xs)
    for (x, v, c), got in zip(rows, codes):
        assert got == c, (x, got, c)
        dv = oracle.e2m1_decode(np.array([got], np.uint8))[0]
        assert dv == v and np.signbit(dv) == np.signbit(v)


def _probe_points(values):
    """Every representable value, every midpoint, and their fp32 neighbours."""
    pts = set()
    vals = sorted(set(values))
    for v in vals:
        pts.add(v)
    for a, b in zip(vals[:-1], vals[1:]):
        pts.add((a + b) / 2)
    out = []
    for p in pts:
        f = np.float32(p)
        out += [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))]
    return np.array([x for x in out if x >= 0], dtype=np.float32)


def test_e2m1_encode_bruteforce():
    rng = np.random.default_rng(123)
    pts = _probe_points([v for _, v in E2M1_POS] + [7.0, 12.0])
    rand = rng.uniform(0, 8, 4000).astype(np.float32)
    tiny = np.array([0.0, 1e-30, 2.0 ** -126, 2.0 ** -149, 0.2499999], dtype=np.float32)
    xs = np.concatenate([pts, rand, tiny, np.array([np.inf, 1e38], np.float32)])
    xs = np.concatenate([xs, -xs])
    got = oracle.e2m1_encode(xs)
    for x, g in zip(xs, got):
        a = min(abs(float(x)), 6.0) if np.isfinite(x) else 6.0
        want = brute_nearest_even(a, E2M1_POS) | (8 if np.signbit(x) else 0)
        assert g == want, (float(x), int(g), want)


def test_e2m1_sign_of_zero_follows_input():
    got = oracle.e2m1_encode(np.array([0.0, -0.0, 1e-9, -1e-9, 0.25, -0.25], np.float32))
    assert got.tolist() == [0, 8, 0, 8, 0, 8]


def test_ue4m3_encode_bruteforce_and_saturation():
    pts = _probe_points([v for _, v in E4M3_POS])
    rng = np.random.default_rng(7)
    rand = np.exp2(rng.uniform(-12, 9, 3000)).astype(np.float32)
    xs = np.concatenate([pts, rand])
    xs = xs[xs <= 448.0]
    got = oracle.ue4m3_encode(xs)
    for x, g in zip(xs, got):
        assert g == brute_nearest_even(float(x), E4M3_POS), (float(x), int(g))
    sat = oracle.ue4m3_encode(np.array([448.0, 449.0, 464.0, 500.0, 1e30, np.inf], np.float32))
    assert sat.tolist() == [0x7E] * 6
    zero = oracle.ue4m3_encode(np.array([0.0, -1.0, 2.0 ** -10, 2.0 ** -11], np.float32))
    assert zero.tolist() == [0, 0, 0, 0]  # 2^-10 is the tie between 0 and 2^-9: even code 0


def test_ue4m3_encode_matches_torch_float8_cast():
    # Dense sweep of fp32 bit patterns between 2^-12 and 448 (library cross-check).
    lo = np.float32(2.0 ** -12).view(np.uint32)
    hi = np.float32(448.0).view(np.uint32)
    bits = np.arange(lo, hi, 997, dtype=np.uint32)
    xs = np.concatenate([bits.view(np.float32), _probe_points([v for _, v in E4M3_POS])])
    xs = xs[(xs > 0) & (xs <= 448.0)].astype(np.float32)
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.ue4m3_encode(xs)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(xs[i]), int(got[i]), int(want[i])) for i in bad[:10]]

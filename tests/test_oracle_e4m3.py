"""Pins for the oracle's E4M3 decoder and encoder.

Sources: the OCP 8-bit floating point specification (E4M3) for the code
points; "add static LHS scaling support for GMM v2 FWD" (maxtext PR #4735),
review thread on the LhsRef docstring: values are clipped before the cast,
and on inner_kernel: the cast to the fp8 dtype, which rounds to nearest even.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_points.txt")


def _parse_value(tok: str) -> float:
    if tok == "nan":
        return math.nan
    if tok == "-0":
        return -0.0
    neg = tok.startswith("-")
    t = tok[1:] if neg else tok
    if "*" in t:
        a, b = t.split("*")
        v = float(a) * 2.0 ** int(b.split("^")[1])
    elif t.startswith("2^"):
        v = 2.0 ** int(t[2:])
    else:
        v = float(t)
    return -v if neg else v


def golden_points():
    pts = []
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            code, val = line.split()[:2]
            pts.append((int(code, 16), _parse_value(val)))
    return pts


@pytest.mark.parametrize("code,value", golden_points())
def test_decode_golden_points(code, value):
    got = oracle.e4m3_decode(np.array([code], np.uint8))[0]
    if math.isnan(value):
        assert math.isnan(got)
    else:
        assert got == value and math.copysign(1, got) == math.copysign(1, value)


def test_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    fin = ~np.isnan(ref)
    assert np.array_equal(ref[fin], got[fin])


def test_encode_round_trip_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = oracle.e4m3_decode(codes)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_midpoints_round_to_even():
    pos = np.arange(0, 0x7F, dtype=np.uint8)  # 0 .. 448, increasing values
    v = oracle.e4m3_decode(pos)
    mids = (v[:-1] + v[1:]) / 2.0
    got = oracle.e4m3_encode(mids)
    even = np.where(pos[:-1] % 2 == 0, pos[:-1], pos[1:])
    assert np.array_equal(got, even)
    # just off the midpoint goes to the nearer neighbour
    assert np.array_equal(oracle.e4m3_encode(np.nextafter(mids, 0)), pos[:-1])
    assert np.array_equal(oracle.e4m3_encode(np.nextafter(mids, 1e9)), pos[1:])


def test_clip_saturates_at_448():
    for v in [448.0, 448.5, 460.0, 464.0, 465.0, 480.0, 1e6, 3.0e38]:
        assert oracle.e4m3_encode(np.array([v]))[0] == 0x7E
        assert oracle.e4m3_encode(np.array([-v]))[0] == 0xFE


def test_tiny_values():
    enc = lambda v: int(oracle.e4m3_encode(np.array([v]))[0])  # noqa: E731
    assert enc(2.0 ** -9) == 0x01
    assert enc(2.0 ** -10) == 0x00  # tie between 0 and 2^-9 -> even (0)
    assert enc(-(2.0 ** -10)) == 0x80
    assert enc(3 * 2.0 ** -11) == 0x01  # 0.75 of the spacing -> 1
    assert enc(1e-30) == 0x00
    assert enc(1.5 * 2.0 ** -9) == 0x02  # tie between 1 and 2 -> even (2)
    assert enc(7.5 * 2.0 ** -9) == 0x08  # tie between 7*2^-9 and 2^-6 -> even (0x08)


def test_encode_matches_torch_cast_in_range():
    """torch's float8_e4m3fn cast is round-to-nearest-even inside +-448."""
    gen = torch.Generator().manual_seed(1)
    x = torch.cat([
        (torch.rand(20000, generator=gen) * 2 - 1) * 448,
        torch.randn(20000, generator=gen),
        torch.randn(20000, generator=gen) * 2.0 ** -8,
    ]).to(torch.float32)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x.to(torch.float64).numpy())
    assert np.array_equal(ref, got)

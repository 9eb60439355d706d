"""Pins for the oracle's number-format routines (binary16 and E4M3).

Each is checked against an independent library cast (numpy's binary16, torch's
float8_e4m3fn) and against the spec-fixed bit patterns in tests/golden/formats.txt.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "formats.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, val, bits = line.split()
            rows.append((fmt, float(val), int(bits, 16)))
    return rows


@pytest.mark.parametrize("fmt,val,bits", _golden())
def test_golden_bit_patterns(fmt, val, bits):
    if fmt == "e4m3":
        assert oracle.e4m3_encode(val) == bits
        assert oracle.e4m3_decode(bits) == val
    else:
        assert oracle.f16_to_f64(bits) == val
        assert oracle.round_f16(val) == val


def test_f16_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_f16_round_matches_numpy_on_boundaries():
    # every finite positive binary16 value, the midpoints between neighbours (ties) and
    # one fp64 ulp either side of each midpoint: every rounding decision is exercised
    vals = np.arange(0, 0x7c00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    xs = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf),
                         [65519.99, 65520.0, 70000.0]])
    rng = np.random.default_rng(0)
    xs = xs[rng.permutation(len(xs))[:40000]]
    xs = np.concatenate([xs, -xs[:2000]])
    ref = xs.astype(np.float16).astype(np.float64)
    got = np.array([oracle.round_f16(x) for x in xs])
    assert np.array_equal(got, ref)


def test_e4m3_decode_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_e4m3_encode_matches_torch_on_boundaries():
    finite = np.array([oracle.e4m3_decode(c) for c in range(0, 0x7f)])   # 0 .. 448
    mids = (finite[:-1] + finite[1:]) / 2
    f32 = lambda a: a.astype(np.float32)
    xs = np.concatenate([finite, mids,
                         f32(np.nextafter(f32(mids), np.float32(0))),
                         f32(np.nextafter(f32(mids), np.float32(np.inf)))]).astype(np.float64)
    xs = np.concatenate([xs, -xs])
    ref = torch.from_numpy(xs.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(x) for x in xs], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates_to_448():
    for x in (448.0, 449.0, 463.99, 464.0, 500.0, 1e6):
        assert oracle.e4m3_encode(x) == 0x7E
        assert oracle.e4m3_encode(-x) == 0xFE
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F

"""Pins of the oracle's FP8 / FP16 codecs against the format definitions and
against independent library implementations (CPU only)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_float(tok: str) -> float:
    if "0x" in tok.lower() and "p" in tok.lower():
        return float.fromhex(tok)
    return float(tok)


def test_e4m3_decode_closed_form_points():
    assert oracle.e4m3_decode(0x38) == 1.0
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0xFE) == -448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))
    z = oracle.e4m3_decode(0x80)
    assert z == 0.0 and math.copysign(1.0, z) == -1.0


def test_e4m3_decode_matches_library_table():
    """Second witness: torch's float8_e4m3fn decode of every byte."""
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = oracle.e4m3_table()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    fin = ~np.isnan(ours)
    np.testing.assert_array_equal(ours[fin], lib[fin])
    np.testing.assert_array_equal(np.signbit(ours[fin]), np.signbit(lib[fin]))


def test_e4m3_positive_codes_monotone_and_count():
    t = oracle.e4m3_table()
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.sum(np.isfinite(t)) == 254
    assert np.nanmax(np.abs(t)) == 448.0


def test_e5m2_decode_points_and_library_table():
    assert oracle.e5m2_decode(0x3C) == 1.0
    assert oracle.e5m2_decode(0x7B) == 57344.0
    assert oracle.e5m2_decode(0x01) == 2.0 ** -16
    assert oracle.e5m2_decode(0x04) == 2.0 ** -14
    assert oracle.e5m2_decode(0x7C) == math.inf and oracle.e5m2_decode(0xFC) == -math.inf
    assert math.isnan(oracle.e5m2_decode(0x7D))
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    ours = oracle.e5m2_table()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    fin = ~np.isnan(ours)
    np.testing.assert_array_equal(ours[fin], lib[fin])


def test_fp16_decode_all_patterns_vs_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    lib = bits.view(np.float16).astype(np.float64)
    ours = np.array([oracle.fp16_decode(int(b)) for b in bits])
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    fin = ~np.isnan(lib)
    np.testing.assert_array_equal(ours[fin], lib[fin])
    np.testing.assert_array_equal(np.signbit(ours[fin]), np.signbit(lib[fin]))


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_encode_roundtrip_all_codes(fmt):
    dec = oracle.e4m3_decode if fmt == "e4m3" else oracle.e5m2_decode
    enc = oracle.e4m3_encode if fmt == "e4m3" else oracle.e5m2_encode
    for c in range(256):
        v = dec(c)
        if math.isnan(v) or math.isinf(v):
            continue
        assert enc(v) == c, (fmt, hex(c), v)


def test_e4m3_encode_golden_cases():
    path = os.path.join(GOLDEN, "e4m3_encode_cases.txt")
    n = 0
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            v, code = _parse_float(tok[0]), int(tok[1], 16)
            got = oracle.e4m3_encode(v)
            assert got == code, (line, hex(got))
            n += 1
    assert n >= 15


def test_e4m3_encode_nan_and_inf():
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F
    assert oracle.e4m3_encode(float("inf")) == 0x7E
    assert oracle.e4m3_encode(float("-inf")) == 0xFE


def _midpoints_and_neighbours(table):
    """All in-range float32 values at and around every midpoint of two
    adjacent finite codes, plus the codes themselves."""
    vals = np.unique(table[np.isfinite(table)])
    mids = (vals[:-1] + vals[1:]) / 2.0           # exact in binary64, exact in binary32 too
    m32 = mids.astype(np.float32)
    assert np.all(m32.astype(np.float64) == mids)
    cand = [m32, np.nextafter(m32, np.float32(np.inf)), np.nextafter(m32, np.float32(-np.inf)),
            vals.astype(np.float32)]
    return np.concatenate(cand)


def test_e4m3_encode_vs_library_cast_in_range():
    """Second witness for RNE: torch's float32 -> float8_e4m3fn cast, compared on
    every midpoint of adjacent codes and the float32 neighbours of each."""
    x = _midpoints_and_neighbours(oracle.e4m3_table())
    x = x[np.abs(x) <= 448.0]
    lib = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode_array(x)
    np.testing.assert_array_equal(ours, lib)


def test_e5m2_encode_vs_library_cast_in_range():
    x = _midpoints_and_neighbours(oracle.e5m2_table())
    x = x[np.abs(x) <= 57344.0]
    lib = torch.from_numpy(x.copy()).to(torch.float8_e5m2).view(torch.uint8).numpy()
    ours = oracle.e5m2_encode_array(x)
    np.testing.assert_array_equal(ours, lib)


def test_e4m3_encode_random_float32_vs_library():
    g = np.random.default_rng(7)
    x = (g.standard_normal(20000) * np.exp(g.uniform(-14, 6, 20000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    lib = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode_array(x), lib)

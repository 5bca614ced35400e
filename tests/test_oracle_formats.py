"""Pins for the oracle's number formats (CPU only).

The decoders are checked exhaustively against library conversions (numpy's
binary16, torch's bfloat16 and float8_e4m3fn), and the E4M3 rounding against the
OCP code points in tests/golden/e4m3_code_points.txt, against torch's
round-to-nearest-even conversion inside the finite range, and by round trips.
"""

import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _same(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    both_nan = np.isnan(a) & np.isnan(b)
    eq = (a == b) & (np.signbit(a) == np.signbit(b))
    return bool(np.all(both_nan | eq))


def test_f16_decode_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    assert _same(oracle.f16_decode(bits), ref)


def test_bf16_decode_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert _same(oracle.bf16_decode(bits), ref)


def test_e4m3_decode_exhaustive():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    assert _same(got, ref)
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert np.nanmax(np.abs(got)) == 448.0


def _golden_points():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_code_points.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            x, code = line.split()[:2]
            v = float.fromhex(x) if "p" in x else float(x)
            rows.append((v, int(code, 16)))
    return rows


@pytest.mark.parametrize("x,code", _golden_points())
def test_e4m3_encode_code_points(x, code):
    assert int(oracle.e4m3_encode(np.float32(x)).reshape(-1)[0]) == code


def test_e4m3_encode_nan():
    assert int(oracle.e4m3_encode(np.float32("nan")).reshape(-1)[0]) == 0x7F


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32) * 50,
        rng.uniform(-448, 448, 200_000).astype(np.float32),
        (rng.standard_normal(200_000) * 1e-2).astype(np.float32),
        np.ldexp(rng.uniform(-1, 1, 100_000), rng.integers(-14, 9, 100_000)).astype(np.float32),
    ])
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def test_e4m3_encode_all_f16_values():
    bits = np.arange(1 << 16, dtype=np.uint16)
    x = bits.view(np.float16).astype(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) < 448)]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def test_e4m3_round_trip_and_saturation():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)
    big = np.array([449, 500, 1e4, np.inf, -np.inf, -460], dtype=np.float32)
    assert list(oracle.e4m3_encode(big)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_to_f64_f32_passthrough():
    x = np.array([1.5, -2.25, 3e-40], dtype=np.float32)
    assert _same(oracle.to_f64(x, "f32"), x.astype(np.float64))

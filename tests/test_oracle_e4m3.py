"""Pins for the oracle's FP8 e4m3 codec (OCP 8-bit floating point, E4M3 variant).

The codec decides every V code and every P code of the method, so it is pinned against
values fixed by the format's definition and against an independent library cast
(torch.float8_e4m3fn, round-to-nearest-even inside the finite range).
"""
import math

import numpy as np
import pytest
import torch


def test_decode_all_codes_match_library(oracle):
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        ours = oracle.e4m3_to_f32(c)
        if math.isnan(lib[c]):
            assert math.isnan(ours), c
        else:
            assert ours == lib[c] and math.copysign(1, ours) == math.copysign(1, lib[c]), c


@pytest.mark.parametrize("x,code", [
    (0.0, 0x00), (-0.0, 0x80), (1.0, 0x38), (-1.0, 0xB8),
    (448.0, 0x7E), (-448.0, 0xFE),
    (464.0, 0x7E), (1e9, 0x7E), (-1e9, 0xFE), (float("inf"), 0x7E),  # satfinite
    (2.0 ** -9, 0x01),          # smallest subnormal
    (2.0 ** -10, 0x00),         # half of it: tie between 0 and 2^-9 -> even code 0
    (3 * 2.0 ** -10, 0x02),     # tie between codes 1 and 2 -> even code 2
    (2.0 ** -6, 0x08),          # smallest normal
    (7 * 2.0 ** -9, 0x07),      # largest subnormal
    (1.0625, 0x38),             # tie between 1.0 (0x38) and 1.125 (0x39) -> 0x38
    (1.1875, 0x3A),             # tie between 1.125 (0x39) and 1.25 (0x3A) -> 0x3A
    (240.0, 0x77), (256.0, 0x78), (416.0, 0x7D),
])
def test_encode_closed_forms(oracle, x, code):
    assert oracle.e4m3_from_f32(x) == code


def test_encode_matches_library_inside_range(oracle):
    rng = np.random.default_rng(3)
    # random magnitudes over the whole exponent range, plus every midpoint between
    # adjacent codes and its fp32 neighbours (the rounding decisions that matter)
    mags = np.exp2(rng.uniform(-12, np.log2(463.9), 4000)).astype(np.float32)
    vals = [float(v) for v in mags] + [-float(v) for v in mags[:1000]]
    codes = [oracle.e4m3_to_f32(c) for c in range(0x7F)]
    for a, b in zip(codes[:-1], codes[1:]):
        mid = np.float32((a + b) / 2)
        vals += [float(mid), float(np.nextafter(mid, np.float32(0))),
                 float(np.nextafter(mid, np.float32(1e9)))]
    x = torch.tensor(vals, dtype=torch.float32)
    lib = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_from_f32(v) for v in vals], np.uint8)
    assert np.array_equal(ours, lib)


def test_round_trip_every_finite_code(oracle):
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_from_f32(oracle.e4m3_to_f32(c)) == c


def test_monotone(oracle):
    xs = np.linspace(-470, 470, 20001, dtype=np.float32)
    dec = [oracle.e4m3_to_f32(oracle.e4m3_from_f32(float(v))) for v in xs]
    assert all(b >= a for a, b in zip(dec[:-1], dec[1:]))

"""Pins for the oracle's FP8 / bf16 codecs (no GPU).

The codec is pinned against (a) the maxima printed on the AstrAI pages
(``FP8_MAX = {"e4m3": 448.0, "e5m2": 57344.0}`` in ``astrai/extension/fp8.py``;
``kFp8Max`` in ``csrc/kernels/fp8/common.h``), (b) values that follow by hand from
the bit-field definitions, (c) the full 256-code round trip and round-half-even
at every midpoint, and (d) PyTorch's own float8 / bfloat16 casts, an independent
implementation, inside their non-saturating range.
"""

import numpy as np
import pytest
import torch

from oracle import fp8_codec as C


def test_fp8_max_matches_pages():
    assert C.FP8_MAX["e4m3"] == 448.0
    assert C.FP8_MAX["e5m2"] == 57344.0
    assert C.max_code("e4m3") == 0x7E
    assert C.max_code("e5m2") == 0x7B
    assert C.decode_code(0x7E, "e4m3") == 448.0
    assert C.decode_code(0x7B, "e5m2") == 57344.0


@pytest.mark.parametrize("fmt,code,value", [
    # E4M3FN: bias 7, 3 mantissa bits
    ("e4m3", 0x00, 0.0),
    ("e4m3", 0x01, 2.0 ** -9),            # smallest subnormal 0.001 * 2^-6
    ("e4m3", 0x07, 7 * 2.0 ** -9),        # largest subnormal
    ("e4m3", 0x08, 2.0 ** -6),            # smallest normal
    ("e4m3", 0x38, 1.0),                  # exponent field 7
    ("e4m3", 0x39, 1.125),
    ("e4m3", 0x3C, 1.5),
    ("e4m3", 0x40, 2.0),
    ("e4m3", 0x7D, 416.0),
    ("e4m3", 0xB8, -1.0),
    ("e4m3", 0xFE, -448.0),
    # E5M2: bias 15, 2 mantissa bits
    ("e5m2", 0x01, 2.0 ** -16),
    ("e5m2", 0x03, 3 * 2.0 ** -16),
    ("e5m2", 0x04, 2.0 ** -14),
    ("e5m2", 0x3C, 1.0),
    ("e5m2", 0x3D, 1.25),
    ("e5m2", 0x7A, 49152.0),
    ("e5m2", 0xBC, -1.0),
])
def test_hand_decoded_values(fmt, code, value):
    assert C.decode_code(code, fmt) == value


def test_specials():
    assert np.isnan(C.decode_code(0x7F, "e4m3"))
    assert np.isnan(C.decode_code(0xFF, "e4m3"))
    assert C.decode_code(0x7C, "e5m2") == np.inf
    assert C.decode_code(0xFC, "e5m2") == -np.inf
    for c in (0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF):
        assert np.isnan(C.decode_code(c, "e5m2"))
    # E4M3FN has exactly two NaN codes and no infinities
    tab = C.decode_table("e4m3")
    assert np.isnan(tab).sum() == 2 and not np.isinf(tab).any()
    tab = C.decode_table("e5m2")
    assert np.isnan(tab).sum() == 6 and np.isinf(tab).sum() == 2
    assert np.signbit(C.decode_code(0x80, "e4m3")) and C.decode_code(0x80, "e4m3") == 0.0


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_round_trip_every_code(fmt):
    tab = C.decode_table(fmt)
    top = C.max_code(fmt)
    for code in range(256):
        v = tab[code]
        if np.isnan(v):
            continue
        got = int(C.encode(np.array([v]), fmt)[0])
        if np.isinf(v):  # E5M2 infinities saturate to the finite max
            assert got == (top | (code & 0x80))
        else:
            assert got == code, (fmt, hex(code), v, hex(got))


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_midpoints_round_to_even_and_neighbours(fmt):
    tab = C.decode_table(fmt)
    top = C.max_code(fmt)
    for c in range(top):
        lo, hi = tab[c], tab[c + 1]
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2  # midpoints are exact in fp32
        even = c if c % 2 == 0 else c + 1
        for sign, sbit in ((1.0, 0), (-1.0, 0x80)):
            assert C.encode(np.array([sign * mid]), fmt)[0] == (even | sbit)
            up = np.nextafter(mid, np.float32(np.inf), dtype=np.float32)
            dn = np.nextafter(mid, np.float32(0), dtype=np.float32)
            assert C.encode(np.array([sign * up], np.float32), fmt)[0] == ((c + 1) | sbit)
            assert C.encode(np.array([sign * dn], np.float32), fmt)[0] == (c | sbit)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_saturation_and_signed_zero(fmt):
    mx = C.FP8_MAX[fmt]
    top = C.max_code(fmt)
    vals = np.array([mx, mx * 1.01, 1e30, np.inf, -mx * 3, -np.inf], dtype=np.float32)
    got = C.encode(vals, fmt)
    assert list(got) == [top, top, top, top, top | 0x80, top | 0x80]
    tiny = np.array([-1e-30, 1e-30, -0.0, 0.0], dtype=np.float32)
    assert list(C.encode(tiny, fmt)) == [0x80, 0x00, 0x80, 0x00]
    assert C.encode(np.array([np.nan], np.float32), fmt)[0] == 0x7F


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_monotone(fmt):
    v = np.linspace(0, C.FP8_MAX[fmt] * 1.2, 200001).astype(np.float32)
    codes = C.encode(v, fmt).astype(np.int64)
    assert np.all(np.diff(codes) >= 0)


@pytest.mark.parametrize("fmt,dt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_agrees_with_torch_cast_in_range(fmt, dt):
    """PyTorch's float8 casts round to nearest even; inside +-max they must agree."""
    rng = np.random.default_rng(1234)
    mx = C.FP8_MAX[fmt]
    # log-uniform magnitudes across the whole range including subnormals
    mag = np.exp(rng.uniform(np.log(2.0 ** -20), np.log(mx), 400000))
    sign = rng.choice([-1.0, 1.0], mag.size)
    v = (sign * mag).astype(np.float32)
    v = v[np.abs(v) <= mx]
    tab = C.decode_table(fmt)
    top = C.max_code(fmt)
    mids = np.array([(tab[c] + tab[c + 1]) / 2 for c in range(top)], dtype=np.float32)
    v = np.concatenate([v, mids, -mids])
    ours = C.encode(v, fmt)
    theirs = torch.from_numpy(v).to(dt).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_bf16_round_trip_and_torch_agreement():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    ours = C.f64_to_bf16_bits(v.astype(np.float64))
    theirs = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)
    back = C.bf16_bits_to_f64(ours)
    assert np.array_equal(C.f64_to_bf16_bits(back), ours)


def test_bf16_hand_values():
    # 1 + 2^-8 is the midpoint between 1 and 1 + 2^-7: ties go to the even 1.0
    assert C.round_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 is the midpoint between 1+2^-7 (odd) and 1+2^-6 (even)
    assert C.round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    assert C.round_to_bf16(np.array([1.0 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1.0 + 2.0 ** -7
    assert C.f64_to_bf16_bits(np.array([1.0]))[0] == 0x3F80
    assert C.f64_to_bf16_bits(np.array([-2.0]))[0] == 0xC000
    assert np.isinf(C.round_to_bf16(np.array([3.5e38]))[0])

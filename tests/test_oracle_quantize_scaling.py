"""Pins for the oracle's quantize, scale formula and history ring (no GPU).

Sources: AstrAI compare view -- ``astrai/extension/fp8.py`` (``FP8Recipe``,
``_ScaleRing``, ``fp8_linear_forward``) and ``csrc/kernels/fp8/quantize.cuh``
(``publish_amax``, ``fp8_quantize_kernel``); the extension commit log (amax is the
raw-domain max; transposed copies do not fold rings; no scale leak across two
delayed steps).  Closed forms and brute force stand in for stored goldens: the
pages print no worked FP8 numbers.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp8_codec as C
from oracle import quantize as Q
from oracle import scaling as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _exact_rn32(fr: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32 (ties to even), by search."""
    f = np.float32(float(fr))  # within one ulp
    best = None
    for cand in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        err = abs(Fraction(float(cand)) - fr)
        key = (err, int(np.float32(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return np.float32(best[1])


def test_reciprocal_is_correctly_rounded():
    rng = np.random.default_rng(3)
    s = np.exp(rng.uniform(-30, 10, 3000)).astype(np.float32)
    for v in s:
        assert Q.reciprocal_f32(v) == _exact_rn32(Fraction(1) / Fraction(float(v)))


def test_quantize_matches_torch_reference_path():
    """q(RN32(x*RN32(1/s))) against PyTorch: fp32 multiply, clamp to +-max, cast."""
    for fmt, dt in (("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)):
        mx = C.FP8_MAX[fmt]
        for seed, s in ((0, 1.0), (1, 0.0173), (2, 3.3e-4), (3, 17.25), (4, 1e-12)):
            g = torch.Generator().manual_seed(seed)
            x = (torch.randn(4096, generator=g) * 3).to(torch.bfloat16).float()
            ours = Q.quantize_values(x.numpy(), s, fmt)
            mult = torch.tensor(1.0, dtype=torch.float32) / torch.tensor(s, dtype=torch.float32)
            y = (x * mult).clamp(-mx, mx)
            theirs = y.to(dt).view(torch.uint8).numpy()
            assert np.array_equal(ours, theirs), (fmt, s)


def test_amax_raw_domain_and_nan():
    x = np.array([0.5, -3.0, 2.0], np.float32)
    assert Q.amax(x) == 3.0
    # amax is of the unscaled input: it does not depend on the step
    x8a, a1 = Q.quantize(x, 1.0, "e4m3")
    x8b, a2 = Q.quantize(x, 1e-3, "e4m3")
    assert a1 == a2 == 3.0
    assert Q.amax(np.array([np.nan, -1.0, np.nan], np.float32)) == 1.0
    assert Q.amax(np.zeros(0, np.float32)) == 0.0
    assert Q.amax(np.array([-np.inf, 1.0], np.float32)) == np.inf


def test_transposed_and_dual_orientations():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((37, 53)).astype(np.float32)
    x8, a = Q.quantize(x, 0.01, "e5m2")
    xt, at = Q.quantize_transposed(x, 0.01, "e5m2")
    d8, dt, ad = Q.quantize_dual(x, 0.01, "e5m2")
    assert xt.shape == (53, 37)
    for r in range(37):
        for c in range(53):
            assert xt[c, r] == x8[r, c]
    assert np.array_equal(d8, x8) and np.array_equal(dt, xt)
    assert a == at == ad


def test_golden_quantize_examples():
    """Hand-worked examples (format definitions + RN32 arithmetic) in a fixture."""
    with open(os.path.join(GOLDEN, "quantize_examples.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        x = np.array(case["x"], np.float32)
        got = Q.quantize_values(x, case["scale"], case["fmt"])
        assert [int(v) for v in got] == [int(h, 16) for h in case["codes"]], case["why"]


def test_scale_formula_closed_forms():
    assert S.scale_from_peak(448.0, 448.0, 1.0) == 1.0
    assert S.scale_from_peak(57344.0, 57344.0, 1.0) == 1.0
    assert S.scale_from_peak(896.0, 448.0, 2.0) == 1.0
    assert S.scale_from_peak(0.0, 448.0, 1.0) == np.float32(1e-12)  # floor
    assert S.scale_from_peak(1e-20, 448.0, 1.0) == np.float32(1e-12)
    # margin m divides the step by exactly 2^m
    for m in range(6):
        base = S.scale_from_peak(3.7, 448.0, 1.0)
        assert S.scale_from_peak(3.7, 448.0, 2.0 ** m) == base / np.float32(2.0 ** m)
    # peak/fp8_max is one IEEE fp32 division
    for p in (1.0, 3.14159, 1000.5, 7e-3):
        assert S.scale_from_peak(p, 448.0) == _exact_rn32(Fraction(float(np.float32(p))) / 448)


def test_ring_window_matches_sliding_max():
    n = 4
    rng = np.random.default_rng(11)
    amaxes = np.float32(np.exp(rng.uniform(-5, 5, 13)))
    ring = S.Ring(n, "e4m3")
    ring.seed(np.array([amaxes[0]], np.float32))
    used = []
    for t, a in enumerate(amaxes):
        step = ring.scale
        used.append(step)
        ring.fold(a, step)
        ring.advance()
        window = amaxes[max(0, t - n + 1): t + 1]
        want = np.float32(np.float32(np.max(window)) / np.float32(448.0))
        assert ring.scale == max(want, np.float32(1e-12))
        assert ring.scale_used == step
        assert ring.state[n + 2] == 0 and ring.state[n + 3] == 0
        assert ring.idx == (t + 1) % n


def test_step0_delayed_equals_dynamic():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 64)) * 5).astype(np.float32)
    ring = S.Ring(16, "e4m3")
    ring.seed(x)
    assert ring.scale == S.dynamic_scale(x, "e4m3")
    ring.fold(Q.amax(x), ring.scale)  # the first fold re-records the same amax
    assert ring.scale == S.dynamic_scale(x, "e4m3")


def test_no_scale_leak_two_delayed_steps():
    """Two delayed steps whose amax changes by 2^k.  Bytes quantized with s_used
    and dequantized with s_used reproduce clip(x, +-FP8_MAX * s_used) within fp8
    error; dequantizing with the just-published step instead would be off by
    exactly the ratio of the two steps (the leak the pages' regression test guards)."""
    rng = np.random.default_rng(9)
    x0 = rng.standard_normal(2048).astype(np.float32)
    for k in (3, -3):
        x1 = x0 * np.float32(2.0 ** k)
        ring = S.Ring(16, "e4m3")
        ring.seed(x0)
        for t, x in enumerate((x0, x1)):
            s_used = ring.scale
            x8, a = Q.quantize(x, s_used, "e4m3")
            ring.fold(a, s_used)
            ring.advance()
            deq = C.decode(x8, "e4m3") * np.float64(s_used)
            want = np.clip(x.astype(np.float64), -448.0 * s_used, 448.0 * s_used)
            big = np.abs(want) >= 2.0 ** -6 * s_used  # values in the normal range of E4M3
            rel = np.abs(deq - want)[big] / np.abs(want)[big]
            assert rel.max() <= 2.0 ** -4 + 1e-9
            if t == 1 and k > 0:
                # the window grew: the published step differs from the one used
                assert ring.scale == np.float32(np.float32(Q.amax(x1)) / np.float32(448.0))
                wrong = C.decode(x8, "e4m3") * np.float64(ring.scale)
                nz = deq != 0
                assert np.allclose(wrong[nz] / deq[nz], float(ring.scale) / float(s_used))
                assert float(ring.scale) / float(s_used) == pytest.approx(2.0 ** k, rel=1e-6)
            if t == 1 and k < 0:
                # the window still holds step 0's larger amax: step unchanged
                assert ring.scale == s_used

"""Pins for the oracle's GEMM and linear compositions (no GPU).

Sources: AstrAI compare view -- ``astrai/extension/ops/fp8.py`` (``mm_fp8``:
``a @ b * scale (+ bias)``, 2-D / 3-D with batch broadcast),
``csrc/kernels/fp8/gemm/epilogue.cuh`` (bias added to the fp32 accumulator before
one bf16 rounding), ``csrc/kernels/fp8/common.h`` (layout tags) and
``astrai/extension/fp8.py`` (``_LinearFp8``: NT routing of forward, dX, dW).
The GEMM is pinned against an exact-rational brute-force triple loop, layout
equivalences, one-hot and zero operands, and the batch broadcast rule.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import fp8_codec as C
from oracle import gemm as G
from oracle import linear as L
from oracle import quantize as Q
from oracle import scaling as S


def _rand_codes(rng, shape, fmt):
    """Random finite fp8 codes (all magnitudes, both signs)."""
    tab = C.decode_table(fmt)
    finite = np.array([c for c in range(256) if np.isfinite(tab[c])], np.uint8)
    return rng.choice(finite, size=shape)


def _brute(a_codes, b_codes, fmt_a, fmt_b, sa, sb, bias_bits):
    """Exact rational A[M,K] @ B[K,N] * RN32(sa*sb) + bias, triple loop."""
    m, k = a_codes.shape
    n = b_codes.shape[1]
    sc = Fraction(float(np.float32(sa) * np.float32(sb)))
    out = np.zeros((m, n), dtype=object)
    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for p in range(k):
                acc += Fraction(C.decode_code(int(a_codes[i, p]), fmt_a)) * \
                    Fraction(C.decode_code(int(b_codes[p, j]), fmt_b))
            v = acc * sc
            if bias_bits is not None:
                v += Fraction(float(C.bf16_bits_to_f64(bias_bits[j:j + 1])[0]))
            out[i, j] = v
    return out


@pytest.mark.parametrize("fmt_a,fmt_b", [("e4m3", "e4m3"), ("e5m2", "e5m2"), ("e5m2", "e4m3")])
def test_gemm_equals_exact_brute_force(fmt_a, fmt_b):
    rng = np.random.default_rng(21)
    for m, n, k in ((1, 1, 1), (3, 5, 7), (16, 16, 16), (9, 4, 13)):
        a = _rand_codes(rng, (m, k), fmt_a)
        b = _rand_codes(rng, (k, n), fmt_b)
        bias = C.f64_to_bf16_bits(rng.standard_normal(n))
        ref, s_abs, sc = G.gemm_ref(a, b, "NN", fmt_a, fmt_b, 0.75, 1.3, bias)
        exact = _brute(a, b, fmt_a, fmt_b, 0.75, 1.3, bias)
        for i in range(m):
            for j in range(n):
                # one fp64 rounding for the scale product and one for the bias
                # add, each relative to the magnitudes involved
                mag = Fraction(float(s_abs[i, j])) * Fraction(float(sc)) + \
                    abs(Fraction(float(C.bf16_bits_to_f64(bias[j:j + 1])[0])))
                tol = mag * Fraction(2) ** -51
                if not fmt_a == fmt_b == "e4m3":
                    # E5M2 partial sums may round in fp64
                    tol += Fraction(2) ** -45 * Fraction(float(s_abs[i, j])) * Fraction(float(sc))
                assert abs(Fraction(ref[i, j]) - exact[i, j]) <= tol


def test_e4m3_accumulation_is_order_independent_at_k8192():
    """E4M3 partial sums are multiples of 2^-18 below 2^31, so fp64 is exact."""
    rng = np.random.default_rng(4)
    k = 8192
    a = _rand_codes(rng, (1, k), "e4m3")
    b = _rand_codes(rng, (k, 1), "e4m3")
    av = C.decode(a, "e4m3")[0]
    bv = C.decode(b, "e4m3")[:, 0]
    scaled = [int(x * 2 ** 9) * int(y * 2 ** 9) for x, y in zip(av, bv)]
    exact = Fraction(sum(scaled), 2 ** 18)
    ref, _, _ = G.gemm_ref(a, b, "NN", sa=1.0, sb=1.0)
    assert Fraction(ref[0, 0]) == exact
    assert Fraction(float(np.sum(av[::-1] * bv[::-1]))) == exact


def test_layouts_are_equivalent():
    rng = np.random.default_rng(8)
    a = _rand_codes(rng, (24, 40), "e4m3")   # [M][K]
    b = _rand_codes(rng, (40, 17), "e4m3")   # [K][N]
    ref, _, _ = G.gemm_ref(a, b, "NN", sa=0.5, sb=2.0)
    for layout, a_st, b_st in (("NT", a, b.T), ("TN", a.T, b), ("TT", a.T, b.T)):
        got, _, _ = G.gemm_ref(np.ascontiguousarray(a_st), np.ascontiguousarray(b_st),
                               layout, sa=0.5, sb=2.0)
        assert np.array_equal(got, ref), layout


def test_one_hot_rows_copy_columns_and_zero_gives_bias():
    rng = np.random.default_rng(1)
    k, n = 32, 20
    b = _rand_codes(rng, (n, k), "e4m3")  # stored [N][K] (NT)
    one = C.encode(np.array([1.0]), "e4m3")[0]
    a = np.zeros((k, k), np.uint8)
    a[np.arange(k), np.arange(k)] = one
    bias = C.f64_to_bf16_bits(rng.standard_normal(n))
    ref, _, sc = G.gemm_ref(a, b, "NT", sa=1.0, sb=1.0, bias=bias)
    want = C.decode(b, "e4m3").T + C.bf16_bits_to_f64(bias)[None, :]
    assert np.array_equal(ref, want)
    zero = np.zeros((5, k), np.uint8)
    ref0, s_abs0, _ = G.gemm_ref(zero, b, "NT", sa=3.0, sb=7.0, bias=bias)
    assert np.array_equal(ref0, np.broadcast_to(C.bf16_bits_to_f64(bias), (5, n)))
    assert np.all(s_abs0 == 0)


def test_batch_broadcast_and_entry():
    rng = np.random.default_rng(2)
    a = _rand_codes(rng, (3, 8, 16), "e4m3")
    b = _rand_codes(rng, (1, 12, 16), "e4m3")  # one B shared by every batch
    ref, s_abs, sc = G.gemm_ref(a, b, "NT", sa=1.5, sb=0.5)
    assert ref.shape == (3, 8, 12)
    for i in range(3):
        r_i, _, _ = G.gemm_ref(a[i], b[0], "NT", sa=1.5, sb=0.5)
        assert np.array_equal(ref[i], r_i)
        e, e_abs, _ = G.gemm_entry(a, b, "NT", "e4m3", "e4m3", 1.5, 0.5, None, None, i, 5, 7)
        assert e == ref[i, 5, 7] and e_abs == s_abs[i, 5, 7]


def test_fp8_bias_with_scale():
    rng = np.random.default_rng(3)
    a = _rand_codes(rng, (4, 8), "e4m3")
    b = _rand_codes(rng, (6, 8), "e4m3")
    b8 = _rand_codes(rng, (6,), "e4m3")
    ref, _, sc = G.gemm_ref(a, b, "NT", sa=1.0, sb=1.0, bias=b8, bias_scale=0.125)
    plain, _, _ = G.gemm_ref(a, b, "NT", sa=1.0, sb=1.0)
    assert np.array_equal(ref - plain, np.broadcast_to(C.decode(b8, "e4m3") * 0.125, (4, 6)))


def test_tolerance_formula():
    ref = np.array([1.0, -2.0, 0.0])
    s_abs = np.array([4.0, 4.0, 1024.0])
    tol = G.gemm_tolerance(ref, s_abs, np.float32(0.5))
    assert np.allclose(tol, [2 ** -8 + 2 ** -19, 2 ** -7 + 2 ** -19, 2 ** -11])


def _bits(x):
    return C.f64_to_bf16_bits(np.asarray(x, np.float64))


def test_linear_forward_dynamic_close_to_fp64():
    rng = np.random.default_rng(0)
    x = _bits(rng.standard_normal((64, 128)))
    w = _bits(rng.standard_normal((96, 128)) * 0.02)
    b = _bits(rng.standard_normal(96) * 0.1)
    out = L.forward(x, w, b, "e4m3")
    exact = C.bf16_bits_to_f64(x) @ C.bf16_bits_to_f64(w).T + C.bf16_bits_to_f64(b)
    err = np.abs(out["y"] - exact)
    # each product carries <= 2 * 2^-4 relative quantization error
    bound = 2 * 2.0 ** -4 * (np.abs(C.bf16_bits_to_f64(x)) @ np.abs(C.bf16_bits_to_f64(w)).T) + 1e-6
    assert np.all(err <= bound)
    assert out["sx"] == S.dynamic_scale(C.bf16_bits_to_f64(x).astype(np.float32), "e4m3")


def test_linear_backward_routes_and_grad_bias():
    rng = np.random.default_rng(5)
    m, k, n = 48, 32, 40
    g = _bits(rng.standard_normal((m, n)) * 1e-3)
    x = _bits(rng.standard_normal((m, k)))
    w = _bits(rng.standard_normal((n, k)) * 0.02)
    out = L.backward(g, x, w, "e5m2")
    gv, xv, wv = (C.bf16_bits_to_f64(t) for t in (g, x, w))
    # the NT routing computes g @ w and g^T @ x on the quantized operands
    g8 = C.decode(out["g8"], "e5m2") * float(out["sg"])
    w8 = C.decode(out["w8t"], "e5m2").T * float(out["sw"])
    x8 = C.decode(out["x8t"], "e5m2").T * float(out["sx"])
    sc_dx = float(np.float32(out["sg"]) * np.float32(out["sw"]))
    assert np.allclose(out["dx"], (C.decode(out["g8"], "e5m2") @ C.decode(out["w8t"], "e5m2").T) * sc_dx)
    assert np.allclose(out["dx"], g8 @ w8, rtol=1e-6, atol=1e-12)
    assert np.allclose(out["dw"], g8.T @ x8, rtol=1e-6, atol=1e-12)
    # and against full precision within E5M2's 2^-3 relative step per operand
    assert np.all(np.abs(out["dx"] - gv @ wv) <= 2 * 2.0 ** -3 * (np.abs(gv) @ np.abs(wv)) + 1e-9)
    assert np.array_equal(out["grad_b"], C.round_to_bf16(gv.sum(0)))


def test_delayed_linear_sequence_and_backward_reuses_forward_steps():
    rng = np.random.default_rng(12)
    m, k, n = 32, 64, 48
    w = _bits(rng.standard_normal((n, k)) * 0.02)
    rx, rw = S.Ring(16, "e4m3"), S.Ring(16, "e4m3")
    rg = S.Ring(16, "e5m2")
    amax_hist = []
    for t in range(6):
        x = _bits(rng.standard_normal((m, k)) * 2.0 ** rng.uniform(-4, 4))
        g = _bits(rng.standard_normal((m, n)) * 1e-3)
        if t == 0:
            rx.seed(C.bf16_bits_to_f64(x).astype(np.float32))
            rw.seed(C.bf16_bits_to_f64(w).astype(np.float32))
            rg.seed(C.bf16_bits_to_f64(g).astype(np.float32))
        sx_before = rx.scale
        fwd = L.forward(x, w, None, "e4m3", rx, rw)
        assert fwd["sx"] == sx_before and rx.scale_used == sx_before
        amax_hist.append(fwd["amax_x"])
        assert rx.scale == np.float32(np.float32(max(amax_hist)) / np.float32(448.0))
        bwd = L.backward(g, x, w, "e5m2", fwd["sx"], fwd["sw"], rg)
        assert bwd["sx"] == fwd["sx"] and bwd["sw"] == fwd["sw"]
        for r in (rx, rw, rg):
            r.advance()


def test_backward_mixed_equals_exact_brute_force():
    """E5M2 g8 times the forward's E4M3 bytes: grad_x = g8 @ w8 and grad_w = g8^T @ x8, each
    scaled by RN32(sg * s_operand), against the exact rational triple loop.  The operands are
    transposed here with numpy, not through the oracle's layout handling."""
    rng = np.random.default_rng(31)
    for m, k, n in ((2, 3, 4), (5, 7, 3), (16, 8, 12)):
        g = _bits(rng.standard_normal((m, n)) * 1e-3)
        x8 = _rand_codes(rng, (m, k), "e4m3")
        w8 = _rand_codes(rng, (n, k), "e4m3")
        sx, sw = np.float32(0.0625), np.float32(1.5e-4)
        out = L.backward_mixed(g, x8, w8, "e5m2", "e4m3", "e4m3", sx, sw)
        g8 = out["g8"]
        exact_dx = _brute(g8, w8, "e5m2", "e4m3", out["sg"], sw, None)
        exact_dw = _brute(np.ascontiguousarray(g8.T), x8, "e5m2", "e4m3", out["sg"], sx, None)
        for ref, abs_, sc, exact in ((out["dx"], out["dx_abs"], out["dx_sc"], exact_dx),
                                     (out["dw"], out["dw_abs"], out["dw_sc"], exact_dw)):
            for i in range(ref.shape[0]):
                for j in range(ref.shape[1]):
                    tol = Fraction(2) ** -45 * Fraction(float(abs_[i, j])) * Fraction(float(sc))
                    assert abs(Fraction(ref[i, j]) - exact[i, j]) <= tol


def test_backward_mixed_with_one_format_is_the_backward():
    """With every operand in the backward's format and x8 / w8 quantized at the forward's
    steps, reusing the bytes gives exactly the backward that re-quantizes x and w
    transposed: same g8, step, ring fold, grad_x, grad_w and grad_b."""
    rng = np.random.default_rng(6)
    m, k, n = 48, 32, 40
    g = _bits(rng.standard_normal((m, n)) * 1e-3)
    x = _bits(rng.standard_normal((m, k)))
    w = _bits(rng.standard_normal((n, k)) * 0.02)
    sx, sw = np.float32(3.0e-3), np.float32(1.1e-4)
    x8, _ = Q.quantize(C.bf16_bits_to_f64(x).astype(np.float32), sx, "e5m2")
    w8, _ = Q.quantize(C.bf16_bits_to_f64(w).astype(np.float32), sw, "e5m2")
    r1, r2 = S.Ring(4, "e5m2"), S.Ring(4, "e5m2")
    gv = C.bf16_bits_to_f64(g).astype(np.float32)
    r1.seed(gv)
    r2.seed(gv)
    ref = L.backward(g, x, w, "e5m2", sx, sw, r1)
    mix = L.backward_mixed(g, x8, w8, "e5m2", "e5m2", "e5m2", sx, sw, r2)
    assert np.array_equal(ref["g8"], mix["g8"]) and ref["sg"] == mix["sg"]
    assert np.array_equal(r1.state.view(np.uint32), r2.state.view(np.uint32))
    for key in ("dx", "dw", "dx_abs", "dw_abs"):
        assert np.array_equal(ref[key], mix[key]), key
    assert np.array_equal(ref["grad_b"], mix["grad_b"])


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_fp8_output_gemm_one_hot_returns_the_codes(fmt):
    """A one-hot A with unit scales copies rows of B into the output: every output is an fp8
    value of B's format, exactly representable in bf16, so quantizing it with step 1 in the
    same format must give back B's codes (signed zeros included) and the amax of those rows."""
    rng = np.random.default_rng(12)
    m, k, n = 9, 16, 24
    b = _rand_codes(rng, (k, n), fmt)
    pick = rng.integers(0, k, size=m)
    a = np.full((m, k), 0x00, np.uint8)  # +0
    one = 0x38 if fmt == "e4m3" else 0x3C  # the code of 1.0
    a[np.arange(m), pick] = one
    ref, s_abs, sc, y_bits, out8, am = G.gemm_fp8_out(a, b, "NN", fmt, fmt, 1.0, 1.0, None, None, fmt, 1.0)
    want = b[pick]
    assert np.array_equal(out8, want)
    assert np.float32(am) == np.float32(np.max(np.abs(C.decode(want, fmt))))
    assert np.array_equal(C.bf16_bits_to_f64(y_bits), C.decode(want, fmt))


def test_fp8_output_gemm_is_the_quantized_bf16_output():
    """The fp8 output is the quantize of the bf16 output at out8_step (any scales, bias)."""
    rng = np.random.default_rng(13)
    a = _rand_codes(rng, (20, 48), "e4m3")
    b = _rand_codes(rng, (48, 32), "e4m3")
    bias = C.f64_to_bf16_bits(rng.standard_normal(32))
    ref, s_abs, sc, y_bits, out8, am = G.gemm_fp8_out(a, b, "NN", "e4m3", "e4m3", 0.02, 0.5, bias, None, "e5m2", 0.37)
    y = C.bf16_bits_to_f64(y_bits)
    assert np.array_equal(y, C.round_to_bf16(ref))
    mult = Q.reciprocal_f32(0.37)
    for i in (0, 7, 19):
        for j in (0, 5, 31):
            prod = np.float32(np.float32(y[i, j]) * mult)
            assert out8[i, j] == C.encode(np.array([prod], np.float64), "e5m2")[0]
    assert np.float32(am) == np.float32(np.max(np.abs(y)))


# --- pre-quantized operands (AstrAI astrai/extension commit log: linear_forward_fp8 accepts a
# pre-quantized w8 in the forward's format, skips the weight quantize and reports amax_w = 0;
# the bias may be fp8 with bias_scale; the backward takes g / x / w as bf16 or fp8 in its
# format, and a pre-quantized g folds no ring, reports amax_g = 0 and is dequantized before
# the bias-gradient sum) ---------------------------------------------------------------------

def _dec(codes, fmt):
    return [[Fraction(C.decode_code(int(c), fmt)) for c in row] for row in np.atleast_2d(codes)]


def test_forward_prequantized_weight_is_the_quantized_path():
    """A weight quantized beforehand at the ring's step gives the same bytes, output and x ring
    as quantizing it inside the forward; the weight's ring is left alone and amax_w is 0."""
    rng = np.random.default_rng(40)
    m, k, n = 24, 48, 40
    x = _bits(rng.standard_normal((m, k)))
    w = _bits(rng.standard_normal((n, k)) * 0.02)
    b = _bits(rng.standard_normal(n) * 0.1)
    wv = C.bf16_bits_to_f64(w).astype(np.float32)
    xv = C.bf16_bits_to_f64(x).astype(np.float32)
    rx1, rw1, rx2, rw2 = S.Ring(4, "e4m3"), S.Ring(4, "e4m3"), S.Ring(4, "e4m3"), S.Ring(4, "e4m3")
    for r in (rx1, rx2):
        r.seed(xv)
    for r in (rw1, rw2):
        r.seed(wv)
    sw = rw1.scale
    w8, _ = Q.quantize(wv, sw, "e4m3")
    rw2_before = rw2.state.copy()
    ref = L.forward(x, w, b, "e4m3", rx1, rw1)
    pre = L.forward(x, None, b, "e4m3", rx2, rw2, w8=w8, w_step=sw)
    assert np.array_equal(ref["y"], pre["y"]) and np.array_equal(ref["s_abs"], pre["s_abs"])
    assert np.array_equal(ref["x8"], pre["x8"]) and np.array_equal(pre["w8"], w8)
    assert pre["sw"] == sw and pre["amax_w"] == 0.0 and ref["amax_w"] > 0.0
    assert np.array_equal(rx1.state.view(np.uint32), rx2.state.view(np.uint32))
    assert np.array_equal(rw2.state.view(np.uint32), rw2_before.view(np.uint32))
    # dynamic scaling: x is measured, the weight keeps the step it came with
    sw_dyn = S.dynamic_scale(wv, "e4m3")
    w8d, _ = Q.quantize(wv, sw_dyn, "e4m3")
    assert np.array_equal(L.forward(x, w, b, "e4m3")["y"],
                          L.forward(x, None, b, "e4m3", w8=w8d, w_step=sw_dyn)["y"])


def test_forward_prequantized_weight_and_fp8_bias_brute_force():
    """y = x8 . w8^T * RN32(sx * w_step) + dec(b8) * bias_scale, exactly (tiny shapes)."""
    rng = np.random.default_rng(41)
    for m, k, n in ((2, 16, 3), (5, 32, 7)):
        x = _bits(rng.standard_normal((m, k)))
        w8 = _rand_codes(rng, (n, k), "e4m3")
        b8 = _rand_codes(rng, (n,), "e4m3")
        w_step, bias_scale = np.float32(0.013), np.float32(0.0371)
        out = L.forward(x, None, b8, "e4m3", w8=w8, w_step=w_step, bias_scale=bias_scale)
        sc = Fraction(float(np.float32(out["sx"]) * w_step))
        xs, ws, bs = _dec(out["x8"], "e4m3"), _dec(w8, "e4m3"), _dec(b8, "e4m3")[0]
        for i in range(m):
            for j in range(n):
                exact = sum(xs[i][p] * ws[j][p] for p in range(k)) * sc + bs[j] * Fraction(float(bias_scale))
                assert abs(Fraction(out["y"][i, j]) - exact) <= abs(exact) * Fraction(2) ** -50 + Fraction(2) ** -80


def test_dynamic_steps_use_each_formats_fp8_max():
    """Closed forms from FP8_MAX = 448 (E4M3) and 57344 (E5M2): planted maxima make every
    dynamic step a power of two, and the planted element encodes as the format's largest
    code.  The backward re-measures g, x and w at E5M2's maximum."""
    rng = np.random.default_rng(42)
    m, k, n = 32, 48, 40
    gv = rng.standard_normal((m, n)) * 1e-3
    xv = rng.standard_normal((m, k))
    wv = rng.standard_normal((n, k)) * 0.02
    gv[3, 5] = -57344.0 * 2.0 ** -10   # amax(g) = 56
    xv[7, 9] = 57344.0 * 2.0 ** -3     # amax(x) = 7168
    wv[11, 2] = 57344.0 * 2.0 ** -12   # amax(w) = 14
    g, x, w = _bits(gv), _bits(xv), _bits(wv)
    bwd = L.backward(g, x, w, "e5m2")
    assert (bwd["sg"], bwd["sx"], bwd["sw"]) == (2.0 ** -10, 2.0 ** -3, 2.0 ** -12)
    assert bwd["g8"][3, 5] == 0xFB and bwd["x8t"][9, 7] == 0x7B and bwd["w8t"][2, 11] == 0x7B
    xf = xv.copy()
    xf[7, 9] = 448.0 * 2.0 ** -2      # amax(x) = 112 in the forward (E4M3)
    wf = wv.copy()
    wf[11, 2] = 448.0 * 2.0 ** -7     # amax(w) = 3.5
    fwd = L.forward(_bits(xf), _bits(wf), None, "e4m3")
    assert (fwd["sx"], fwd["sw"]) == (2.0 ** -2, 2.0 ** -7)
    assert fwd["x8"][7, 9] == 0x7E and fwd["w8"][11, 2] == 0x7E


def test_backward_prequant_all_bf16_is_the_backward():
    rng = np.random.default_rng(43)
    m, k, n = 48, 32, 40
    g = _bits(rng.standard_normal((m, n)) * 1e-3)
    x = _bits(rng.standard_normal((m, k)))
    w = _bits(rng.standard_normal((n, k)) * 0.02)
    for delayed in (False, True):
        r1, r2 = (S.Ring(4, "e5m2"), S.Ring(4, "e5m2")) if delayed else (None, None)
        if delayed:
            for r in (r1, r2):
                r.seed(C.bf16_bits_to_f64(g).astype(np.float32))
        sx, sw = (np.float32(3e-3), np.float32(1.1e-4)) if delayed else (None, None)
        ref = L.backward(g, x, w, "e5m2", sx, sw, r1)
        got = L.backward_prequant(g, x, w, "e5m2", sx=sx, sw=sw, ring_g=r2)
        for key in ("dx", "dw", "dx_abs", "dw_abs", "grad_b", "g8"):
            assert np.array_equal(ref[key], got[key]), key
        assert (ref["sg"], ref["sx"], ref["sw"], ref["amax_g"]) == (got["sg"], got["sx"], got["sw"], got["amax_g"])
        if delayed:
            assert np.array_equal(r1.state.view(np.uint32), r2.state.view(np.uint32))


def test_backward_prequant_operands_skip_their_quantize():
    """Operands quantized beforehand at the same steps give the same grad_x / grad_w; a
    pre-quantized g leaves the ring alone, reports amax_g = 0, and its grad_b is the column
    sum of the dequantized bytes."""
    rng = np.random.default_rng(44)
    m, k, n = 40, 32, 48
    gv = rng.standard_normal((m, n)) * 1e-3
    g, x, w = _bits(gv), _bits(rng.standard_normal((m, k))), _bits(rng.standard_normal((n, k)) * 0.02)
    sx, sw = np.float32(2.5e-3), np.float32(9e-5)
    ring = S.Ring(4, "e5m2")
    ring.seed(C.bf16_bits_to_f64(g).astype(np.float32))
    sg = ring.scale
    ref = L.backward(g, x, w, "e5m2", sx, sw, ring)
    g8, _ = Q.quantize(C.bf16_bits_to_f64(g).astype(np.float32), sg, "e5m2")
    x8, _ = Q.quantize(C.bf16_bits_to_f64(x).astype(np.float32), sx, "e5m2")
    w8, _ = Q.quantize(C.bf16_bits_to_f64(w).astype(np.float32), sw, "e5m2")
    for fl in ((1, 0, 0), (0, 1, 0), (0, 0, 1), (1, 1, 1)):
        ops = [g8 if fl[0] else g, x8 if fl[1] else x, w8 if fl[2] else w]
        r2 = S.Ring(4, "e5m2")
        r2.seed(C.bf16_bits_to_f64(g).astype(np.float32))
        before = r2.state.copy()
        got = L.backward_prequant(*ops, "e5m2", *map(bool, fl), g_step=sg, sx=sx, sw=sw, ring_g=r2)
        assert np.array_equal(ref["dx"], got["dx"]) and np.array_equal(ref["dw"], got["dw"]), fl
        if fl[0]:
            assert got["amax_g"] == 0.0
            assert np.array_equal(r2.state.view(np.uint32), before.view(np.uint32))
            want = C.round_to_bf16((C.decode(g8, "e5m2") * float(sg)).sum(0))
            assert np.array_equal(got["grad_b"], want)
        else:
            assert got["amax_g"] == ref["amax_g"] and np.array_equal(got["grad_b"], ref["grad_b"])
    # closed form: every code 1.0 at step 2^-7 over m rows sums to m * 2^-7 in every column
    ones = np.full((m, n), 0x3C, np.uint8)
    got = L.backward_prequant(ones, x, w, "e5m2", True, False, False, g_step=2.0 ** -7, sx=sx, sw=sw)
    assert np.all(got["grad_b"] == m * 2.0 ** -7)


def test_backward_prequant_equals_exact_brute_force():
    rng = np.random.default_rng(45)
    for m, k, n in ((2, 3, 4), (6, 5, 7)):
        g8 = _rand_codes(rng, (m, n), "e5m2")
        x8 = _rand_codes(rng, (m, k), "e5m2")
        w8 = _rand_codes(rng, (n, k), "e5m2")
        sg, sx, sw = np.float32(3e-5), np.float32(0.07), np.float32(2e-3)
        out = L.backward_prequant(g8, x8, w8, "e5m2", True, True, True, g_step=sg, sx=sx, sw=sw)
        gs, xs, ws = _dec(g8, "e5m2"), _dec(x8, "e5m2"), _dec(w8, "e5m2")
        sc_x = Fraction(float(sg * sw))
        sc_w = Fraction(float(sg * sx))
        for i in range(m):
            for j in range(k):
                exact = sum(gs[i][p] * ws[p][j] for p in range(n)) * sc_x
                assert abs(Fraction(out["dx"][i, j]) - exact) <= Fraction(2) ** -45 * Fraction(float(out["dx_abs"][i, j])) * sc_x
        for i in range(n):
            for j in range(k):
                exact = sum(gs[p][i] * xs[p][j] for p in range(m)) * sc_w
                assert abs(Fraction(out["dw"][i, j]) - exact) <= Fraction(2) ** -45 * Fraction(float(out["dw_abs"][i, j])) * sc_w


def _bf16_bits(rng, shape, sd):
    """bf16 bit patterns of N(0, sd) samples (truncated fp32)."""
    v = (rng.standard_normal(shape) * sd).astype(np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)


def test_empty_batch_follows_the_definition():
    """No rows: amax of nothing is 0 (the ring records 0 and, from a window of zeros, publishes the
    1e-12 floor of the formula), grad_w and grad_b are sums over no rows (0); no output columns:
    grad_x is a sum over no columns (0); no inner dimension: y is the bias."""
    rng = np.random.default_rng(5)
    k, n = 64, 48
    x = np.zeros((0, k), dtype=np.uint16)
    g = np.zeros((0, n), dtype=np.uint16)
    w = _bf16_bits(rng, (n, k), 0.02)
    b = _bf16_bits(rng, (n,), 0.1)
    rx, rw, rg = S.Ring(4, "e4m3"), S.Ring(4, "e4m3"), S.Ring(4, "e5m2")
    rx.seed(np.zeros((0, k), np.float32))
    rw.seed(C.bf16_bits_to_f64(w).astype(np.float32))
    rg.seed(np.zeros((0, n), np.float32))
    assert rx.scale == np.float32(1e-12) and rg.scale == np.float32(1e-12)
    f = L.forward(x, w, b, "e4m3", rx, rw)
    assert f["y"].shape == (0, n) and f["amax_x"] == 0.0
    assert rx.state[0] == 0.0 and rx.state[4] == np.float32(1e-12)  # hist[idx] = 0; the floor
    r = L.backward(g, x, w, "e5m2", f["sx"], f["sw"], rg)
    assert r["dx"].shape == (0, k) and r["dw"].shape == (n, k)
    assert not r["dw"].any() and not r["grad_b"].any() and r["amax_g"] == 0.0
    # no output columns: grad_x = g . w over nothing
    x2 = _bf16_bits(rng, (32, k), 1.0)
    r2 = L.backward(np.zeros((32, 0), np.uint16), x2, np.zeros((0, k), np.uint16), "e5m2", 1.0, 1.0)
    assert r2["dx"].shape == (32, k) and not r2["dx"].any() and r2["dw"].shape == (0, k)
    # no inner dimension: y[i][j] = bias[j]
    f3 = L.forward(np.zeros((32, 0), np.uint16), np.zeros((n, 0), np.uint16), b, "e4m3")
    assert np.array_equal(f3["y"], np.broadcast_to(C.bf16_bits_to_f64(b), (32, n)))

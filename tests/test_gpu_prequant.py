"""GPU parity: the linear entries' pre-quantized and fp8-bias input modes, and the dynamic
backward's choice of FP8_MAX.

* linear_forward_fp8 with ``w_is_fp8 = 1``: the weight arrives as fp8 bytes in the forward's
  format with its step; its quantize is skipped, its ring (if one is passed) is neither read
  nor folded, and ``sw_used`` is that step.  Delayed (x ring) and dynamic, bf16 / fp8 / no
  bias, a training-linear shape and a ragged one.
* an fp8 bias with ``bias_scale`` through linear_forward_fp8 (bf16 weight, delayed rings).
* the dynamic backward measures g, x and w at E5M2's maximum 57344: planted maxima make the
  steps powers of two, and the bytes of every operand (g8, g8T, x8T, w8T, read from the
  workspace at the offsets of its documented layout) equal the oracle's.

Definitions: AstrAI astrai/extension commit log (pre-quantized w8 skips the weight quantize
and reports amax_w = 0; FP8Params.bias with bias_scale: fp8 storage dequantized after the
operand scaling) and the compare view, astrai/extension/fp8.py (fp8_linear_forward,
_LinearFp8.backward with _dynamic_scale at the backward format).
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
from oracle import fp8_codec as C
from oracle import linear as L
from oracle import scaling as S
from helpers import np_u8, np_bf16_bits, bf16_out_to_f64, assert_within_gemm_bound, assert_bf16_within_ulp

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ring(hist_len, fmt):
    st = torch.zeros(hist_len + 4, dtype=torch.float32, device=DEV)
    F.fp8_scale_ring_init(st, hist_len)
    return F.Ring(st, hist_len, fmt)


def _state_bits(r):
    return r.state.detach().cpu().numpy().view(np.uint32)


def _bias(kind, n, seed):
    """(device bias, device bias_scale or None, oracle bias, oracle bias_scale)."""
    if kind == "none":
        return None, None, None, None
    if kind == "bf16":
        b = W.normal_bf16((n,), 0.1, seed=seed)
        return b.to(DEV), None, W.bf16_bits(b), None
    b8 = W.fp8_bytes((n,), seed=seed, fmt="e4m3")
    bs = float(W.uniform(0.01, 0.05, seed=seed + 1)[0])
    return b8.to(DEV), torch.tensor([bs], device=DEV), W.u8(b8), np.float32(bs)


@pytest.mark.parametrize("delayed", [False, True])
@pytest.mark.parametrize("bias_kind", ["none", "bf16", "fp8"])
@pytest.mark.parametrize("mkn", [(2048, 1024, 3072), (300, 272, 400)])
def test_forward_prequantized_weight(delayed, bias_kind, mkn):
    m, k, n = mkn
    x = W.normal_bf16((m, k), 1.0, seed=700 + m)
    w8, s8 = W.amax_scaled_fp8_bytes((n, k), seed=701 + n)
    w_step = np.float32(0.02 * s8)
    bias_d, bs_d, bias_o, bs_o = _bias(bias_kind, n, seed=702)
    xd, w8d = x.to(DEV), w8.to(DEV)
    w_step_d = torch.tensor([float(w_step)], device=DEV)
    xr = wr = oxr = None
    if delayed:
        xr, wr = _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3)
        F.fp8_scale_ring_seed(xr, xd, F.FP8_IN_BF16, xd.numel())
        oxr = S.Ring(16, "e4m3")
        oxr.seed(bf16_out_to_f64(x).astype(np.float32))
        wr_before = _state_bits(wr).copy()
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    sx = torch.zeros(1, device=DEV)
    sw = torch.zeros(1, device=DEV)
    F.linear_forward_fp8(xd, w8d, 1, w_step_d, bias_d, bs_d, m, k, n, F.FP8_E4M3, xr, wr, 1.0, sx, sw, ws, nbytes, y)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    f = L.forward(W.bf16_bits(x), None, bias_o, "e4m3", oxr, None, w8=W.u8(w8), w_step=w_step, bias_scale=bs_o)
    assert f["amax_w"] == 0.0
    assert sx.item() == f["sx"] and sw.item() == f["sw"] == w_step
    assert np.array_equal(np_u8(ws[:m * k]).reshape(m, k), f["x8"])
    if delayed:
        assert np.array_equal(_state_bits(xr), oxr.state.view(np.uint32))
        assert np.array_equal(_state_bits(wr), wr_before), "the pre-quantized weight's ring was touched"
    assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], f"y ({bias_kind})")


def test_forward_fp8_bias_through_linear_delayed():
    """Config 2's shapes over three delayed steps with an fp8 bias dequantized by bias_scale."""
    m, k, n = 512, 1024, 1024
    w = W.normal_bf16((n, k), 0.02, seed=720)
    wd = w.to(DEV)
    b8d, bsd, b8, bs = _bias("fp8", n, seed=721)
    xr, wr = _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3)
    oxr, owr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3")
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    for t, fct in enumerate(W.delayed_sequence_factors(3, seed=5)):
        x = W.delayed_ring_inputs(t, fct, rows=m, cols=k, seed=730)
        xd = x.to(DEV)
        if t == 0:
            F.fp8_scale_ring_seed(xr, xd, F.FP8_IN_BF16, xd.numel())
            F.fp8_scale_ring_seed(wr, wd, F.FP8_IN_BF16, wd.numel())
            oxr.seed(bf16_out_to_f64(x).astype(np.float32))
            owr.seed(bf16_out_to_f64(w).astype(np.float32))
        y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
        sx = torch.zeros(1, device=DEV)
        sw = torch.zeros(1, device=DEV)
        F.linear_forward_fp8(xd, wd, 0, None, b8d, bsd, m, k, n, F.FP8_E4M3, xr, wr, 1.0, sx, sw, ws, nbytes, y)
        torch.cuda.synchronize()
        f = L.forward(W.bf16_bits(x), W.bf16_bits(w), b8, "e4m3", oxr, owr, bias_scale=bs)
        assert (sx.item(), sw.item()) == (f["sx"], f["sw"]), t
        assert np.array_equal(_state_bits(xr), oxr.state.view(np.uint32)), t
        assert np.array_equal(_state_bits(wr), owr.state.view(np.uint32)), t
        assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], f"y step {t}")
        for r in (xr, wr, oxr, owr):
            r.advance()
    assert F.fp8_get_device_status() == 0


def _align(v, a=256):
    return (v + a - 1) // a * a


def test_dynamic_backward_measures_at_e5m2_max():
    """Planted maxima: amax(g) = 57344 * 2^-10, amax(x) = 57344 * 2^-3, amax(w) = 57344 * 2^-12,
    so the E5M2 steps are 2^-10, 2^-3 and 2^-12 exactly (448 would give 2^-3, 2^4 and 2^-5).
    The workspace holds g8 | g8T | x8T | w8T at 256-byte aligned offsets."""
    t = W.tiny_linear(3)
    g, x, w = t["g"].clone(), t["x"].clone(), t["w"].clone()
    g[3, 5] = -57344.0 * 2.0 ** -10
    x[7, 9] = 57344.0 * 2.0 ** -3
    w[11, 2] = 57344.0 * 2.0 ** -12
    m, k = x.shape
    n = w.shape[0]
    gd, xd, wd = g.to(DEV), x.to(DEV), w.to(DEV)
    nbytes = F.linear_backward_fp8_workspace_size(m, k, n)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    gx = torch.empty((m, k), dtype=torch.bfloat16, device=DEV)
    gw = torch.empty((n, k), dtype=torch.bfloat16, device=DEV)
    gb = torch.empty((n,), dtype=torch.bfloat16, device=DEV)
    sg = torch.zeros(1, device=DEV)
    F.linear_backward_fp8(gd, xd, wd, m, k, n, F.FP8_E5M2, 1, 1, 1, None, None, None, 1.0, sg, ws, nbytes, gx, gw, gb)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    assert sg.item() == 2.0 ** -10
    r = L.backward(W.bf16_bits(g), W.bf16_bits(x), W.bf16_bits(w), "e5m2")
    assert (r["sg"], r["sx"], r["sw"]) == (2.0 ** -10, 2.0 ** -3, 2.0 ** -12)
    o_g8t = _align(m * n)
    o_x8t = _align(o_g8t + m * n)
    o_w8t = _align(o_x8t + k * m)
    host = np_u8(ws)
    assert np.array_equal(host[:m * n].reshape(m, n), r["g8"])
    assert np.array_equal(host[o_g8t:o_g8t + m * n].reshape(n, m), r["g8t"])
    assert np.array_equal(host[o_x8t:o_x8t + k * m].reshape(k, m), r["x8t"])
    assert np.array_equal(host[o_w8t:o_w8t + k * n].reshape(k, n), r["w8t"])
    assert r["x8t"][9, 7] == 0x7B and r["w8t"][2, 11] == 0x7B and r["g8"][3, 5] == 0xFB
    assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
    assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")


# --- the backward with pre-quantized operands ------------------------------------------------

FLAGS = [(0, 0, 0), (1, 0, 0), (0, 1, 0), (0, 0, 1), (1, 1, 1)]


def _operand(shape, std, seed, fp8):
    """bf16 N(0, std^2), or E5M2 codes of N(0,1) samples whose step is std (so the values
    carry the same spread)."""
    if fp8:
        return W.fp8_bytes(shape, seed=seed, fmt="e5m2"), np.float32(std)
    return W.normal_bf16(shape, std, seed=seed), None


def _backward_prequant(mkn, flags, delayed, seed):
    m, k, n = mkn
    gf, xf, wf = flags
    g, g_step = _operand((m, n), 1e-3, seed, gf)
    x, _ = _operand((m, k), 1.0, seed + 1, xf)
    w, _ = _operand((n, k), 0.02, seed + 2, wf)
    sx, sw = np.float32(0.75 / 448), np.float32(0.02 * 3.5 / 448)  # the forward's steps
    if xf:
        sx = np.float32(1.0)
    if wf:
        sw = np.float32(0.02)
    gd, xd, wd = g.to(DEV), x.to(DEV), w.to(DEV)
    gr = ogr = None
    if delayed:
        gr = _ring(16, F.FP8_E5M2)
        ogr = S.Ring(16, "e5m2")
        seed_g = W.normal_bf16((m, n), 1e-3, seed=seed + 9)
        F.fp8_scale_ring_seed(gr, seed_g.to(DEV), F.FP8_IN_BF16, seed_g.numel())
        ogr.seed(bf16_out_to_f64(seed_g).astype(np.float32))
        before = _state_bits(gr).copy()
    pre = lambda v: None if v is None else torch.tensor([float(v)], device=DEV)  # noqa: E731
    # delayed: the forward's steps; dynamic: only the pre-quantized operands carry a step
    sxd = pre(sx) if (delayed or xf) else None
    swd = pre(sw) if (delayed or wf) else None
    nbytes = F.linear_backward_fp8_workspace_size(m, k, n)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    gx = torch.empty((m, k), dtype=torch.bfloat16, device=DEV)
    gw = torch.empty((n, k), dtype=torch.bfloat16, device=DEV)
    gb = torch.empty((n,), dtype=torch.bfloat16, device=DEV)
    sg = torch.zeros(1, device=DEV)
    F.linear_backward_fp8_prequant(gd, gf, pre(g_step), xd, xf, wd, wf, m, k, n, F.FP8_E5M2, 1, 1, 1, sxd, swd, gr, 1.0,
                                   sg, ws, nbytes, gx, gw, gb)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    conv = lambda t, f: W.u8(t) if f else W.bf16_bits(t)  # noqa: E731
    r = L.backward_prequant(conv(g, gf), conv(x, xf), conv(w, wf), "e5m2", bool(gf), bool(xf), bool(wf),
                            g_step=g_step, sx=sx if (delayed or xf) else None, sw=sw if (delayed or wf) else None,
                            ring_g=ogr)
    assert sg.item() == r["sg"]
    if delayed:
        if gf:
            assert np.array_equal(_state_bits(gr), before), "a pre-quantized g must leave its ring alone"
            assert r["amax_g"] == 0.0
        else:
            assert np.array_equal(_state_bits(gr), ogr.state.view(np.uint32))
    assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], f"dX {flags}")
    assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], f"dW {flags}")
    gsum = (C.decode(W.u8(g), "e5m2") * float(g_step)).sum(0) if gf else bf16_out_to_f64(g).sum(0)
    assert_bf16_within_ulp(np_bf16_bits(gb), gsum, 1, f"grad_b {flags}")
    assert np.array_equal(r["grad_b"], C.round_to_bf16(gsum))


@pytest.mark.parametrize("flags", FLAGS)
@pytest.mark.parametrize("mkn", [(2048, 1024, 3072), (2048, 4096, 1024), (304, 272, 400)])
def test_backward_prequant_delayed_hybrid(mkn, flags):
    _backward_prequant(mkn, flags, True, seed=800 + sum(mkn))


@pytest.mark.parametrize("flags", FLAGS)
def test_backward_prequant_dynamic_tiny(flags):
    _backward_prequant((128, 256, 256), flags, False, seed=850)

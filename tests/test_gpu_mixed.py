"""GPU parity: the mixed-format backward that reuses the forward's quantized operands.

linear_forward_fp8_keep leaves x8 / w8 (E4M3) in caller buffers; linear_backward_fp8_mixed
quantizes only g (E5M2, row-major, ring fold, column sums) and reads x8 / w8 in place.  Against
the oracle's ``forward`` and ``backward_mixed``: kept bytes, steps and ring states bit-exact;
grad_x / grad_w within the GEMM bound; grad_b within one bf16 ulp.

Definitions: AstrAI compare view, astrai/extension/fp8.py (fp8_linear_forward,
_LinearFp8.backward) and the linear backward binding in an earlier state (operands the forward
already quantized are reused); the independent operand formats are this library's reading.
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
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


def _forward_keep(x, w, b, xr=None, wr=None):
    m, k = x.shape
    n = w.shape[0]
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = torch.full((nbytes,), 0x3C, dtype=torch.uint8, device=DEV)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    x8 = torch.empty((m, k), dtype=torch.uint8, device=DEV)
    w8 = torch.empty((n, k), dtype=torch.uint8, device=DEV)
    sx, sw = torch.zeros(1, device=DEV), torch.zeros(1, device=DEV)
    F.linear_forward_fp8_keep(x, w, 0, None, b, None, m, k, n, F.FP8_E4M3, xr, wr, 1.0, sx, sw, x8, w8, ws, nbytes, y)
    return y, x8, w8, sx, sw


def _backward_mixed(g, x8, w8, sx, sw, gr=None, need=(1, 1, 1)):
    m, n = g.shape
    k = x8.shape[1]
    nbytes = F.linear_backward_fp8_mixed_workspace_size(m, k, n)
    ws = torch.full((nbytes,), 0xC3, dtype=torch.uint8, device=DEV)
    gx = torch.full((m, k), float("nan"), dtype=torch.bfloat16, device=DEV)
    gw = torch.full((n, k), float("nan"), dtype=torch.bfloat16, device=DEV)
    gb = torch.full((n,), float("nan"), dtype=torch.bfloat16, device=DEV)
    sg = torch.zeros(1, device=DEV)
    F.linear_backward_fp8_mixed(g, x8, w8, m, k, n, F.FP8_E5M2, F.FP8_E4M3, F.FP8_E4M3, need[0], need[1], need[2],
                                sx, sw, gr, 1.0, sg, ws, nbytes, gx, gw, gb)
    return gx, gw, gb, sg


@pytest.mark.parametrize("kn", W.TRAINING_LINEARS)
def test_training_linear_mixed_backward_delayed(kn, tiled_path):
    k, n = kn
    m = W.TRAINING_TOKENS
    xr, wr, gr = _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E5M2)
    oxr, owr, ogr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3"), S.Ring(16, "e5m2")
    for step in range(2):
        t = W.training_linear(m, k, n, seed=3000 + 10 * step + k + n)
        x, w, b, g = (t[key].to(DEV) for key in ("x", "w", "b", "g"))
        xb, wb, bb, gbits = (W.bf16_bits(t[key]) for key in ("x", "w", "b", "g"))
        if step == 0:
            for dr, orr, v, key in ((xr, oxr, x, "x"), (wr, owr, w, "w"), (gr, ogr, g, "g")):
                F.fp8_scale_ring_seed(dr, v, F.FP8_IN_BF16, v.numel())
                orr.seed(bf16_out_to_f64(t[key]).astype(np.float32))
        y, x8, w8, sx, sw = _forward_keep(x, w, b, xr, wr)
        gx, gw, gbias, sg = _backward_mixed(g, x8, w8, sx, sw, gr)
        torch.cuda.synchronize()
        assert F.fp8_get_device_status() == 0
        f = L.forward(xb, wb, bb, "e4m3", oxr, owr)
        r = L.backward_mixed(gbits, f["x8"], f["w8"], "e5m2", "e4m3", "e4m3", f["sx"], f["sw"], ogr)
        assert np.array_equal(np_u8(x8), f["x8"]) and np.array_equal(np_u8(w8), f["w8"])
        assert (sx.item(), sw.item(), sg.item()) == (f["sx"], f["sw"], r["sg"])
        for dev_r, ora_r in ((xr, oxr), (wr, owr), (gr, ogr)):
            assert np.array_equal(_state_bits(dev_r), ora_r.state.view(np.uint32))
        assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], "y")
        assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX mixed")
        assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW mixed")
        assert_bf16_within_ulp(np_bf16_bits(gbias), np.sum(bf16_out_to_f64(t["g"]), axis=0), 1, "grad_b")
        for rr in (xr, wr, gr, oxr, owr, ogr):
            rr.advance()


@pytest.mark.parametrize("need", [(1, 1, 1), (1, 0, 0), (0, 1, 0), (1, 1, 0)])
def test_tiny_linear_mixed_backward_dynamic(need):
    """Dynamic scaling (no rings), ragged M, every subset of outputs: without grad_b, g is
    quantized by the row-major kernel instead of the tiled one."""
    m, k, n = 200, 256, 272
    t = W.training_linear(m, k, n, seed=77)
    x, w, b, g = (t[key].to(DEV) for key in ("x", "w", "b", "g"))
    xb, wb, bb, gbits = (W.bf16_bits(t[key]) for key in ("x", "w", "b", "g"))
    y, x8, w8, sx, sw = _forward_keep(x, w, b)
    gx, gw, gbias, sg = _backward_mixed(g, x8, w8, sx, sw, None, need)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    f = L.forward(xb, wb, bb, "e4m3")
    r = L.backward_mixed(gbits, f["x8"], f["w8"], "e5m2", "e4m3", "e4m3", f["sx"], f["sw"])
    assert sg.item() == r["sg"]
    if need[0]:
        assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
    else:
        assert torch.isnan(gx.float()).all()
    if need[1]:
        assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")
    else:
        assert torch.isnan(gw.float()).all()
    if need[2]:
        assert_bf16_within_ulp(np_bf16_bits(gbias), np.sum(bf16_out_to_f64(t["g"]), axis=0), 1, "grad_b")
    else:
        assert torch.isnan(gbias.float()).all()


def test_mixed_backward_with_one_format_matches_backward():
    """All operands E5M2: the kept bytes re-read by the mixed backward and the re-quantizing
    backward both stay within the bound of the same oracle result."""
    m, k, n = 512, 384, 640
    t = W.training_linear(m, k, n, seed=91)
    x, w, b, g = (t[key].to(DEV) for key in ("x", "w", "b", "g"))
    xb, wb, bb, gbits = (W.bf16_bits(t[key]) for key in ("x", "w", "b", "g"))
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    x8 = torch.empty((m, k), dtype=torch.uint8, device=DEV)
    w8 = torch.empty((n, k), dtype=torch.uint8, device=DEV)
    sx, sw = torch.zeros(1, device=DEV), torch.zeros(1, device=DEV)
    F.linear_forward_fp8_keep(x, w, 0, None, b, None, m, k, n, F.FP8_E5M2, None, None, 1.0, sx, sw, x8, w8, ws,
                              nbytes, y)
    nb = F.linear_backward_fp8_mixed_workspace_size(m, k, n)
    wsm = torch.empty(nb, dtype=torch.uint8, device=DEV)
    gx = torch.empty((m, k), dtype=torch.bfloat16, device=DEV)
    gw = torch.empty((n, k), dtype=torch.bfloat16, device=DEV)
    gb = torch.empty((n,), dtype=torch.bfloat16, device=DEV)
    F.linear_backward_fp8_mixed(g, x8, w8, m, k, n, F.FP8_E5M2, F.FP8_E5M2, F.FP8_E5M2, 1, 1, 1, sx, sw, None,
                                1.0, None, wsm, nb, gx, gw, gb)
    torch.cuda.synchronize()
    f = L.forward(xb, wb, bb, "e5m2")
    r = L.backward_mixed(gbits, f["x8"], f["w8"], "e5m2", "e5m2", "e5m2", f["sx"], f["sw"])
    assert np.array_equal(np_u8(x8), f["x8"]) and np.array_equal(np_u8(w8), f["w8"])
    assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
    assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")
    assert F.fp8_get_device_status() == 0

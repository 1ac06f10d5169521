"""GPU parity: linear_forward_fp8 / linear_backward_fp8 against the oracle's compositions.

* tiny linear (x [128,256], w [256,256], dynamic scaling): steps exact, fp8 operands exact,
  y / dX / dW within the GEMM bound, grad_b within one bf16 ulp;
* delayed ring over 8 steps (x [512,1024] * s_t, w [1024,1024]): ring states exact each step;
* training linears (M = 2048, HYBRID, delayed history 16, bias): rings, steps and bytes exact,
  y / dX / dW within the bound.

Definitions: AstrAI compare view, astrai/extension/fp8.py -- fp8_linear_forward and
_LinearFp8.backward.
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


def _ws(nbytes):
    return torch.empty(nbytes, dtype=torch.uint8, device=DEV)


def _ring(hist_len, fmt):
    st = torch.zeros(hist_len + 4, dtype=torch.float32, device=DEV)
    F.fp8_scale_ring_init(st, hist_len)
    return F.Ring(st, hist_len, fmt)


def _fwd(x, w, b, fmt, xr=None, wr=None):
    m, k = x.shape
    n = w.shape[0]
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = _ws(nbytes)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    sx = torch.zeros(1, device=DEV)
    sw = torch.zeros(1, device=DEV)
    F.linear_forward_fp8(x, w, 0, None, b, None, m, k, n, fmt, xr, wr, 1.0, sx, sw, ws, nbytes, y)
    return y, sx, sw, ws


def _bwd(g, x, w, fmt, sx=None, sw=None, gr=None):
    m, n = g.shape
    k = x.shape[1]
    nbytes = F.linear_backward_fp8_workspace_size(m, k, n)
    ws = _ws(nbytes)
    gx = torch.empty((m, k), dtype=torch.bfloat16, device=DEV)
    gw = torch.empty((n, k), dtype=torch.bfloat16, device=DEV)
    gb = torch.empty((n,), dtype=torch.bfloat16, device=DEV)
    sg = torch.zeros(1, device=DEV)
    F.linear_backward_fp8(g, x, w, m, k, n, fmt, 1, 1, 1, sx, sw, gr, 1.0, sg, ws, nbytes, gx, gw, gb)
    return gx, gw, gb, sg, ws


def test_tiny_linear_dynamic_fwd_bwd():
    t = W.tiny_linear(0)
    x, w, b, g = (t[k].to(DEV) for k in ("x", "w", "b", "g"))
    y, sx, sw, ws = _fwd(x, w, b, F.FP8_E4M3)
    gx, gw, gb, sg, wsb = _bwd(g, x, w, F.FP8_E5M2)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    xb, wb, bb, gbits = (W.bf16_bits(t[k]) for k in ("x", "w", "b", "g"))
    f = L.forward(xb, wb, bb, "e4m3")
    assert sx.item() == f["sx"] and sw.item() == f["sw"]
    m, k = t["x"].shape
    n = t["w"].shape[0]
    assert np.array_equal(np_u8(ws[:m * k]).reshape(m, k), f["x8"])
    w8_off = (m * k + 255) // 256 * 256
    assert np.array_equal(np_u8(ws[w8_off:w8_off + n * k]).reshape(n, k), f["w8"])
    assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], "y")
    r = L.backward(gbits, xb, wb, "e5m2")
    assert sg.item() == r["sg"]
    assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
    assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")
    assert_bf16_within_ulp(np_bf16_bits(gb), np.sum(bf16_out_to_f64(t["g"]), axis=0), 1, "grad_b")


def _state_bits(r):
    return r.state.detach().cpu().numpy().view(np.uint32)


def test_delayed_ring_forward_eight_steps():
    factors = W.delayed_sequence_factors(8, seed=0)
    w = W.normal_bf16((1024, 1024), 0.02, seed=200)
    b = W.normal_bf16((1024,), 0.1, seed=201)
    xr, wr = _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3)
    oxr, owr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3")
    wd, bd = w.to(DEV), b.to(DEV)
    for t, fct in enumerate(factors):
        x = W.delayed_ring_inputs(t, fct)
        xd = x.to(DEV)
        if t == 0:
            F.fp8_scale_ring_seed(xr, xd, F.FP8_IN_BF16, xd.numel())
            F.fp8_scale_ring_seed(wr, wd, F.FP8_IN_BF16, wd.numel())
            oxr.seed(bf16_out_to_f64(x).astype(np.float32))
            owr.seed(bf16_out_to_f64(w).astype(np.float32))
        y, sx, sw, ws = _fwd(xd, wd, bd, F.FP8_E4M3, xr, wr)
        torch.cuda.synchronize()
        f = L.forward(W.bf16_bits(x), W.bf16_bits(w), W.bf16_bits(b), "e4m3", oxr, owr)
        assert sx.item() == f["sx"] and sw.item() == f["sw"], t
        assert np.array_equal(_state_bits(xr), oxr.state.view(np.uint32)), t
        assert np.array_equal(_state_bits(wr), owr.state.view(np.uint32)), t
        assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], f"y step {t}")
        for r in (xr, wr, oxr, owr):
            r.advance()


@pytest.mark.parametrize("kn", W.TRAINING_LINEARS)
def test_training_linear_delayed_hybrid(kn, tiled_path):
    k, n = kn
    m = W.TRAINING_TOKENS
    xr, wr = _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3)
    gr = _ring(16, F.FP8_E5M2)
    oxr, owr, ogr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3"), S.Ring(16, "e5m2")
    steps = 2 if kn == W.TRAINING_LINEARS[0] else 1
    for step in range(steps):
        t = W.training_linear(m, k, n, seed=1000 + 10 * step + k + n)
        x, w, b, g = (t[key].to(DEV) for key in ("x", "w", "b", "g"))
        xb, wb, bb, gb_bits = (W.bf16_bits(t[key]) for key in ("x", "w", "b", "g"))
        if step == 0:
            F.fp8_scale_ring_seed(xr, x, F.FP8_IN_BF16, x.numel())
            F.fp8_scale_ring_seed(wr, w, F.FP8_IN_BF16, w.numel())
            F.fp8_scale_ring_seed(gr, g, F.FP8_IN_BF16, g.numel())
            oxr.seed(bf16_out_to_f64(t["x"]).astype(np.float32))
            owr.seed(bf16_out_to_f64(t["w"]).astype(np.float32))
            ogr.seed(bf16_out_to_f64(t["g"]).astype(np.float32))
        y, sx, sw, _ = _fwd(x, w, b, F.FP8_E4M3, xr, wr)
        gx, gw, gbias, sg, _ = _bwd(g, x, w, F.FP8_E5M2, sx, sw, gr)
        torch.cuda.synchronize()
        assert F.fp8_get_device_status() == 0
        f = L.forward(xb, wb, bb, "e4m3", oxr, owr)
        r = L.backward(gb_bits, xb, wb, "e5m2", f["sx"], f["sw"], ogr)
        assert (sx.item(), sw.item(), sg.item()) == (f["sx"], f["sw"], r["sg"])
        for dev_r, ora_r in ((xr, oxr), (wr, owr), (gr, ogr)):
            assert np.array_equal(_state_bits(dev_r), ora_r.state.view(np.uint32))
        assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], "y")
        assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
        assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")
        assert_bf16_within_ulp(np_bf16_bits(gbias), np.sum(bf16_out_to_f64(t["g"]), axis=0), 1, "grad_b")
        for rr in (xr, wr, gr, oxr, owr, ogr):
            rr.advance()


def test_bounded_wait_reports_status_instead_of_hanging():
    F.fp8_set_wait_timeout_ns(50_000_000)  # 50 ms
    try:
        F.fp8_debug_stalled_wait()
        status = F.fp8_get_device_status()
        assert status == 0x1FF
        assert F.fp8_get_device_status() == 0  # reading clears it
        # the context is still usable afterwards
        x = torch.ones(64, device=DEV)
        assert float(x.sum()) == 64.0
    finally:
        F.fp8_set_wait_timeout_ns(2_000_000_000)

"""GPU parity: the backward's transposed operands formed by the forward's quantize launch.

linear_forward_fp8_save_t quantizes x and w once, writing the forward's row-major bytes (E4M3)
and the backward's transposed bytes (E5M2, same steps) from the same products;
linear_backward_fp8_saved_t then quantizes only g.  Against the oracle's ``forward`` and
``backward`` (which re-quantizes x^T and w^T in the backward, as the pages do): the saved bytes,
steps and ring states bit-exact, y / grad_x / grad_w within the GEMM bound, grad_b within one
bf16 ulp; and against the library's own re-quantizing pair, every output bit-identical.

Definitions: AstrAI compare view, astrai/extension/fp8.py (fp8_linear_forward,
_LinearFp8.backward: x and w re-quantized transposed with the forward's steps and no ring).
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


def _forward_save(x, w, b, xr, wr, fmt_t=F.FP8_E5M2):
    m, k = x.shape
    n = w.shape[0]
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = torch.full((nbytes,), 0x3C, dtype=torch.uint8, device=DEV)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    x8t = torch.full((k, m), 0xA5, dtype=torch.uint8, device=DEV)
    w8t = torch.full((k, n), 0xA5, dtype=torch.uint8, device=DEV)
    sx, sw = torch.zeros(1, device=DEV), torch.zeros(1, device=DEV)
    F.linear_forward_fp8_save_t(x, w, b, None, m, k, n, F.FP8_E4M3, fmt_t, xr, wr, sx, sw, x8t, w8t, ws, nbytes, y)
    return y, x8t, w8t, sx, sw


def _backward_saved(g, x8t, w8t, sx, sw, gr, need=(1, 1, 1), fmt_t=F.FP8_E5M2):
    m, n = g.shape
    k = x8t.shape[0]
    nbytes = F.linear_backward_fp8_saved_t_workspace_size(m, k, n)
    ws = torch.full((nbytes,), 0xC3, dtype=torch.uint8, device=DEV)
    gx = torch.full((m, k), float("nan"), dtype=torch.bfloat16, device=DEV)
    gw = torch.full((n, k), float("nan"), dtype=torch.bfloat16, device=DEV)
    gb = torch.full((n,), float("nan"), dtype=torch.bfloat16, device=DEV)
    sg = torch.zeros(1, device=DEV)
    F.linear_backward_fp8_saved_t(g, x8t, w8t, m, k, n, F.FP8_E5M2, fmt_t, need[0], need[1], need[2], sx, sw, gr,
                                  1.0, sg, ws, nbytes, gx, gw, gb)
    return gx, gw, gb, sg


def _tensors(m, k, n, seed):
    t = W.training_linear(m, k, n, seed=seed)
    dev = {key: t[key].to(DEV) for key in ("x", "w", "b", "g")}
    bits = {key: W.bf16_bits(t[key]) for key in ("x", "w", "b", "g")}
    return t, dev, bits


@pytest.mark.parametrize("kn", W.TRAINING_LINEARS)
def test_training_linear_saved_transposes_delayed(kn, tiled_path):
    k, n = kn
    m = W.TRAINING_TOKENS
    xr, wr, gr = _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E5M2)
    oxr, owr, ogr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3"), S.Ring(16, "e5m2")
    for step in range(2):
        t, d, bits = _tensors(m, k, n, 5000 + 10 * step + k + n)
        if step == 0:
            for dr, orr, key in ((xr, oxr, "x"), (wr, owr, "w"), (gr, ogr, "g")):
                F.fp8_scale_ring_seed(dr, d[key], F.FP8_IN_BF16, d[key].numel())
                orr.seed(bf16_out_to_f64(t[key]).astype(np.float32))
        y, x8t, w8t, sx, sw = _forward_save(d["x"], d["w"], d["b"], xr, wr)
        gx, gw, gbias, sg = _backward_saved(d["g"], x8t, w8t, sx, sw, gr)
        torch.cuda.synchronize()
        assert F.fp8_get_device_status() == 0
        f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3", oxr, owr)
        r = L.backward(bits["g"], bits["x"], bits["w"], "e5m2", f["sx"], f["sw"], ogr)
        assert np.array_equal(np_u8(x8t), r["x8t"]) and np.array_equal(np_u8(w8t), r["w8t"])
        assert (sx.item(), sw.item(), sg.item()) == (f["sx"], f["sw"], r["sg"])
        for dev_r, ora_r in ((xr, oxr), (wr, owr), (gr, ogr)):
            assert np.array_equal(_state_bits(dev_r), ora_r.state.view(np.uint32))
        assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], "y")
        assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
        assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")
        assert_bf16_within_ulp(np_bf16_bits(gbias), np.sum(bf16_out_to_f64(t["g"]), axis=0), 1, "grad_b")
        for rr in (xr, wr, gr, oxr, owr, ogr):
            rr.advance()


@pytest.mark.parametrize("mkn", [(208, 256, 272), (512, 384, 640)])
def test_saved_pair_equals_requantizing_pair(mkn, tiled_path):
    """Ragged tiles: the saved-transpose pair and linear_forward_fp8 + linear_backward_fp8 from
    equal ring states give bit-identical y, grad_x, grad_w, grad_b, steps and rings."""
    m, k, n = mkn
    _, d, _ = _tensors(m, k, n, 6100 + m)
    rings = []
    for _ in range(2):
        rs = (_ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E5M2))
        for rr, key in zip(rs, ("x", "w", "g")):
            F.fp8_scale_ring_seed(rr, d[key], F.FP8_IN_BF16, d[key].numel())
        rings.append(rs)
    (xr, wr, gr), (xr2, wr2, gr2) = rings
    y, x8t, w8t, sx, sw = _forward_save(d["x"], d["w"], d["b"], xr, wr)
    gx, gw, gb, sg = _backward_saved(d["g"], x8t, w8t, sx, sw, gr)
    nf = F.linear_forward_fp8_workspace_size(m, k, n)
    nb = F.linear_backward_fp8_workspace_size(m, k, n)
    wsf, wsb = (torch.empty(v, dtype=torch.uint8, device=DEV) for v in (nf, nb))
    y2 = torch.empty_like(y)
    gx2, gw2, gb2 = torch.empty_like(gx), torch.empty_like(gw), torch.empty_like(gb)
    steps2 = torch.zeros(3, device=DEV)
    F.linear_forward_fp8(d["x"], d["w"], 0, None, d["b"], None, m, k, n, F.FP8_E4M3, xr2, wr2, 1.0, steps2[0:1],
                         steps2[1:2], wsf, nf, y2)
    F.linear_backward_fp8(d["g"], d["x"], d["w"], m, k, n, F.FP8_E5M2, 1, 1, 1, steps2[0:1], steps2[1:2], gr2, 1.0,
                          steps2[2:3], wsb, nb, gx2, gw2, gb2)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    for a, b in ((y, y2), (gx, gx2), (gw, gw2), (gb, gb2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(torch.cat([sx, sw, sg]), steps2)
    for a, b in zip((xr, wr, gr), (xr2, wr2, gr2)):
        assert np.array_equal(_state_bits(a), _state_bits(b))


@pytest.mark.parametrize("need", [(1, 0, 0), (0, 1, 0), (1, 1, 0), (0, 0, 1)])
def test_saved_backward_output_subsets(need):
    m, k, n = 256, 128, 384
    t, d, bits = _tensors(m, k, n, 77)
    xr, wr, gr = _ring(4, F.FP8_E4M3), _ring(4, F.FP8_E4M3), _ring(4, F.FP8_E5M2)
    oxr, owr, ogr = S.Ring(4, "e4m3"), S.Ring(4, "e4m3"), S.Ring(4, "e5m2")
    for dr, orr, key in ((xr, oxr, "x"), (wr, owr, "w"), (gr, ogr, "g")):
        F.fp8_scale_ring_seed(dr, d[key], F.FP8_IN_BF16, d[key].numel())
        orr.seed(bf16_out_to_f64(t[key]).astype(np.float32))
    y, x8t, w8t, sx, sw = _forward_save(d["x"], d["w"], d["b"], xr, wr)
    gx, gw, gbias, sg = _backward_saved(d["g"], x8t, w8t, sx, sw, gr, need)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3", oxr, owr)
    r = L.backward(bits["g"], bits["x"], bits["w"], "e5m2", f["sx"], f["sw"], ogr)
    assert sg.item() == r["sg"]
    assert np.array_equal(_state_bits(gr), ogr.state.view(np.uint32))
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


def test_saved_transposes_in_the_forward_format_match_the_mixed_backward():
    """fmt_t = E4M3: the saved transposes are the forward's own bytes transposed, so the
    backward computes what the mixed-format backward does (oracle ``backward_mixed``)."""
    m, k, n = 512, 256, 384
    t, d, bits = _tensors(m, k, n, 91)
    xr, wr, gr = _ring(8, F.FP8_E4M3), _ring(8, F.FP8_E4M3), _ring(8, F.FP8_E5M2)
    oxr, owr, ogr = S.Ring(8, "e4m3"), S.Ring(8, "e4m3"), S.Ring(8, "e5m2")
    for dr, orr, key in ((xr, oxr, "x"), (wr, owr, "w"), (gr, ogr, "g")):
        F.fp8_scale_ring_seed(dr, d[key], F.FP8_IN_BF16, d[key].numel())
        orr.seed(bf16_out_to_f64(t[key]).astype(np.float32))
    y, x8t, w8t, sx, sw = _forward_save(d["x"], d["w"], d["b"], xr, wr, fmt_t=F.FP8_E4M3)
    gx, gw, gbias, sg = _backward_saved(d["g"], x8t, w8t, sx, sw, gr, fmt_t=F.FP8_E4M3)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3", oxr, owr)
    assert np.array_equal(np_u8(x8t), f["x8"].T) and np.array_equal(np_u8(w8t), f["w8"].T)
    r = L.backward_mixed(bits["g"], f["x8"], f["w8"], "e5m2", "e4m3", "e4m3", f["sx"], f["sw"], ogr)
    assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
    assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")


# --- the backward's copies saved row-major: linear_forward_fp8_save_rm + linear_backward_fp8_mixed
# with every operand in the backward's format (the pages' HYBRID backward, read in place) ---------

def _forward_save_rm(x, w, b, xr, wr, fmt_b=F.FP8_E5M2):
    m, k = x.shape
    n = w.shape[0]
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = torch.full((nbytes,), 0x3C, dtype=torch.uint8, device=DEV)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    x8b = torch.full((m, k), 0xA5, dtype=torch.uint8, device=DEV)
    w8b = torch.full((n, k), 0xA5, dtype=torch.uint8, device=DEV)
    sx, sw = torch.zeros(1, device=DEV), torch.zeros(1, device=DEV)
    F.linear_forward_fp8_save_rm(x, w, b, None, m, k, n, F.FP8_E4M3, fmt_b, xr, wr, sx, sw, x8b, w8b, ws, nbytes, y)
    return y, x8b, w8b, sx, sw


def _backward_rm(g, x8b, w8b, sx, sw, gr, need=(1, 1, 1), fmt_b=F.FP8_E5M2):
    # outputs pre-filled with a finite sentinel (the saved-transpose helper uses NaN), so an
    # output that neither composition writes cannot compare equal
    m, n = g.shape
    k = x8b.shape[1]
    nbytes = F.linear_backward_fp8_mixed_workspace_size(m, k, n)
    ws = torch.full((nbytes,), 0xC3, dtype=torch.uint8, device=DEV)
    gx = torch.full((m, k), -1234.5, dtype=torch.bfloat16, device=DEV)
    gw = torch.full((n, k), -1234.5, dtype=torch.bfloat16, device=DEV)
    gb = torch.full((n,), -1234.5, dtype=torch.bfloat16, device=DEV)
    sg = torch.zeros(1, device=DEV)
    F.linear_backward_fp8_mixed(g, x8b, w8b, m, k, n, F.FP8_E5M2, fmt_b, fmt_b, need[0], need[1], need[2], sx, sw,
                                gr, 1.0, sg, ws, nbytes, gx, gw, gb)
    return gx, gw, gb, sg


@pytest.mark.parametrize("kn", W.TRAINING_LINEARS)
def test_training_linear_saved_row_major_delayed(kn, tiled_path):
    """The pages' HYBRID step with the backward's copies saved row-major: bytes, steps and
    rings exact against the oracle's forward / backward, outputs within the bound."""
    k, n = kn
    m = W.TRAINING_TOKENS
    xr, wr, gr = _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E5M2)
    oxr, owr, ogr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3"), S.Ring(16, "e5m2")
    for step in range(2):
        t, d, bits = _tensors(m, k, n, 5500 + 10 * step + k + n)
        if step == 0:
            for dr, orr, key in ((xr, oxr, "x"), (wr, owr, "w"), (gr, ogr, "g")):
                F.fp8_scale_ring_seed(dr, d[key], F.FP8_IN_BF16, d[key].numel())
                orr.seed(bf16_out_to_f64(t[key]).astype(np.float32))
        y, x8b, w8b, sx, sw = _forward_save_rm(d["x"], d["w"], d["b"], xr, wr)
        gx, gw, gbias, sg = _backward_rm(d["g"], x8b, w8b, sx, sw, gr)
        torch.cuda.synchronize()
        assert F.fp8_get_device_status() == 0
        f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3", oxr, owr)
        r = L.backward(bits["g"], bits["x"], bits["w"], "e5m2", f["sx"], f["sw"], ogr)
        assert np.array_equal(np_u8(x8b), r["x8t"].T) and np.array_equal(np_u8(w8b), r["w8t"].T)
        assert (sx.item(), sw.item(), sg.item()) == (f["sx"], f["sw"], r["sg"])
        for dev_r, ora_r in ((xr, oxr), (wr, owr), (gr, ogr)):
            assert np.array_equal(_state_bits(dev_r), ora_r.state.view(np.uint32))
        assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], "y")
        assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], "dX")
        assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], "dW")
        assert_bf16_within_ulp(np_bf16_bits(gbias), np.sum(bf16_out_to_f64(t["g"]), axis=0), 1, "grad_b")
        for rr in (xr, wr, gr, oxr, owr, ogr):
            rr.advance()


@pytest.mark.parametrize("mkn", [(208, 256, 272), (200, 384, 640), (512, 384, 640)])
def test_saved_row_major_pair_equals_saved_transpose_pair(mkn):
    """Ragged tiles: the row-major pair and the saved-transpose pair from equal ring states
    give bit-identical y, grad_x, grad_w, steps and rings, and grad_b within one bf16 ulp of
    the exact column sum from each."""
    m, k, n = mkn
    _, d, _ = _tensors(m, k, n, 6300 + m)
    rings = []
    for _ in range(2):
        rs = (_ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E5M2))
        for rr, key in zip(rs, ("x", "w", "g")):
            F.fp8_scale_ring_seed(rr, d[key], F.FP8_IN_BF16, d[key].numel())
        rings.append(rs)
    (xr, wr, gr), (xr2, wr2, gr2) = rings
    y, x8b, w8b, sx, sw = _forward_save_rm(d["x"], d["w"], d["b"], xr, wr)
    gx, gw, gb, sg = _backward_rm(d["g"], x8b, w8b, sx, sw, gr)
    if m % 16 == 0:
        y2, x8t, w8t, sx2, sw2 = _forward_save(d["x"], d["w"], d["b"], xr2, wr2)
        gx2, gw2, gb2, sg2 = _backward_saved(d["g"], x8t, w8t, sx2, sw2, gr2)
    else:  # the transposed copy of x needs m % 16 == 0: compare with the re-quantizing pair
        nf = F.linear_forward_fp8_workspace_size(m, k, n)
        nb = F.linear_backward_fp8_workspace_size(m, k, n)
        wsf, wsb = (torch.empty(v, dtype=torch.uint8, device=DEV) for v in (nf, nb))
        y2, gx2, gw2, gb2 = torch.empty_like(y), torch.empty_like(gx), torch.empty_like(gw), torch.empty_like(gb)
        sx2, sw2, sg2 = (torch.zeros(1, device=DEV) for _ in range(3))
        F.linear_forward_fp8(d["x"], d["w"], 0, None, d["b"], None, m, k, n, F.FP8_E4M3, xr2, wr2, 1.0, sx2, sw2,
                             wsf, nf, y2)
        F.linear_backward_fp8(d["g"], d["x"], d["w"], m, k, n, F.FP8_E5M2, 1, 0, 1, sx2, sw2, gr2, 1.0, sg2, wsb, nb,
                              gx2, None, gb2)
        gw2 = gw  # grad_w of the re-quantizing pair needs m % 16 == 0 as well
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    for a, b in ((y, y2), (gx, gx2), (gw, gw2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # grad_b: the two compositions' column-sum kernels add in different orders; each within one
    # bf16 ulp of the exact column sum
    exact = d["g"].double().sum(0).cpu().numpy()
    for v in (gb, gb2):
        assert_bf16_within_ulp(np_bf16_bits(v), exact, 1, "grad_b")
    assert torch.equal(torch.cat([sx, sw, sg]), torch.cat([sx2, sw2, sg2]))
    for a, b in zip((xr, wr, gr), (xr2, wr2, gr2)):
        assert np.array_equal(_state_bits(a), _state_bits(b))


def test_weight_gradient_split_from_the_backward_on_another_stream():
    """The row-major backward run as grad_x + grad_b first (linear_backward_fp8_mixed without
    grad_w; its g8 stays at the start of its workspace), then grad_w on a second stream from those
    bytes (linear_backward_fp8_prequant with g and x pre-quantized): every output and the ring
    bit-identical to the one-launch backward."""
    m, k, n = 512, 384, 640
    _, d, _ = _tensors(m, k, n, 6400)
    rings = []
    for _ in range(2):
        rs = (_ring(16, F.FP8_E4M3), _ring(16, F.FP8_E4M3), _ring(16, F.FP8_E5M2))
        for rr, key in zip(rs, ("x", "w", "g")):
            F.fp8_scale_ring_seed(rr, d[key], F.FP8_IN_BF16, d[key].numel())
        rings.append(rs)
    (xr, wr, gr), (xr2, wr2, gr2) = rings
    y, x8b, w8b, sx, sw = _forward_save_rm(d["x"], d["w"], d["b"], xr, wr)
    gx, gw, gb, sg = _backward_rm(d["g"], x8b, w8b, sx, sw, gr)
    # the split: grad_x + grad_b, then grad_w on a side stream
    nb = F.linear_backward_fp8_mixed_workspace_size(m, k, n)
    ws = torch.empty(nb, dtype=torch.uint8, device=DEV)
    gx2 = torch.empty_like(gx)
    gw2 = torch.full_like(gw, float("nan"))
    gb2 = torch.empty_like(gb)
    sg2 = torch.zeros(1, device=DEV)
    F.linear_backward_fp8_mixed(d["g"], x8b, w8b, m, k, n, F.FP8_E5M2, F.FP8_E5M2, F.FP8_E5M2, 1, 0, 1, sx, sw, gr2,
                                1.0, sg2, ws, nb, gx2, None, gb2)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    nq = F.linear_backward_fp8_workspace_size(m, k, n)
    wsq = torch.empty(nq, dtype=torch.uint8, device=DEV)
    with torch.cuda.stream(side):
        F.linear_backward_fp8_prequant(ws, 1, sg2, x8b, 1, None, 0, m, k, n, F.FP8_E5M2, 0, 1, 0, sx, None, None, 1.0,
                                       None, wsq, nq, None, gw2, None)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    for a, b in ((gx, gx2), (gw, gw2), (gb, gb2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(sg, sg2)
    assert np.array_equal(_state_bits(gr), _state_bits(gr2))

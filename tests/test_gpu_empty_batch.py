"""GPU parity on the degenerate batch: no rows (m = 0), no output columns (n = 0), and no inner
dimension (k = 0).

An empty batch comes with null pointers for its empty tensors (framework tensors without
elements have none).  The linear entries accept them and do what the definition gives for no
rows: the quantize of an empty x or g measures an amax of 0, and the ring records it; y and
grad_x have no elements; grad_w = g^T . x over no rows and grad_b = the column sum of no rows are
zero.  With n = 0, grad_x = g . w over no columns is zero and y, grad_w, grad_b have no
elements.  With k = 0 the product is empty and y is the bias.  Checked against the oracle's forward /
backward on the same tensors: every ring state and step bit-exact, grad_w and grad_b exactly zero,
y exactly the bias, for the pages' split, the row-major and transposed compositions, the
pre-quantized-operand backward and dynamic scaling.

Definitions: AstrAI compare view, astrai/extension/fp8.py (fp8_linear_forward,
_LinearFp8.backward; the amax of an empty tensor is the initial 0 of the reduction).
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
from oracle import linear as L
from oracle import scaling as S
from helpers import bf16_out_to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
E4, E5 = F.FP8_E4M3, F.FP8_E5M2


def _ring(fmt):
    st = torch.zeros(20, dtype=torch.float32, device=DEV)
    F.fp8_scale_ring_init(st, 16)
    return F.Ring(st, 16, fmt)


def _bits(r):
    return r.state.detach().cpu().numpy().view(np.uint32)


def _setup(m, k, n, seed):
    t = W.training_linear(m, k, n, seed=seed)
    d = {key: t[key].to(DEV) for key in ("x", "w", "b", "g")}
    bits = {key: W.bf16_bits(t[key]) for key in ("x", "w", "b", "g")}
    rings = (_ring(E4), _ring(E4), _ring(E5))
    orings = (S.Ring(16, "e4m3"), S.Ring(16, "e4m3"), S.Ring(16, "e5m2"))
    for r, o, key in zip(rings, orings, ("x", "w", "g")):
        F.fp8_scale_ring_seed(r, d[key], F.FP8_IN_BF16, d[key].numel())
        o.seed(bf16_out_to_f64(t[key]).astype(np.float32))
    return t, d, bits, rings, orings


def _zeros_bits(t):
    return torch.equal(t.view(torch.int16), torch.zeros_like(t).view(torch.int16))


def _out(shape, dtype=torch.bfloat16):
    return torch.full(shape, -1234.5, dtype=dtype, device=DEV) if dtype == torch.bfloat16 else \
        torch.full(shape, 0xA5, dtype=dtype, device=DEV)


@pytest.mark.parametrize("mkn", [(0, 256, 384), (256, 128, 0)])
@pytest.mark.parametrize("path", ["split", "rowmajor", "transposed", "prequant"])
def test_empty_batch_delayed(path, mkn):
    m, k, n = mkn
    t, d, bits, (xr, wr, gr), (oxr, owr, ogr) = _setup(m, k, n, 9100 + n)
    steps = torch.zeros(3, device=DEV)
    y = _out((m, n))
    gx, gw, gb = _out((m, k)), _out((n, k)), _out((n,))
    nf = F.linear_forward_fp8_workspace_size(m, k, n)
    wsf = torch.empty(nf, dtype=torch.uint8, device=DEV)
    if path == "split":
        F.linear_forward_fp8(d["x"], d["w"], 0, None, d["b"], None, m, k, n, E4, xr, wr, 1.0, steps[0:1],
                             steps[1:2], wsf, nf, y)
        nb = F.linear_backward_fp8_workspace_size(m, k, n)
        wsb = torch.empty(nb, dtype=torch.uint8, device=DEV)
        F.linear_backward_fp8(d["g"], d["x"], d["w"], m, k, n, E5, 1, 1, 1, steps[0:1], steps[1:2], gr, 1.0,
                              steps[2:3], wsb, nb, gx, gw, gb)
    elif path == "rowmajor":
        x8b, w8b = _out((m, k), torch.uint8), _out((n, k), torch.uint8)
        F.linear_forward_fp8_save_rm(d["x"], d["w"], d["b"], None, m, k, n, E4, E5, xr, wr, steps[0:1], steps[1:2],
                                     x8b, w8b, wsf, nf, y)
        nb = F.linear_backward_fp8_mixed_workspace_size(m, k, n)
        wsb = torch.empty(nb, dtype=torch.uint8, device=DEV)
        F.linear_backward_fp8_mixed(d["g"], x8b, w8b, m, k, n, E5, E5, E5, 1, 1, 1, steps[0:1], steps[1:2], gr, 1.0,
                                    steps[2:3], wsb, nb, gx, gw, gb)
    elif path == "transposed":
        x8t, w8t = _out((k, m), torch.uint8), _out((k, n), torch.uint8)
        F.linear_forward_fp8_save_t(d["x"], d["w"], d["b"], None, m, k, n, E4, E5, xr, wr, steps[0:1], steps[1:2],
                                    x8t, w8t, wsf, nf, y)
        nb = F.linear_backward_fp8_saved_t_workspace_size(m, k, n)
        wsb = torch.empty(nb, dtype=torch.uint8, device=DEV)
        F.linear_backward_fp8_saved_t(d["g"], x8t, w8t, m, k, n, E5, E5, 1, 1, 1, steps[0:1], steps[1:2], gr, 1.0,
                                      steps[2:3], wsb, nb, gx, gw, gb)
    else:
        F.linear_forward_fp8(d["x"], d["w"], 0, None, d["b"], None, m, k, n, E4, xr, wr, 1.0, steps[0:1],
                             steps[1:2], wsf, nf, y)
        nb = F.linear_backward_fp8_workspace_size(m, k, n)
        wsb = torch.empty(nb, dtype=torch.uint8, device=DEV)
        F.linear_backward_fp8_prequant(d["g"], 0, None, d["x"], 0, d["w"], 0, m, k, n, E5, 1, 1, 1, steps[0:1],
                                       steps[1:2], gr, 1.0, steps[2:3], wsb, nb, gx, gw, gb)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3", oxr, owr)
    r = L.backward(bits["g"], bits["x"], bits["w"], "e5m2", f["sx"], f["sw"], ogr)
    assert (steps[0].item(), steps[1].item(), steps[2].item()) == (f["sx"], f["sw"], r["sg"])
    for dev_r, ora_r in ((xr, oxr), (wr, owr), (gr, ogr)):
        assert np.array_equal(_bits(dev_r), ora_r.state.view(np.uint32))
    if m == 0:  # the sums over no rows
        assert _zeros_bits(gw) and _zeros_bits(gb)
        assert not np.abs(r["dw"]).any() and not np.abs(r["grad_b"]).any()
    if n == 0:  # the sum over no columns
        assert _zeros_bits(gx)
        assert not np.abs(r["dx"]).any()


def test_no_rows_dynamic():
    m, k, n = 0, 128, 256
    t = W.training_linear(m, k, n, seed=9200)
    d = {key: t[key].to(DEV) for key in ("x", "w", "b", "g")}
    bits = {key: W.bf16_bits(t[key]) for key in ("x", "w", "b", "g")}
    steps = torch.zeros(3, device=DEV)
    y = _out((m, n))
    gx, gw, gb = _out((m, k)), _out((n, k)), _out((n,))
    nf = F.linear_forward_fp8_workspace_size(m, k, n)
    nb = F.linear_backward_fp8_workspace_size(m, k, n)
    wsf = torch.empty(nf, dtype=torch.uint8, device=DEV)
    wsb = torch.empty(nb, dtype=torch.uint8, device=DEV)
    F.linear_forward_fp8(d["x"], d["w"], 0, None, d["b"], None, m, k, n, E4, None, None, 1.0, steps[0:1],
                         steps[1:2], wsf, nf, y)
    F.linear_backward_fp8(d["g"], d["x"], d["w"], m, k, n, E5, 1, 1, 1, None, None, None, 1.0, steps[2:3], wsb, nb,
                          gx, gw, gb)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3")
    r = L.backward(bits["g"], bits["x"], bits["w"], "e5m2")
    assert (steps[0].item(), steps[1].item(), steps[2].item()) == (f["sx"], f["sw"], r["sg"])
    assert _zeros_bits(gw) and _zeros_bits(gb)


def test_no_inner_dimension_forward_is_the_bias():
    """k = 0: the product is empty, so y[i][j] = bias[j] rounded to bf16 (the bias is bf16
    already); the rings record an amax of 0 for the empty x and w."""
    m, k, n = 64, 0, 192
    t, d, bits, (xr, wr, _), (oxr, owr, _) = _setup(m, k, n, 9300)
    steps = torch.zeros(2, device=DEV)
    y = _out((m, n))
    nf = F.linear_forward_fp8_workspace_size(m, k, n)
    wsf = torch.empty(nf, dtype=torch.uint8, device=DEV)
    F.linear_forward_fp8(d["x"], d["w"], 0, None, d["b"], None, m, k, n, E4, xr, wr, 1.0, steps[0:1], steps[1:2],
                         wsf, nf, y)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3", oxr, owr)
    assert torch.equal(y.view(torch.int16), d["b"].expand(m, n).contiguous().view(torch.int16))
    assert np.array_equal(bf16_out_to_f64(y), f["y"])
    assert (steps[0].item(), steps[1].item()) == (f["sx"], f["sw"])
    for dev_r, ora_r in ((xr, oxr), (wr, owr)):
        assert np.array_equal(_bits(dev_r), ora_r.state.view(np.uint32))

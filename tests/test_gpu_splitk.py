"""GPU parity of the split-K GEMM schedule inside linear_forward_fp8 / linear_backward_fp8.

The linear compositions may cut an output tile's K range across CTAs: contributor CTAs leave
fp32 partial sums in the workspace, the tile's owner adds them in a fixed order before the
dequantize / bias epilogue.  Here every split count (1 = none, 2, 3, 4) is forced on shapes
with ragged M / N edges and K ranges of unequal length, forward and the grouped dX / dW
backward, and each result is held to the GEMM bound of the oracle's fp64 product; the
bytes of a split result are also checked to repeat exactly run after run.

Definitions: AstrAI compare view, astrai/extension/fp8.py -- fp8_linear_forward and
_LinearFp8.backward (the results split-K must reproduce; the split itself is not on the
pages).
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
from oracle import linear as L
from helpers import np_bf16_bits, bf16_out_to_f64, assert_within_gemm_bound, assert_bf16_within_ulp

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (m, k, n): K of 11 and 13 k-blocks split unevenly; M, N with partial edge tiles
SHAPES = [(640, 1408, 384), (512, 1664, 768), (1008, 2048, 272)]


@pytest.fixture
def split_mode(request):
    F.fp8_set_gemm_split_k(request.param)
    yield request.param
    F.fp8_set_gemm_split_k(1)  # the library default


def _run(t, fmt_f, fmt_b):
    x, w, b, g = (t[key].to(DEV) for key in ("x", "w", "b", "g"))
    m, k = x.shape
    n = w.shape[0]
    fb = F.linear_forward_fp8_workspace_size(m, k, n)
    bb = F.linear_backward_fp8_workspace_size(m, k, n)
    # workspaces start with garbage: nothing in them may be assumed zero
    wsf = torch.full((fb,), 0x5A, dtype=torch.uint8, device=DEV)
    wsb = torch.full((bb,), 0xA5, dtype=torch.uint8, device=DEV)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    gx = torch.empty((m, k), dtype=torch.bfloat16, device=DEV)
    gw = torch.empty((n, k), dtype=torch.bfloat16, device=DEV)
    gb = torch.empty((n,), dtype=torch.bfloat16, device=DEV)
    sx, sw, sg = (torch.zeros(1, device=DEV) for _ in range(3))
    F.linear_forward_fp8(x, w, 0, None, b, None, m, k, n, fmt_f, None, None, 1.0, sx, sw, wsf, fb, y)
    F.linear_backward_fp8(g, x, w, m, k, n, fmt_b, 1, 1, 1, None, None, None, 1.0, sg, wsb, bb, gx, gw, gb)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    return y, gx, gw, gb


_ORACLE = {}


def _oracle(shape):
    """Inputs and the oracle's forward / backward for one shape (computed once per shape)."""
    if shape not in _ORACLE:
        m, k, n = shape
        t = W.training_linear(m, k, n, seed=7000 + m + k + n)
        xb, wb, bb, gbits = (W.bf16_bits(t[key]) for key in ("x", "w", "b", "g"))
        _ORACLE[shape] = (t, L.forward(xb, wb, bb, "e4m3"), L.backward(gbits, xb, wb, "e5m2", None, None))
    return _ORACLE[shape]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("split_mode", [1, 0, 2, 3, 4], indirect=True)
def test_split_k_linear_within_bound(split_mode, shape):
    t, f, r = _oracle(shape)
    y, gx, gw, gb = _run(t, F.FP8_E4M3, F.FP8_E5M2)
    assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], f"y split {split_mode}")
    assert_within_gemm_bound(bf16_out_to_f64(gx), r["dx"], r["dx_abs"], r["dx_sc"], f"dX split {split_mode}")
    assert_within_gemm_bound(bf16_out_to_f64(gw), r["dw"], r["dw_abs"], r["dw_sc"], f"dW split {split_mode}")
    assert_bf16_within_ulp(np_bf16_bits(gb), np.sum(bf16_out_to_f64(t["g"]), axis=0), 1, "grad_b")


@pytest.mark.parametrize("split_mode", [3], indirect=True)
def test_split_k_is_deterministic(split_mode):
    t = W.training_linear(512, 1664, 768, seed=7100)
    first = [v.clone() for v in _run(t, F.FP8_E4M3, F.FP8_E5M2)]
    for _ in range(3):
        again = _run(t, F.FP8_E4M3, F.FP8_E5M2)
        for a, b in zip(first, again):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))

"""GPU parity of the data-parallel fold path on one rank (no collective needed).

Under fp8_set_ring_fold_mode(1) the linear entries leave the measured amax in each ring's
amax slot; fp8_scale_ring_collect_amax gathers the slots and fp8_scale_ring_fold folds the
rings.  Against the oracle: the slots hold exactly the oracle's amax of x, w and g, the rest
of each ring is untouched until the fold, and after the fold the rings are bit-identical to
the oracle's rings folded in the call.

Definitions: AstrAI compare view, astrai/extension/fp8.py (_ScaleRing fold); the deferred,
cross-rank fold is this library's data-parallel reading.
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
from fp8_delayed_scaling_amax_b200 import dp
import workloads as W
from oracle import linear as L
from oracle import scaling as S
from helpers import bf16_out_to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture
def deferred_folds():
    F.fp8_set_ring_fold_mode(1)
    yield
    F.fp8_set_ring_fold_mode(0)


def _ring(fmt):
    st = torch.zeros(16 + 4, dtype=torch.float32, device=DEV)
    F.fp8_scale_ring_init(st, 16)
    return F.Ring(st, 16, fmt)


def _bits(r):
    return r.state.detach().cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("use_buffer", [True, False])
def test_deferred_fold_then_collect_and_fold(deferred_folds, use_buffer):
    m, k, n = 1024, 512, 768
    xr, wr, gr = _ring(F.FP8_E4M3), _ring(F.FP8_E4M3), _ring(F.FP8_E5M2)
    oxr, owr, ogr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3"), S.Ring(16, "e5m2")
    for step in range(3):
        t = W.training_linear(m, k, n, seed=8100 + step)
        x, w, b, g = (t[key].to(DEV) for key in ("x", "w", "b", "g"))
        xb, wb, bb, gbits = (W.bf16_bits(t[key]) for key in ("x", "w", "b", "g"))
        if step == 0:
            for dr, orr, v, key in ((xr, oxr, x, "x"), (wr, owr, w, "w"), (gr, ogr, g, "g")):
                F.fp8_scale_ring_seed(dr, v, F.FP8_IN_BF16, v.numel())
                orr.seed(bf16_out_to_f64(t[key]).astype(np.float32))
        before = [_bits(r).copy() for r in (xr, wr, gr)]
        nf = F.linear_forward_fp8_workspace_size(m, k, n)
        nb = F.linear_backward_fp8_workspace_size(m, k, n)
        wsf, wsb = (torch.empty(v, dtype=torch.uint8, device=DEV) for v in (nf, nb))
        y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
        gx = torch.empty((m, k), dtype=torch.bfloat16, device=DEV)
        gw = torch.empty((n, k), dtype=torch.bfloat16, device=DEV)
        gbias = torch.empty((n,), dtype=torch.bfloat16, device=DEV)
        steps = torch.zeros(3, device=DEV)
        F.linear_forward_fp8(x, w, 0, None, b, None, m, k, n, F.FP8_E4M3, xr, wr, 1.0, steps[0:1], steps[1:2], wsf,
                             nf, y)
        F.linear_backward_fp8(g, x, w, m, k, n, F.FP8_E5M2, 1, 1, 1, steps[0:1], steps[1:2], gr, 1.0, steps[2:3],
                              wsb, nb, gx, gw, gbias)
        torch.cuda.synchronize()
        assert F.fp8_get_device_status() == 0
        f = L.forward(xb, wb, bb, "e4m3", oxr, owr)
        r = L.backward(gbits, xb, wb, "e5m2", f["sx"], f["sw"], ogr)
        # the call left only the amax slot (and nothing else) of each ring changed
        for dev_r, old, am in ((xr, before[0], f["amax_x"]), (wr, before[1], f["amax_w"]), (gr, before[2], r["amax_g"])):
            now = _bits(dev_r)
            slot = dev_r.hist_len + 2
            assert np.float32(dev_r.state[slot].item()) == np.float32(am)
            mask = np.ones(now.shape, bool)
            mask[slot] = False
            assert np.array_equal(now[mask], old[mask])
        assert (steps[0].item(), steps[1].item(), steps[2].item()) == (f["sx"], f["sw"], r["sg"])
        rings = [xr, wr, gr]
        if use_buffer:
            buf = torch.full((4,), -1.0, device=DEV)
            dp.fold_rings_data_parallel(rings, buf)
            torch.cuda.synchronize()
            assert buf[:3].cpu().numpy().tolist() == [float(f["amax_x"]), float(f["amax_w"]), float(r["amax_g"])]
        else:
            F.fp8_scale_ring_fold(rings)
            torch.cuda.synchronize()
        for dev_r, ora_r in ((xr, oxr), (wr, owr), (gr, ogr)):
            assert np.array_equal(_bits(dev_r), ora_r.state.view(np.uint32))
        for rr in (xr, wr, gr, oxr, owr, ogr):
            rr.advance()

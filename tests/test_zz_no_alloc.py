"""The allocation-free forward entry point (`linear_forward_fp8_noalloc`).

It serves callers that cannot allocate device memory when they run the forward pass -- for
example a plug-in whose host application owns the device-memory budget, or a service that
keeps a fixed footprint after start-up: its scratch is one built-in 16 MiB device array
instead of a caller workspace.  Here it is called through the C ABI twice in a row and its
output is compared with the workspace entry point's (run with the same unsplit GEMM
schedule) bit for bit, and with the oracle's forward (dynamic, or delayed with the oracle's
own rings) within the GEMM bound the other tests use.  Also covered: no step snapshots
requested (the steps then live in the built-in array), a pre-quantized weight, and a shape
whose operand buffers exceed the array.  This file is named so pytest collects it last.
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
from oracle import linear as L
from oracle import scaling as S
from helpers import bf16_out_to_f64, assert_within_gemm_bound

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ring(fmt):
    st = torch.zeros(16 + 4, dtype=torch.float32, device=DEV)
    F.fp8_scale_ring_init(st, 16)
    return F.Ring(st, 16, fmt)


def _forward_both(t, delayed, rings, snapshots=True):
    x, w, b = (t[key].to(DEV) for key in ("x", "w", "b"))
    m, k = x.shape
    n = w.shape[0]
    nbytes = F.linear_forward_fp8_workspace_size(m, k, n)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    y_ws = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    y_na = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    s_ws = torch.zeros(2, device=DEV)
    s_na = torch.zeros(2, device=DEV)
    (rx1, rw1), (rx2, rw2) = rings if delayed else ((None, None), (None, None))
    F.linear_forward_fp8(x, w, 0, None, b, None, m, k, n, F.FP8_E4M3, rx1, rw1, 1.0, s_ws[0:1], s_ws[1:2], ws,
                         nbytes, y_ws)
    F.linear_forward_fp8_noalloc(x, w, 0, None, b, None, m, k, n, F.FP8_E4M3, rx2, rw2, 1.0,
                                 s_na[0:1] if snapshots else None, s_na[1:2] if snapshots else None, y_na)
    torch.cuda.synchronize()
    return y_ws, y_na, s_ws, s_na


@pytest.fixture
def unsplit_gemm():
    """The no-alloc entry never splits the GEMM's K; with splitting also off in the workspace
    entry both run the same kernels, so their outputs must agree bit for bit."""
    F.fp8_set_gemm_split_k(1)
    yield
    F.fp8_set_gemm_split_k(1)  # the library default


@pytest.mark.parametrize("snapshots", [True, False])
@pytest.mark.parametrize("delayed", [False, True])
def test_noalloc_forward_matches_workspace_forward_twice(delayed, snapshots, unsplit_gemm):
    rings = [(_ring(F.FP8_E4M3), _ring(F.FP8_E4M3)) for _ in range(2)]
    oxr, owr = S.Ring(16, "e4m3"), S.Ring(16, "e4m3")
    for call in range(2):
        t = W.training_linear(384, 512, 640, seed=500 + call)
        xb, wb, bb = (W.bf16_bits(t[key]) for key in ("x", "w", "b"))
        if delayed and call == 0:
            for rx, rw in rings:
                F.fp8_scale_ring_seed(rx, t["x"].to(DEV), F.FP8_IN_BF16, t["x"].numel())
                F.fp8_scale_ring_seed(rw, t["w"].to(DEV), F.FP8_IN_BF16, t["w"].numel())
            oxr.seed(bf16_out_to_f64(t["x"]).astype(np.float32))
            owr.seed(bf16_out_to_f64(t["w"]).astype(np.float32))
        y_ws, y_na, s_ws, s_na = _forward_both(t, delayed, rings, snapshots)
        if snapshots:
            assert torch.equal(s_ws, s_na)
        # the oracle's forward: dynamic, or delayed with its own rings
        f = L.forward(xb, wb, bb, "e4m3", oxr if delayed else None, owr if delayed else None)
        assert_within_gemm_bound(bf16_out_to_f64(y_na), f["y"], f["s_abs"], f["sc"], f"no-alloc vs oracle, call {call}")
        assert (s_ws[0].item(), s_ws[1].item()) == (f["sx"], f["sw"])
        # and bit for bit against the workspace entry point
        assert torch.equal(y_na.view(torch.int16), y_ws.view(torch.int16)), f"call {call}"
        if delayed:
            assert torch.equal(rings[0][0].state, rings[1][0].state)
            assert torch.equal(rings[0][1].state, rings[1][1].state)
            assert np.array_equal(rings[1][0].state.cpu().numpy().view(np.uint32), oxr.state.view(np.uint32))
            for r in (*rings[0], *rings[1], oxr, owr):
                r.advance()
    assert F.fp8_get_device_status() == 0


def test_noalloc_prequantized_weight(unsplit_gemm):
    """A weight passed as fp8 bytes with its step: only x is quantized into the array."""
    m, k, n = 256, 512, 384
    x = W.normal_bf16((m, k), 1.0, seed=520)
    w8, s8 = W.amax_scaled_fp8_bytes((n, k), seed=521)
    w_step = np.float32(0.02 * s8)
    xd, w8d = x.to(DEV), w8.to(DEV)
    step = torch.tensor([float(w_step)], device=DEV)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    sx = torch.zeros(1, device=DEV)
    sw = torch.zeros(1, device=DEV)
    for _ in range(2):
        F.linear_forward_fp8_noalloc(xd, w8d, 1, step, None, None, m, k, n, F.FP8_E4M3, None, None, 1.0, sx, sw, y)
        torch.cuda.synchronize()
        f = L.forward(W.bf16_bits(x), None, None, "e4m3", w8=W.u8(w8), w_step=w_step)
        assert (sx.item(), sw.item()) == (f["sx"], w_step)
        assert_within_gemm_bound(bf16_out_to_f64(y), f["y"], f["s_abs"], f["sc"], "no-alloc, fp8 weight")
    assert F.fp8_get_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_array():
    m, k, n = 4096, 4096, 4096  # needs 32 MiB of operand scratch
    assert F.linear_forward_fp8_workspace_size(m, k, n) > F.NOALLOC_WORKSPACE_BYTES
    with pytest.raises(F.FP8Error) as err:
        F.linear_forward_fp8_noalloc(16, 16, 0, None, None, None, m, k, n, F.FP8_E4M3, None, None, 1.0, None, None,
                                     16)
    assert err.value.code == -5 and "built-in array" in str(err.value)
    # sizes whose products would wrap are rejected before any pointer is used
    with pytest.raises(F.FP8Error) as err:
        F.linear_forward_fp8_noalloc(16, 16, 0, None, None, None, 1 << 62, 16, 16, F.FP8_E4M3, None, None, 1.0, None,
                                     None, 16)
    assert err.value.code == -5

"""GPU parity: quantize (row-major / transposed / dual), amax, the history-ring fold, seeding
and dynamic steps -- bit-exact against the oracle, through the C ABI.

Definitions: AstrAI compare view -- csrc/kernels/fp8/quantize.cuh (fp8_quantize_kernel,
fp8_quantize_tiled_kernel, publish_amax) and astrai/extension/fp8.py (_ScaleRing,
FP8Recipe, _dynamic_scale).
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
from oracle import quantize as Q
from oracle import scaling as S
from helpers import np_u8, in_values_f32

pytestmark = pytest.mark.gpu

DEV = "cuda"
FMTS = [(F.FP8_E4M3, "e4m3"), (F.FP8_E5M2, "e5m2")]
IN_TYPES = [(F.FP8_IN_BF16, torch.bfloat16), (F.FP8_IN_F16, torch.float16), (F.FP8_IN_F32, torch.float32)]
SHAPES = [(1, 1), (3, 5), (17, 8), (128, 128), (130, 257), (256, 1024), (1000, 24), (2048, 1024), (257, 4112)]


def _scale(s):
    return torch.tensor([s], dtype=torch.float32, device=DEV)


def _input(shape, dtype, seed, spread=3.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g) * spread
    # sprinkle values that exercise saturation, subnormals and signed zero
    flat = x.view(-1)
    n = flat.numel()
    if n >= 8:
        flat[0] = 1e6
        flat[1] = -1e6
        flat[2] = 1e-9
        flat[3] = -0.0
        flat[4] = 0.0
    return x.to(dtype)


def _quantize(x, in_type, s, fmt, mode, ring=None, amax=True):
    rows, cols = x.shape
    out = torch.full((rows, cols), 0xAB, dtype=torch.uint8, device=DEV)
    out_t = torch.full((cols, rows), 0xCD, dtype=torch.uint8, device=DEV)
    a = torch.full((1,), -1.0, dtype=torch.float32, device=DEV) if amax else None
    sc = s if isinstance(s, torch.Tensor) else _scale(s)
    if mode == "row":
        F.fp8_quantize(x, in_type, rows, cols, sc, fmt, 0, out, a, ring)
        return out, None, a
    if mode == "t":
        F.fp8_quantize(x, in_type, rows, cols, sc, fmt, 1, out_t, a, ring)
        return None, out_t, a
    F.fp8_quantize_dual(x, in_type, rows, cols, sc, fmt, out, out_t, a, ring)
    return out, out_t, a


@pytest.mark.parametrize("fmt,fname", FMTS)
@pytest.mark.parametrize("in_type,dtype", IN_TYPES)
@pytest.mark.parametrize("mode", ["row", "t", "dual"])
def test_quantize_bit_exact(fmt, fname, in_type, dtype, mode, tiled_path):
    for i, shape in enumerate(SHAPES):
        x = _input(shape, dtype, seed=i + 10 * fmt)
        s = [1.0, 0.0173, 3.3e-3, 17.25][i % 4]
        out, out_t, a = _quantize(x.to(DEV), in_type, s, fmt, mode)
        torch.cuda.synchronize()
        xv = in_values_f32(x)
        want = Q.quantize_values(xv, s, fname)
        if out is not None:
            assert np.array_equal(np_u8(out), want), (shape, mode)
        if out_t is not None:
            assert np.array_equal(np_u8(out_t), want.T), (shape, mode)
        assert a.item() == Q.amax(xv), shape


@pytest.mark.parametrize("mode", ["row", "t", "dual"])
def test_quantize_misaligned_and_strided_bases(mode, tiled_path):
    """A base pointer off the 16-byte grid takes the element path; results are identical."""
    big = _input((129 * 77 + 1,), torch.bfloat16, seed=3).to(DEV)
    x = big[1:].view(129, 77)
    out, out_t, a = _quantize(x, F.FP8_IN_BF16, 0.05, F.FP8_E4M3, mode)
    torch.cuda.synchronize()
    xv = in_values_f32(x)
    want = Q.quantize_values(xv, 0.05, "e4m3")
    if out is not None:
        assert np.array_equal(np_u8(out), want)
    if out_t is not None:
        assert np.array_equal(np_u8(out_t), want.T)
    assert a.item() == Q.amax(xv)


@pytest.mark.parametrize("in_type,dtype", IN_TYPES)
@pytest.mark.parametrize("mode", ["row", "t", "dual"])
def test_quantize_special_values(in_type, dtype, mode, tiled_path):
    """NaN, +-inf, subnormals and signed zeros in 16-bit and 32-bit inputs, on the vector and
    tiled paths: amax ignores NaN and is inf when an inf is present; inf saturates; every
    non-NaN byte equals the oracle's; a NaN's byte is a NaN code (0x7F with either sign)."""
    g = torch.Generator().manual_seed(77)
    x = torch.randn((256, 384), generator=g)
    tiny = {torch.bfloat16: 3e-39, torch.float16: 3e-6, torch.float32: 1e-41}[dtype]
    flat = x.view(-1)
    flat[5::97] = float("nan")
    flat[11::301] = tiny
    flat[12::301] = -tiny
    flat[13::211] = -0.0
    for case in ("nan_only", "with_inf"):
        xc = x.clone()
        if case == "with_inf":
            xc.view(-1)[7] = float("inf")
            xc.view(-1)[9000] = float("-inf")
        xd = xc.to(dtype)
        out, out_t, a = _quantize(xd.to(DEV), in_type, 0.0173, F.FP8_E4M3, mode)
        torch.cuda.synchronize()
        xv = in_values_f32(xd)
        want = Q.quantize_values(xv, 0.0173, "e4m3")
        nan = np.isnan(xv)
        for got, ref, mask in ((out, want, nan), (out_t, want.T, nan.T)):
            if got is None:
                continue
            b = np_u8(got)
            assert np.array_equal(b[~mask], ref[~mask]), (case, mode)
            assert ((b[mask] & 0x7F) == 0x7F).all(), (case, mode)
        assert a.item() == Q.amax(xv), (case, mode)


def test_quantize_empty_and_nan():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((0, 64), dtype=torch.uint8, device=DEV)
    a = torch.full((1,), 5.0, device=DEV)
    F.fp8_quantize(x, F.FP8_IN_BF16, 0, 64, _scale(1.0), F.FP8_E4M3, 0, out, a)
    torch.cuda.synchronize()
    assert a.item() == 0.0
    # NaN is ignored by amax; its byte is the canonical NaN code of the device conversion
    x = torch.tensor([[1.0, float("nan"), -2.0, 0.5]] * 4, dtype=torch.float32, device=DEV)
    out = torch.empty((4, 4), dtype=torch.uint8, device=DEV)
    F.fp8_quantize(x, F.FP8_IN_F32, 4, 4, _scale(1.0), F.FP8_E4M3, 0, out, a)
    torch.cuda.synchronize()
    assert a.item() == 2.0
    b = np_u8(out)
    assert (b[:, 1] & 0x7F).tolist() == [0x7F] * 4
    assert b[0, 0] == 0x38 and b[0, 2] == 0xC0


def _ring(hist_len, fmt, margin=0):
    state = torch.zeros(hist_len + 4, dtype=torch.float32, device=DEV)
    F.fp8_scale_ring_init(state, hist_len)
    return F.Ring(state, hist_len, fmt, margin)


def _state_bits(r):
    return r.state.detach().cpu().numpy().view(np.uint32)


def test_delayed_ring_sequence_bit_exact():
    """history 16, margin 0, E4M3: x [512,1024] * s_t over 8 steps; the ring state, the
    used step and the bytes match the oracle exactly after every step."""
    factors = W.delayed_sequence_factors(8, seed=0)
    ring = _ring(16, F.FP8_E4M3)
    oring = S.Ring(16, "e4m3")
    x0 = W.delayed_ring_inputs(0, factors[0])
    F.fp8_scale_ring_seed(ring, x0.to(DEV), F.FP8_IN_BF16, x0.numel())
    oring.seed(in_values_f32(x0))
    torch.cuda.synchronize()
    assert np.array_equal(_state_bits(ring), oring.state.view(np.uint32))
    for t, f in enumerate(factors):
        x = W.delayed_ring_inputs(t, f)
        xd = x.to(DEV)
        step = ring.state[16:17]  # the ring's own step slot: read before the fold publishes
        out = torch.empty(x.shape, dtype=torch.uint8, device=DEV)
        a = torch.zeros(1, device=DEV)
        F.fp8_quantize(xd, F.FP8_IN_BF16, x.shape[0], x.shape[1], step, F.FP8_E4M3, 0, out, a, ring)
        torch.cuda.synchronize()
        xv = in_values_f32(x)
        s_used = oring.scale
        want, am = Q.quantize(xv, s_used, "e4m3")
        oring.fold(am, s_used)
        assert np.array_equal(np_u8(out), want), t
        assert a.item() == am
        assert np.array_equal(_state_bits(ring), oring.state.view(np.uint32)), t
        ring.advance()
        oring.advance()


@pytest.mark.parametrize("mode", ["row", "t", "dual"])
def test_ring_fold_every_mode_and_margin(mode, tiled_path):
    ring = _ring(4, F.FP8_E5M2, margin=2)
    oring = S.Ring(4, "e5m2", margin=2)
    for t in range(6):
        x = _input((300, 200), torch.bfloat16, seed=50 + t, spread=2.0 ** (t - 2))
        if t == 0:
            F.fp8_scale_ring_seed(ring, x.to(DEV), F.FP8_IN_BF16, x.numel())
            oring.seed(in_values_f32(x))
        step = ring.state[4:5]
        out, out_t, a = _quantize(x.to(DEV), F.FP8_IN_BF16, step, F.FP8_E5M2, mode, ring=ring)
        torch.cuda.synchronize()
        s_used = oring.scale
        want, am = Q.quantize(in_values_f32(x), s_used, "e5m2")
        oring.fold(am, s_used)
        if out is not None:
            assert np.array_equal(np_u8(out), want)
        if out_t is not None:
            assert np.array_equal(np_u8(out_t), want.T)
        assert np.array_equal(_state_bits(ring), oring.state.view(np.uint32)), (mode, t)
        ring.advance()
        oring.advance()


def test_dynamic_amax_scale():
    scratch = torch.zeros(4, dtype=torch.int32, device=DEV)
    for i, (shape, fmt, fname, margin) in enumerate([((128, 256), 0, "e4m3", 0), ((2048, 4096), 1, "e5m2", 1),
                                                     ((7, 3), 0, "e4m3", 3), ((0, 5), 0, "e4m3", 0)]):
        x = _input(shape, torch.bfloat16, seed=70 + i)
        s = torch.zeros(1, device=DEV)
        a = torch.zeros(1, device=DEV)
        for _ in range(2):  # scratch is self-cleaning: the second call sees it zeroed
            F.fp8_amax_scale(x.to(DEV), F.FP8_IN_BF16, x.numel(), F.FP8_MAX[fmt], 2.0 ** margin, s, a, scratch)
            torch.cuda.synchronize()
            assert s.item() == S.dynamic_scale(in_values_f32(x), fname, margin)
            assert a.item() == Q.amax(in_values_f32(x))
        assert int(scratch.abs().sum()) == 0


def test_quantize_is_deterministic():
    x = _input((1024, 2048), torch.bfloat16, seed=5).to(DEV)
    res = []
    for _ in range(3):
        out, out_t, a = _quantize(x, F.FP8_IN_BF16, 0.01, F.FP8_E4M3, "dual")
        torch.cuda.synchronize()
        res.append((np_u8(out).copy(), np_u8(out_t).copy(), a.item()))
    for r in res[1:]:
        assert np.array_equal(r[0], res[0][0]) and np.array_equal(r[1], res[0][1]) and r[2] == res[0][2]

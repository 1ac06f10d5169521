"""GPU parity at full sizes: the quantize sweep's largest tensor (16384 x 16384) and a tensor of
more than 2^31 elements, in the launch configurations the bench times.

The oracle cannot encode every byte of these in seconds, so the check samples: fp8 bytes at
random positions plus every corner of the tensor, against the oracle's encoding of those
input values; amax exact over the whole tensor (the oracle's amax, taken chunk by chunk on
the host); and the ring after the fold bit-exact against the oracle's ring folded with that
amax.

Definitions: AstrAI compare view -- csrc/kernels/fp8/quantize.cuh (fp8_quantize_kernel,
fp8_quantize_tiled_kernel, publish_amax) and astrai/extension/fp8.py (_ScaleRing).
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
from oracle import quantize as Q
from oracle import scaling as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
CHUNK = 1 << 24


def _host_amax(x_dev):
    """The oracle's amax of a device bf16 tensor, one host chunk at a time."""
    flat = x_dev.view(-1)
    best = np.float32(0.0)
    for start in range(0, flat.numel(), CHUNK):
        bits = flat[start:start + CHUNK].cpu().view(torch.int16).numpy().view(np.uint16)
        vals = (bits.astype(np.uint32) << 16).view(np.float32)
        best = max(best, Q.amax(vals))
    return np.float32(best)


def _positions(rows, cols, n, seed):
    rng = np.random.default_rng(seed)
    r = rng.integers(0, rows, n, dtype=np.int64)
    c = rng.integers(0, cols, n, dtype=np.int64)
    corners_r = np.array([0, 0, rows - 1, rows - 1, rows // 2, rows - 1], dtype=np.int64)
    corners_c = np.array([0, cols - 1, 0, cols - 1, cols // 2, cols // 2], dtype=np.int64)
    return np.concatenate([r, corners_r]), np.concatenate([c, corners_c])


def _values_at(x_dev, r, c):
    cols = x_dev.shape[1]
    idx = torch.from_numpy(r * cols + c).to(DEV)
    bits = x_dev.view(-1)[idx].cpu().view(torch.int16).numpy().view(np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _ring_pair(fmt, fname, seed_shape=(64, 64)):
    st = torch.zeros(16 + 4, dtype=torch.float32, device=DEV)
    F.fp8_scale_ring_init(st, 16)
    ring = F.Ring(st, 16, fmt)
    seed_x = W.normal_bf16(seed_shape, 2.0, seed=11)
    F.fp8_scale_ring_seed(ring, seed_x.to(DEV), F.FP8_IN_BF16, seed_x.numel())
    oring = S.Ring(16, fname)
    oring.seed((W.bf16_bits(seed_x).astype(np.uint32) << 16).view(np.float32))
    return st, ring, oring


def _check(x, out, out_t, st, oring, fname, samples, seed):
    rows, cols = x.shape
    step = np.float32(oring.scale)
    am = _host_amax(x)
    r, c = _positions(rows, cols, samples, seed)
    want = Q.quantize_values(_values_at(x, r, c), step, fname)
    if out is not None:
        got = out.view(-1)[torch.from_numpy(r * cols + c).to(DEV)].cpu().numpy()
        assert np.array_equal(got, want)
    if out_t is not None:
        got_t = out_t.view(-1)[torch.from_numpy(c * rows + r).to(DEV)].cpu().numpy()
        assert np.array_equal(got_t, want)
    oring.fold(am, step)
    assert np.array_equal(st.cpu().numpy().view(np.uint32), oring.state.view(np.uint32))


@pytest.mark.parametrize("mode", ["row", "t", "dual"])
def test_quantize_sweep_size_sampled(mode):
    """16384 x 16384 bf16 -> E4M3 with a ring (the sweep's largest size, persistent tiled
    kernel for t / dual)."""
    rows = cols = 16384
    x = W.normal_bf16((rows, cols), 1.0, seed=4242, device=DEV)
    st, ring, oring = _ring_pair(F.FP8_E4M3, "e4m3")
    step_dev = st[16:17]
    out = torch.empty((rows, cols), dtype=torch.uint8, device=DEV) if mode != "t" else None
    out_t = torch.empty((cols, rows), dtype=torch.uint8, device=DEV) if mode != "row" else None
    if mode == "row":
        F.fp8_quantize(x, F.FP8_IN_BF16, rows, cols, step_dev, F.FP8_E4M3, 0, out, None, ring)
    elif mode == "t":
        F.fp8_quantize(x, F.FP8_IN_BF16, rows, cols, step_dev, F.FP8_E4M3, 1, out_t, None, ring)
    else:
        F.fp8_quantize_dual(x, F.FP8_IN_BF16, rows, cols, step_dev, F.FP8_E4M3, out, out_t, None, ring)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    _check(x, out, out_t, st, oring, "e4m3", 200_000, 17)


@pytest.mark.parametrize("mode", ["row", "dual"])
def test_quantize_beyond_2_31_elements(mode):
    """32769 x 65536 = 2^31 + 2^16 elements: 64-bit element and byte offsets in the flat and
    the tiled kernels (E5M2, ring); the odd row count also sends the transposed bytes through
    the unvectorised store path."""
    rows, cols = 32769, 65536
    assert rows * cols > 2 ** 31
    x = W.normal_bf16((rows, cols), 1.0, seed=777, device=DEV)
    st, ring, oring = _ring_pair(F.FP8_E5M2, "e5m2")
    step_dev = st[16:17]
    out = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    out_t = torch.empty((cols, rows), dtype=torch.uint8, device=DEV) if mode == "dual" else None
    if mode == "row":
        F.fp8_quantize(x, F.FP8_IN_BF16, rows, cols, step_dev, F.FP8_E5M2, 0, out, None, ring)
    else:
        F.fp8_quantize_dual(x, F.FP8_IN_BF16, rows, cols, step_dev, F.FP8_E5M2, out, out_t, None, ring)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    _check(x, out, out_t, st, oring, "e5m2", 200_000, 23)
    del x, out, out_t
    torch.cuda.empty_cache()

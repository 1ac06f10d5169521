"""GPU parity: the FP8-output GEMM (the quantize fused into the producer's epilogue).

fp8_gemm_fp8out writes the bf16 output of fp8_gemm and, from the same values, fp8 bytes at a
given step plus their amax.  Against the oracle: the bf16 output within the GEMM bound; the
fp8 bytes exactly the oracle's quantize of the GPU's own bf16 output, the amax exactly its
amax (the fused path must equal "GEMM, then quantize"), the bytes unchanged when the bf16
output is not written, padding untouched, and a history ring fed through its slots folding
exactly like the oracle's.

Definitions: AstrAI compare view -- csrc/kernels/fp8/gemm/epilogue.cuh (out_dtype / out_scale
in an earlier state); astrai/extension/fp8.py (_ScaleRing fold).
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
from oracle import fp8_codec as C
from oracle import gemm as G
from oracle import quantize as Q
from oracle import scaling as S
from helpers import np_u8, np_bf16_bits, bf16_out_to_f64, assert_within_gemm_bound

pytestmark = pytest.mark.gpu
DEV = "cuda"
LAYOUTS = {"NT": F.FP8_LAYOUT_NT, "NN": F.FP8_LAYOUT_NN, "TN": F.FP8_LAYOUT_TN, "TT": F.FP8_LAYOUT_TT}
FMT = {"e4m3": F.FP8_E4M3, "e5m2": F.FP8_E5M2}


def _codes(rng, shape, fmt="e4m3", spread=1.0):
    dt = torch.float8_e4m3fn if fmt == "e4m3" else torch.float8_e5m2
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * spread)
    return v.to(dt).view(torch.uint8).numpy()


def _case(layout, m, n, k, batch=1, ldo_pad=0, out8_fmt="e4m3", step=0.0123, seed=0, with_bf16=True):
    rng = np.random.default_rng(seed)
    a_shape = (batch, m, k) if layout[0] == "N" else (batch, k, m)
    b_shape = (batch, n, k) if layout[1] == "T" else (batch, k, n)
    a = _codes(rng, a_shape)
    b = _codes(rng, b_shape)
    lda, ldb = a_shape[2], b_shape[2]
    ldo = n + ldo_pad
    sto = m * ldo
    bias = torch.from_numpy(rng.standard_normal(n).astype(np.float32) * 0.5).to(torch.bfloat16)
    sa, sb = torch.tensor([0.75], device=DEV), torch.tensor([1.5], device=DEV)
    out = torch.full((batch * sto,), 0x7FC1, dtype=torch.int16, device=DEV) if with_bf16 else None
    out8 = torch.full((batch * sto,), 0xAB, dtype=torch.uint8, device=DEV)
    amax = torch.zeros(1, device=DEV)
    step_t = torch.tensor([step], device=DEV)
    used = torch.zeros(1, device=DEV)
    F.fp8_gemm_fp8out(torch.from_numpy(a).to(DEV), torch.from_numpy(b).to(DEV), F.FP8_E4M3, F.FP8_E4M3,
                      LAYOUTS[layout], m, n, k, lda, ldb, ldo, batch, a[0].size if batch > 1 else 0,
                      b[0].size if batch > 1 else 0, sto, sa, sb, bias.to(DEV), None, out, FMT[out8_fmt], step_t,
                      out8, amax, used)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    assert used.item() == np.float32(step)
    o8 = np_u8(out8).reshape(batch, m, ldo)
    y = None
    if with_bf16:
        y = out.cpu().numpy().view(np.uint16).reshape(batch, m, ldo)
    ref = G.gemm_ref(a if batch > 1 else a[0], b if batch > 1 else b[0], layout, "e4m3", "e4m3", 0.75, 1.5,
                     np_bf16_bits(bias))
    return o8, y, amax.item(), ref


@pytest.mark.parametrize("layout,m,n,k", [("NT", 200, 272, 384), ("NT", 512, 1024, 1024), ("NN", 256, 384, 512),
                                          ("TN", 384, 256, 256), ("NT", 2048, 3072, 1024)])
@pytest.mark.parametrize("out8_fmt", ["e4m3", "e5m2"])
def test_fp8_output_is_the_quantized_bf16_output(layout, m, n, k, out8_fmt):
    o8, y, am, (ref, s_abs, sc) = _case(layout, m, n, k, out8_fmt=out8_fmt, seed=m + n + k)
    yv = C.bf16_bits_to_f64(y[0][:, :n].copy()).astype(np.float32)
    assert_within_gemm_bound(yv.astype(np.float64), ref, s_abs, sc, "bf16 output")
    assert np.array_equal(o8[0][:, :n], Q.quantize_values(yv, 0.0123, out8_fmt))
    assert np.float32(am) == Q.amax(yv)
    # without the bf16 output the fp8 bytes and the amax are the same
    o8b, _, amb, _ = _case(layout, m, n, k, out8_fmt=out8_fmt, seed=m + n + k, with_bf16=False)
    assert np.array_equal(o8b, o8) and amb == am


def test_fp8_output_batched_with_padding():
    """Batched (batch 3), padded rows (ldo > n): every batch quantized, padding bytes kept."""
    m, n, k, batch, pad = 136, 200, 256, 3, 24
    o8, y, am, (ref, s_abs, sc) = _case("NT", m, n, k, batch=batch, ldo_pad=pad, out8_fmt="e5m2", step=0.02, seed=5)
    yv = C.bf16_bits_to_f64(y[:, :, :n].copy()).astype(np.float32)
    assert_within_gemm_bound(yv.astype(np.float64), ref, s_abs, sc, "bf16 output")
    assert np.array_equal(o8[:, :, :n], Q.quantize_values(yv, 0.02, "e5m2"))
    assert (o8[:, :, n:] == 0xAB).all()
    assert np.float32(am) == Q.amax(yv)


def test_fp8_output_ragged_half_tiles_with_padding():
    """80 pair tiles on 74 pairs: the last round runs as 256 x 128 half tiles, and with n = 2400
    the last tile column holds 96 valid columns, so one half lies wholly past n.  Padded rows
    (ldo > n): neither bf16 nor fp8 bytes may land past n, and the amax covers only the valid
    columns."""
    m, n, k, pad = 2000, 2400, 384, 32
    o8, y, am, (ref, s_abs, sc) = _case("NT", m, n, k, ldo_pad=pad, out8_fmt="e4m3", step=0.05, seed=31)
    yv = C.bf16_bits_to_f64(y[0][:, :n].copy()).astype(np.float32)
    assert_within_gemm_bound(yv.astype(np.float64), ref, s_abs, sc, "bf16 output")
    assert np.array_equal(o8[0][:, :n], Q.quantize_values(yv, 0.05, "e4m3"))
    assert (o8[0][:, n:] == 0xAB).all(), "fp8 bytes written past n"
    assert (y[0][:, n:] == 0x7FC1).all(), "bf16 values written past n"
    assert np.float32(am) == Q.amax(yv)


def test_fp8_output_feeds_a_ring():
    """out8_step = a ring's step and out8_amax = its amax slot: after fp8_scale_ring_fold the
    ring equals the oracle's ring folded with the amax of the bf16 output."""
    rng = np.random.default_rng(9)
    m, n, k = 512, 768, 512
    a = _codes(rng, (m, k))
    b = _codes(rng, (n, k))
    st = torch.zeros(16 + 4, device=DEV)
    F.fp8_scale_ring_init(st, 16)
    ring = F.Ring(st, 16, F.FP8_E4M3)
    seed_x = torch.from_numpy(rng.standard_normal((64, 64)).astype(np.float32)).to(torch.bfloat16)
    F.fp8_scale_ring_seed(ring, seed_x.to(DEV), F.FP8_IN_BF16, seed_x.numel())
    oring = S.Ring(16, "e4m3")
    oring.seed(seed_x.float().numpy())
    out = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    out8 = torch.empty((m, n), dtype=torch.uint8, device=DEV)
    used = torch.zeros(1, device=DEV)
    one = torch.ones(1, device=DEV)
    F.fp8_gemm_fp8out(torch.from_numpy(a).to(DEV), torch.from_numpy(b).to(DEV), F.FP8_E4M3, F.FP8_E4M3,
                      F.FP8_LAYOUT_NT, m, n, k, k, k, n, 1, 0, 0, 0, one, one, None, None, out, F.FP8_E4M3,
                      st[16:17], out8, st[18:19], used)
    F.fp8_scale_ring_fold([ring])
    torch.cuda.synchronize()
    yv = bf16_out_to_f64(out).astype(np.float32)
    assert used.item() == oring.scale
    assert np.array_equal(np_u8(out8), Q.quantize_values(yv, oring.scale, "e4m3"))
    oring.fold(Q.amax(yv), oring.scale)
    assert np.array_equal(st.cpu().numpy().view(np.uint32), oring.state.view(np.uint32))

"""GPU parity: the FP8 GEMM (tcgen05 + TMA) against the oracle, within the stated bound

    |gpu - ref| <= 2^-8 |ref| + 2^-20 * sum_k |a_k b_k| * RN32(sa * sb)

for the four layouts, both formats and mixed formats, ragged M / N / K, padded leading
dimensions, batched and broadcast operands, bf16 and fp8 (+ bias_scale) bias, k = 0, every
output of the full-size skinny / batched workloads and of the squares up to 4096^3, and
sampled outputs of the 8192^3 square.

Definitions: AstrAI compare view -- astrai/extension/ops/fp8.py (mm_fp8),
csrc/kernels/fp8/common.h (layout tags) and csrc/kernels/fp8/gemm/epilogue.cuh.
"""

import numpy as np
import pytest
import torch

import fp8_delayed_scaling_amax_b200 as F
import workloads as W
from oracle import fp8_codec as C
from oracle import gemm as G
from helpers import np_u8, np_bf16_bits, bf16_out_to_f64, assert_within_gemm_bound

pytestmark = pytest.mark.gpu
DEV = "cuda"
LAYOUTS = {"NT": F.FP8_LAYOUT_NT, "NN": F.FP8_LAYOUT_NN, "TN": F.FP8_LAYOUT_TN, "TT": F.FP8_LAYOUT_TT}
FMT = {"e4m3": F.FP8_E4M3, "e5m2": F.FP8_E5M2}
NAN_CODE = 0x7F  # NaN in both formats: padding the kernel must never read


def _codes(rng, shape, fmt, spread=1.0):
    dt = torch.float8_e4m3fn if fmt == "e4m3" else torch.float8_e5m2
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * spread)
    return v.to(dt).view(torch.uint8).numpy()


def _stored(rng, batch, rows, cols, ld, bstride, fmt):
    """A padded device buffer holding `batch` [rows][cols] fp8 matrices at row stride `ld`
    and batch stride `bstride`; padding bytes are NaN codes."""
    total = (batch - 1) * bstride + rows * ld if batch > 0 else 0
    buf = np.full(max(total, 16) + 64, NAN_CODE, np.uint8)
    logical = _codes(rng, (batch, rows, cols), fmt)
    for b in range(batch):
        for r in range(rows):
            o = b * bstride + r * ld
            buf[o:o + cols] = logical[b, r]
    return torch.from_numpy(buf).to(DEV), logical


def _run(layout, fmt_a, fmt_b, m, n, k, batch=1, bcast=None, pad=16, bias="bf16", seed=0, sa=1.25, sb=0.75):
    rng = np.random.default_rng(seed)
    a_rows, a_cols = (m, k) if layout[0] == "N" else (k, m)
    b_rows, b_cols = (n, k) if layout[1] == "T" else (k, n)
    lda = (a_cols + 15) // 16 * 16 + pad
    ldb = (b_cols + 15) // 16 * 16 + pad
    ba = 1 if bcast == "a" else batch
    bb = 1 if bcast == "b" else batch
    sta = 0 if ba == 1 else a_rows * lda + 32
    stb = 0 if bb == 1 else b_rows * ldb + 48
    a_dev, a_log = _stored(rng, ba, a_rows, a_cols, lda, sta, fmt_a)
    b_dev, b_log = _stored(rng, bb, b_rows, b_cols, ldb, stb, fmt_b)
    ldo = n + 8
    sto = m * ldo + 24
    out = torch.full((batch * sto + 64,), 0x7FC1, dtype=torch.int16, device=DEV)  # NaN canary
    sa_t = torch.tensor([sa], device=DEV)
    sb_t = torch.tensor([sb], device=DEV)
    bias_t = bias_s = None
    bias_np = bias_scale = None
    if bias == "bf16":
        bt = torch.from_numpy(rng.standard_normal(n).astype(np.float32) * 0.5).to(torch.bfloat16)
        bias_t, bias_np = bt.to(DEV), np_bf16_bits(bt)
    elif bias == "fp8":
        bias_np = _codes(rng, (n,), fmt_a)
        bias_t = torch.from_numpy(bias_np).to(DEV)
        bias_scale = 0.375
        bias_s = torch.tensor([bias_scale], device=DEV)
    F.fp8_gemm(a_dev, b_dev, FMT[fmt_a], FMT[fmt_b], LAYOUTS[layout], m, n, k, lda, ldb, ldo, batch, sta, stb, sto,
               sa_t, sb_t, bias_t, bias_s, out)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    o = out.cpu().numpy().view(np.uint16)
    got = np.zeros((batch, m, n))
    for b in range(batch):
        blk = o[b * sto: b * sto + m * ldo].reshape(m, ldo) if m > 0 else np.zeros((0, ldo), np.uint16)
        got[b] = C.bf16_bits_to_f64(blk[:, :n])
        assert np.all(blk[:, n:] == 0x7FC1), "wrote past n"
    ref, s_abs, sc = G.gemm_ref(a_log, b_log, layout, fmt_a, fmt_b, sa, sb, bias_np, bias_scale)
    ref = np.broadcast_to(ref, (batch, m, n))
    s_abs = np.broadcast_to(s_abs, (batch, m, n))
    return assert_within_gemm_bound(got, ref, s_abs, sc, f"{layout} {fmt_a}x{fmt_b} {m}x{n}x{k} b{batch}")


SHAPES = [(128, 256, 128), (200, 300, 176), (64, 16, 32), (1, 16, 16), (129, 264, 1040), (384, 640, 512),
          (256, 128, 4096)]


@pytest.mark.parametrize("layout", ["NT", "NN", "TN", "TT"])
@pytest.mark.parametrize("fmts", [("e4m3", "e4m3"), ("e5m2", "e5m2"), ("e5m2", "e4m3")])
def test_layouts_formats_shapes(layout, fmts):
    for i, (m, n, k) in enumerate(SHAPES):
        _run(layout, fmts[0], fmts[1], m, n, k, seed=i)


@pytest.mark.parametrize("bias", [None, "bf16", "fp8"])
def test_bias_kinds(bias):
    _run("NT", "e4m3", "e4m3", 160, 272, 256, bias=bias, seed=3)
    _run("NT", "e5m2", "e5m2", 96, 48, 64, bias=bias, seed=4)


@pytest.mark.parametrize("bcast", [None, "a", "b"])
@pytest.mark.parametrize("layout", ["NT", "NN", "TN"])
def test_batched_and_broadcast(bcast, layout):
    _run(layout, "e4m3", "e4m3", 130, 200, 160, batch=3, bcast=bcast, seed=7)


@pytest.mark.parametrize("layout", ["NT", "TN"])
def test_last_round_half_tiles(layout):
    """80 pair tiles of 256 x 256 on the 74 pairs of a B200: the last round's 6 tiles run as 12
    halves of 256 x 128 (K-major B).  Ragged M and N: the last tile column holds 96 valid
    columns, so one of its halves lies wholly past n (nothing may be written there)."""
    _run(layout, "e4m3", "e4m3", 2000, 2400, 384, bias="bf16", seed=21)


@pytest.mark.parametrize("layout", ["NT", "TN"])
def test_wide_pair_tiles(layout):
    """A problem large enough for 256 x 512 pair tiles (two N = 256 MMAs per K step into one
    512-column accumulator): ragged M and N, so the last tile column holds 416 valid columns and
    its second MMA half is partly past n."""
    _run(layout, "e4m3", "e4m3", 4000, 4000, 2048, bias="bf16", seed=23)


def test_k_zero_writes_bias():
    _run("NT", "e4m3", "e4m3", 70, 90, 0, bias="bf16")
    _run("NT", "e4m3", "e4m3", 70, 90, 0, bias=None)


def test_empty_m_n_are_noops():
    out = torch.full((16,), 7, dtype=torch.int16, device=DEV)
    one = torch.ones(1, device=DEV)
    F.fp8_gemm(None, None, 0, 0, 0, 0, 16, 16, 16, 16, 16, 1, 0, 0, 0, one, one, None, None, out)
    # an output without elements may be NULL (m = 0, n = 0 or batch = 0)
    F.fp8_gemm(None, None, 0, 0, 0, 0, 16, 16, 16, 16, 16, 1, 0, 0, 0, one, one, None, None, None)
    F.fp8_gemm(None, None, 0, 0, 0, 16, 0, 16, 16, 16, 16, 1, 0, 0, 0, one, one, None, None, None)
    torch.cuda.synchronize()
    assert int(out[0]) == 7
    assert F.fp8_get_device_status() == 0


def test_accumulation_precision_k_sweep():
    """Adversarial cancellation: half of each dot product is the negation of the other half,
    so |ref| << S_abs and the error is pure accumulation error.  Reports and bounds
    max |gpu - ref| / (S_abs * sc) against the 2^-20 term."""
    worst = 0.0
    for k in (256, 1024, 4096, 8192):
        rng = np.random.default_rng(k)
        m, n = 128, 256
        half = _codes(rng, (m, k // 2), "e4m3", spread=8.0)
        a = np.concatenate([half, half ^ 0x80], axis=1)  # second half negated
        perm = rng.permutation(k)
        a = np.ascontiguousarray(a[:, perm])
        bh = _codes(rng, (n, k // 2), "e4m3", spread=8.0)
        bfull = np.concatenate([bh, bh], axis=1)[:, perm]
        # perturb a few b entries so sums are not exactly zero
        bfull[:, :8] = _codes(rng, (n, 8), "e4m3")
        bfull = np.ascontiguousarray(bfull)
        out = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
        one = torch.ones(1, device=DEV)
        F.fp8_gemm(torch.from_numpy(a).to(DEV), torch.from_numpy(bfull).to(DEV), 0, 0, F.FP8_LAYOUT_NT, m, n, k, k, k,
                   n, 1, 0, 0, 0, one, one, None, None, out)
        torch.cuda.synchronize()
        ref, s_abs, sc = G.gemm_ref(a, bfull, "NT", "e4m3", "e4m3", 1.0, 1.0)
        got = bf16_out_to_f64(out)
        # remove the bf16 output rounding allowance, keep the accumulation part
        acc_err = np.maximum(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref), 0.0)
        ratio = float(np.max(acc_err / np.maximum(s_abs, 1e-30)))
        worst = max(worst, ratio)
        assert_within_gemm_bound(got, ref, s_abs, sc, f"cancellation K={k}")
    print(f"max accumulation error / S_abs = {worst:.3e} (bound {2.0 ** -20:.3e})")


def _sampled_check(a_dev, b_dev, layout, fmt, m, n, k, sa, sb, bias_t, out, batch=1, bcast_b=False, samples=512,
                   seed=0):
    """Compare `samples` random outputs with the oracle computed one by one."""
    rng = np.random.default_rng(seed)
    o = np_bf16_bits(out).reshape(batch, m, n)
    bias_np = np_bf16_bits(bias_t) if bias_t is not None else None
    a_all = a_dev.view(-1)
    b_all = b_dev.view(-1)
    for _ in range(samples):
        bi = int(rng.integers(batch))
        i = int(rng.integers(m))
        j = int(rng.integers(n))
        arow = np_u8(a_all[(bi * m + i) * k:(bi * m + i + 1) * k]).reshape(1, k)
        bb = 0 if bcast_b else bi
        bcol = np_u8(b_all[(bb * n + j) * k:(bb * n + j + 1) * k]).reshape(1, k)
        ref, s_abs, sc = G.gemm_ref(arow, bcol, "NT", fmt, fmt, sa, sb,
                                    None if bias_np is None else bias_np[j:j + 1])
        got = C.bf16_bits_to_f64(o[bi, i, j:j + 1])
        assert_within_gemm_bound(got.reshape(1, 1), ref, s_abs, sc, f"sample ({bi},{i},{j})")


@pytest.mark.parametrize("size", W.SQUARE_SIZES)
def test_square_full_size(size):
    """Square NT sweep, pre-quantized E4M3 from N(0,1), scales U(0.5, 2), bias on.  Every
    output is compared with the oracle up to 4096^3 (the oracle's fp64 product takes seconds
    there); 8192^3 is checked on sampled outputs."""
    m = n = k = size
    a = W.fp8_bytes((m, k), seed=11, device=DEV)
    b = W.fp8_bytes((n, k), seed=12, device=DEV)
    sa, sb = [float(v) for v in W.uniform(0.5, 2.0, seed=13, n=2)]
    bias = W.normal_bf16((n,), 0.1, seed=14, device=DEV)
    out = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    F.fp8_gemm(a, b, 0, 0, F.FP8_LAYOUT_NT, m, n, k, k, k, n, 1, 0, 0, 0, torch.tensor([sa], device=DEV),
               torch.tensor([sb], device=DEV), bias, None, out)
    torch.cuda.synchronize()
    if size <= 4096:
        ref, s_abs, sc = G.gemm_ref(np_u8(a).reshape(m, k), np_u8(b).reshape(n, k), "NT", "e4m3", "e4m3", sa, sb,
                                    np_bf16_bits(bias))
        assert_within_gemm_bound(bf16_out_to_f64(out), ref, s_abs, sc, f"square {size}")
    else:
        _sampled_check(a, b, "NT", "e4m3", m, n, k, sa, sb, bias, out, samples=256, seed=size)


@pytest.mark.parametrize("ba,bb,m,n,k", W.SKINNY_BATCHED)
def test_skinny_batched_full_size(ba, bb, m, n, k):
    batch = max(ba, bb)
    a, sa = W.amax_scaled_fp8_bytes((ba, m, k), seed=21, device=DEV)
    b, sb = W.amax_scaled_fp8_bytes((bb, n, k), seed=22, device=DEV)
    out = torch.empty((batch, m, n), dtype=torch.bfloat16, device=DEV)
    F.fp8_gemm(a, b, 0, 0, F.FP8_LAYOUT_NT, m, n, k, k, k, n, batch, 0 if ba == 1 else m * k,
               0 if bb == 1 else n * k, m * n, torch.tensor([sa], device=DEV), torch.tensor([sb], device=DEV), None,
               None, out)
    torch.cuda.synchronize()
    # every output against the oracle (at most 69 GFLOP of fp64 products on the host)
    ref, s_abs, sc = G.gemm_ref(np_u8(a).reshape(ba, m, k), np_u8(b).reshape(bb, n, k), "NT", "e4m3", "e4m3", sa, sb)
    assert_within_gemm_bound(bf16_out_to_f64(out), ref, s_abs, sc, f"{batch}x{m}x{n}x{k}")


def test_gemm_deterministic():
    rng = np.random.default_rng(1)
    a = torch.from_numpy(_codes(rng, (512, 1024), "e4m3")).to(DEV)
    b = torch.from_numpy(_codes(rng, (768, 1024), "e4m3")).to(DEV)
    one = torch.ones(1, device=DEV)
    outs = []
    for _ in range(3):
        out = torch.empty((512, 768), dtype=torch.bfloat16, device=DEV)
        F.fp8_gemm(a, b, 0, 0, 0, 512, 768, 1024, 1024, 1024, 768, 1, 0, 0, 0, one, one, None, None, out)
        torch.cuda.synchronize()
        outs.append(np_bf16_bits(out))
    assert all(np.array_equal(o, outs[0]) for o in outs)

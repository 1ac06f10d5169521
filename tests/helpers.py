"""Test utilities: tensor <-> numpy views and the parity comparisons (no method arithmetic)."""

import numpy as np
import torch

from oracle import fp8_codec as C
from oracle import gemm as G


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def np_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def np_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().astype(np.float32)


def bf16_out_to_f64(t: torch.Tensor) -> np.ndarray:
    return C.bf16_bits_to_f64(np_bf16_bits(t))


def in_values_f32(t: torch.Tensor) -> np.ndarray:
    """The input tensor's values as fp32 (exact for bf16 / f16 / f32)."""
    return t.detach().cpu().float().numpy()


def assert_within_gemm_bound(gpu_f64, ref64, s_abs, sc, what=""):
    tol = G.gemm_tolerance(ref64, s_abs, sc)
    err = np.abs(gpu_f64 - ref64)
    # a NaN where the reference has a number (an output never written, say) is outside the
    # bound too: comparisons with NaN are false, so test for "inside" and negate
    both_nan = np.isnan(gpu_f64) & np.isnan(ref64)
    bad = ~(err <= tol) & ~both_nan
    if bad.any():
        idx = np.argwhere(bad)[:5]
        msg = "; ".join(f"{tuple(i)}: gpu={gpu_f64[tuple(i)]!r} ref={ref64[tuple(i)]!r} tol={tol[tuple(i)]!r}"
                        for i in idx)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside the bound; {msg}")
    return float(np.max(err / np.maximum(tol, 1e-300))) if err.size else 0.0


def assert_bf16_within_ulp(gpu_bits, ref_values, ulps=1, what=""):
    """bf16 results within `ulps` bf16 units of the oracle's bf16-rounded value."""
    g = C.bf16_bits_to_f64(gpu_bits)
    r = C.round_to_bf16(ref_values)
    ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(r), 1e-38))[1] - 8)
    bad = ~(np.abs(g - r) <= ulps * ulp) & ~(np.isnan(g) & np.isnan(r))  # a stray NaN counts as a miss
    assert not bad.any(), f"{what}: {int(bad.sum())} values differ by more than {ulps} bf16 ulp"

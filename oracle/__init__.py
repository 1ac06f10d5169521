"""Plain, slow CPU oracle for the FP8 linear layer with per-tensor delayed scaling.

This package is TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference`` arm) may import
it.  The product library never calls it, and it shares no code, header, table or
constant generator with the CUDA path under ``fp8_delayed_scaling_amax_b200/``.

Everything here is written from the AstrAI pages (commit logs and the compare view
``3e57cc8...main`` of ``astrai/extension/fp8.py``, ``astrai/extension/ops/fp8.py``
and ``csrc/kernels/fp8/*``) and from the IEEE / OCP FP8 format definitions:

=====================  ======================================================
module                 what it computes
=====================  ======================================================
``fp8_codec``          E4M3FN / E5M2 decode tables from the bit-field
                       definition; round-to-nearest-even encode with
                       saturation to +-FP8_MAX; bf16 decode/encode.
``quantize``           ``x8 = q(RN32(x * RN32(1/s)))`` and the raw-domain amax,
                       row-major, transposed and dual orientations.
``scaling``            the scale formula ``max(RN32(peak/fp8_max)/2^m, 1e-12)``,
                       the history ring ``[hist n | scale | scale_used | amax |
                       done]`` and its last-block fold, seed and dynamic scale.
``gemm``               dequantized GEMM accumulated in fp64, scaled by
                       ``RN32(sa*sb)``, plus bias (bf16, or fp8 * bias_scale);
                       returns the unrounded fp64 result and ``sum|a*b|`` for
                       the error bound.
``linear``             forward / dX / dW compositions (delayed and dynamic).
=====================  ======================================================

Parity pins (``tests/test_oracle_*.py``, all ``-m "not gpu"``) tie every function
to something other than itself: the 256-code round trip, midpoints that must
round to the even code, agreement with PyTorch's own float8 casts inside the
non-saturating range, the FP8_MAX constants printed on the pages, closed-form
ring windows, the no-scale-leak invariant, and a brute-force exact-rational
triple loop for the GEMM on tiny shapes.
"""

"""CPU oracle for the block-scaled MXFP4 matrix product (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the library calls this module; only the test suite and
the benchmark's CPU-baseline leg may import it. It shares no code with the CUDA sources.

What it follows: the MX block format of the "Quantization Error" page (section "Where the
error comes from": each element is one E2M1 grid value times its block's exact power-of-two
scale), applied to both operands of a matrix product with blocks of 32 along the contraction
axis (the K-major W4A4 layout). The plain definition:

    C[m, n] = sum_k dq(A)[m, k] * dq(B)[n, k]

written out as exact dequantization of both operands followed by one fp64 matrix product (a
library routine as a single step; no blocking or reordering beyond it). Every dequantized value
is a short dyadic number, so the fp64 product is exact up to the rounding of the running sum.

Operands are in the library's canonical layout: codes [R, K/2] bytes (element 2i in the low
nibble), E8M0 scales [R, K/32].
"""
from __future__ import annotations

import numpy as np

from . import mxfp4 as mx
from . import nvfp4 as nv


def mxgemm(a_codes, a_scales, b_codes, b_scales, K: int) -> np.ndarray:
    """C = dq(A) dq(B)^T in fp64 for A [M, K] and B [N, K] in MXFP4."""
    ad = mx.dequantize_rows(a_codes, a_scales, K)
    bd = mx.dequantize_rows(b_codes, b_scales, K)
    return ad @ bd.T


def mxgemm_abs(a_codes, a_scales, b_codes, b_scales, K: int) -> np.ndarray:
    """|dq(A)| |dq(B)|^T: the size of the terms each C[m, n] sums (sets fp32 error bounds)."""
    ad = np.abs(mx.dequantize_rows(a_codes, a_scales, K))
    bd = np.abs(mx.dequantize_rows(b_codes, b_scales, K))
    return ad @ bd.T


def nvgemm(a_codes, a_scales, b_codes, b_scales, K: int) -> np.ndarray:
    """C = dq(A) dq(B)^T in fp64 for A [M, K] and B [N, K] in NVFP4 (blocks of 16, E4M3 scales)."""
    return nv.dequantize_rows(a_codes, a_scales, K) @ nv.dequantize_rows(b_codes, b_scales, K).T


def nvgemm_abs(a_codes, a_scales, b_codes, b_scales, K: int) -> np.ndarray:
    return np.abs(nv.dequantize_rows(a_codes, a_scales, K)) @ np.abs(nv.dequantize_rows(b_codes, b_scales, K)).T

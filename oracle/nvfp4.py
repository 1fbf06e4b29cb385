"""CPU oracle for NVFP4 block quantization (fp64 numpy), the comparison format the MXAttention
abstract measures MXFP4 attention against ("competitive with strong NVFP4-based baselines").

TEST INFRASTRUCTURE ONLY. Nothing in the library calls this module; only the test suite may
import it. It shares no code with the CUDA sources.

The pages name NVFP4 but give no recipe. Reading taken (also listed in the design notes): the
plainest block-scaled form with NVFP4's parameters --
  * blocks of 16 elements along the contraction axis, E2M1 elements (the same grid as MXFP4);
  * one unsigned FP8 E4M3 scale per block (OCP FP8: bias 7, 3 mantissa bits, subnormals down to
    2^-9, no infinities, 0x7F = NaN, largest finite 448), s = E4M3(amax / 6), rounded to
    nearest-even and saturated at 448, so the block maximum lands on the top grid value;
  * no second, tensor-level scale;
  * elements y = x / s rounded to nearest-even on the E2M1 grid, saturating at 6; a block whose
    scale rounds to 0 encodes as all-zero codes.
Decision precision: amax / 6 and x / s are taken as correctly rounded fp32 quotients (the
precision a GPU kernel computes them in), then rounded onto the E4M3 / E2M1 grids. For fp32
operands the fp64 quotient rounded once to fp32 is the correctly rounded fp32 quotient.
"""
from __future__ import annotations

import numpy as np

from . import mxfp4 as mx

BLOCK = 16
SCALE_NVFP4 = 2          # the attention oracle's mode number for this format (MXFP4: OCP 0, UOS 1)
E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_decode(codes) -> np.ndarray:
    """Unsigned E4M3 byte -> value (0x7F and 0xFF -> NaN; the sign bit gives a negative value)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((c & 0x7F) == E4M3_NAN, np.nan, val)
    return sign * val


def e4m3_encode(v) -> np.ndarray:
    """Non-negative finite value -> E4M3 byte, round to nearest with ties to the even mantissa,
    saturating at 448 (0x7E)."""
    v = np.asarray(v, dtype=np.float64)
    assert np.all(v >= 0) and np.all(np.isfinite(v))
    out = np.zeros(v.shape, dtype=np.int64)
    pos = v > 0
    _, ex = np.frexp(np.where(pos, v, 1.0))
    e = ex - 1                                            # floor(log2 v)
    sub = pos & (e < -6)
    # subnormal range: multiples of 2^-9
    qs = np.round(np.where(sub, v, 0.0) * 2.0 ** 9)       # np.round: half to even
    out = np.where(sub, qs.astype(np.int64), out)        # 8 -> 0x08, the smallest normal
    nrm = pos & ~sub
    frac = np.where(nrm, v, 1.0) / np.exp2(np.where(nrm, e, 0)) - 1.0   # [0, 1)
    q = np.round(frac * 8.0).astype(np.int64)
    e2 = np.where(q == 8, e + 1, e)
    q = np.where(q == 8, 0, q)
    code = ((e2 + 7) << 3) | q
    out = np.where(nrm, code, out)
    return np.minimum(out, 0x7E)


def _fp32_div(a, b) -> np.ndarray:
    with np.errstate(divide="ignore", invalid="ignore"):
        return (np.asarray(a, dtype=np.float64) / np.asarray(b, dtype=np.float64)).astype(np.float32).astype(np.float64)


def quantize_blocks(xb):
    """xb [..., 16] -> (codes [..., 16] uint8 sign|index, scale bytes [...])."""
    xb = np.asarray(xb, dtype=np.float64)
    amax = np.abs(xb).max(axis=-1)
    sbyte = e4m3_encode(_fp32_div(amax, 6.0))
    s = e4m3_decode(sbyte)
    y = _fp32_div(xb, s[..., None])
    y = np.where((s > 0)[..., None], y, 0.0)
    return mx.e2m1_encode(y), sbyte.astype(np.uint8)


def quantize_rows(x):
    """Blocks of 16 along the last axis: codes [..., ceil(C/16)*8] (element 2i in the low nibble),
    E4M3 scale bytes [..., ceil(C/16)]."""
    x = np.asarray(x, dtype=np.float64)
    C = x.shape[-1]
    pad = (-C) % BLOCK
    if pad:
        x = np.concatenate([x, np.zeros(x.shape[:-1] + (pad,))], axis=-1)
    xb = x.reshape(x.shape[:-1] + (x.shape[-1] // BLOCK, BLOCK))
    codes, sbytes = quantize_blocks(xb)
    return mx.pack_nibbles(codes.reshape(x.shape)), sbytes


def dequantize_rows(codes, scales, C: int | None = None) -> np.ndarray:
    vals = mx.e2m1_decode(mx.unpack_nibbles(codes))
    s = e4m3_decode(scales)
    vb = vals.reshape(vals.shape[:-1] + (vals.shape[-1] // BLOCK, BLOCK)) * s[..., None]
    out = vb.reshape(vals.shape)
    return out if C is None else out[..., :C]

"""CPU oracle for the MXFP4 format and its block quantizer (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the library calls this module; only the test
suite, the package smoke check and the benchmark's CPU-baseline leg may import it.
It shares no code, tables or constants with the CUDA sources.

What it follows
---------------
* MXFP4 element: E2M1, a sign bit and eight magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}
  ("Quantization Error" page, section "Where the error comes from": the grid is
  linear below 1.0 and geometric above it, spacing 0.5 in [1, 1.5], spacing 2.0
  between 4.0 and 6.0). Bit layout sign<<3 | {exponent:2, mantissa:1} with bias 1,
  and saturation at 6, follow the OCP Microscaling Formats (MX) v1.0 specification.
* Rounding: round to nearest, ties to the even code (RTNE). The page's worst cases
  (5.0 -> 4.0 and 1.25 -> 1.0, both 20% relative error) are exactly RTNE's ties.
* Shared scale: one E8M0 power of two per 32-element block, applied exactly (same
  page: "The scale is a power of two and applies exactly", no dependence on block
  order). E8M0 byte = exponent + 127; byte 0xFF (NaN) is never produced.
* Scale rules (MXAttention abstract: "the clipping-underflow trade-off from
  power-of-two scaling"; Universal Optimal Scaling with boundary Qmax = 7.25):
    - OCP:  e = floor(log2 amax) - 2, so amax / 2^e lies in [4, 8) and values above 6
      saturate (the OCP MX v1.0 rule, the paper's baseline).
    - UOS:  the smallest integer e with amax / 2^e <= 7.25.
  Readings taken where the pages are silent: an all-zero block gets byte 0x00 (e = -127)
  and all-zero codes; exponents are clamped to [-127, 127]; a value that rounds to zero
  keeps its sign bit (code 0x8 for a negative input), IEEE style; a partial last block
  is zero-padded, and the padding never raises amax and encodes as +0.

Layout conventions (the library's canonical layout)
---------------------------------------------------
Blocks run along the last axis. Codes are packed two per byte, element 2i in the low
nibble and element 2i+1 in the high nibble: ``codes[..., ceil(C/32)*16]`` (uint8).
Scales are one byte per block: ``scales[..., ceil(C/32)]`` (uint8).

Every function here is pinned by tests/test_oracle_pins.py against values printed on
the pages, closed forms, brute force and invariants.
"""
from __future__ import annotations

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0
BLOCK = 32
E8M0_BIAS = 127
E_MIN, E_MAX = -127, 127
QMAX_UOS = 7.25
SCALE_OCP, SCALE_UOS = 0, 1


def e2m1_decode(codes) -> np.ndarray:
    """Value of each 4-bit code (low 4 bits of the input): (-1)^s * magnitude[k]."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    mag = E2M1_MAGNITUDES[c & 0x7]
    return np.where((c & 0x8) != 0, -mag, mag)


def e2m1_encode(y) -> np.ndarray:
    """4-bit codes of already-scaled values y (float64 array).

    Nearest of the eight magnitudes to min(|y|, 6); on an exact tie the even index
    wins (RTNE: the candidate whose mantissa bit is 0). Sign bit kept for every value,
    including those that round to zero.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), E2M1_MAX)
    dist = np.abs(a[..., None] - E2M1_MAGNITUDES)          # exact for dyadic a
    dmin = dist.min(axis=-1, keepdims=True)
    cand = dist == dmin                                    # one or two candidates
    even = (np.arange(8) % 2) == 0
    has_even = (cand & even).any(axis=-1, keepdims=True)
    pick = np.where(has_even, cand & even, cand)
    k = np.argmax(pick, axis=-1).astype(np.uint8)
    sign = np.signbit(y).astype(np.uint8)
    return (sign << 3) | k


def scale_exponent(amax, mode: int) -> np.ndarray:
    """Shared exponent e (int64) of blocks with the given amax (float64, >= 0).

    OCP: e = floor(log2 amax) - 2. UOS: the smallest e with amax / 2^e <= 7.25, i.e. the
    OCP exponent plus one exactly when amax / 2^e_ocp > 7.25. floor(log2) is read off
    frexp, which is exact. amax == 0 -> e = -127. Result clamped to [-127, 127].
    """
    amax = np.asarray(amax, dtype=np.float64)
    frac, ex = np.frexp(amax)            # amax = frac * 2^ex, frac in [0.5, 1)
    e0 = ex.astype(np.int64) - 1         # floor(log2 amax)
    e = e0 - 2
    if mode == SCALE_UOS:
        over = np.ldexp(amax, -e) > QMAX_UOS   # exact: scaling by a power of two
        e = np.where(over, e + 1, e)
    elif mode != SCALE_OCP:
        raise ValueError(f"unknown scale mode {mode}")
    e = np.where(amax == 0.0, E_MIN, e)
    return np.clip(e, E_MIN, E_MAX)


def quantize_blocks(xb, mode: int):
    """Quantize blocks xb[..., 32] (float64). Returns (codes uint8 [...,32], e int64 [...])."""
    xb = np.asarray(xb, dtype=np.float64)
    amax = np.abs(xb).max(axis=-1)
    e = scale_exponent(amax, mode)
    y = np.ldexp(xb, -e[..., None])      # x / 2^e, exact (no underflow for finite bf16 input
    #                                      except values far below the 0.25 rounding midpoint)
    return e2m1_encode(y), e


def pack_nibbles(codes) -> np.ndarray:
    """[..., 2n] 4-bit codes -> [..., n] bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def _pad_last(x: np.ndarray, mult: int) -> np.ndarray:
    C = x.shape[-1]
    Cp = -(-C // mult) * mult
    if Cp == C:
        return x
    pad = np.zeros(x.shape[:-1] + (Cp - C,), dtype=x.dtype)
    return np.concatenate([x, pad], axis=-1)


def quantize_rows(x, mode: int):
    """MXFP4-quantize along the last axis in 32-element blocks.

    x: float array [..., C] (fp32/bf16 values held in float64 or float32).
    Returns (codes uint8 [..., ceil(C/32)*16], scales uint8 [..., ceil(C/32)]).
    """
    x = _pad_last(np.asarray(x, dtype=np.float64), BLOCK)
    xb = x.reshape(x.shape[:-1] + (x.shape[-1] // BLOCK, BLOCK))
    codes, e = quantize_blocks(xb, mode)
    codes = codes.reshape(x.shape)
    return pack_nibbles(codes), (e + E8M0_BIAS).astype(np.uint8)


def dequantize_rows(codes, scales, C: int | None = None) -> np.ndarray:
    """Inverse of quantize_rows: value = e2m1(code) * 2^(scale - 127), exact in float64."""
    v = e2m1_decode(unpack_nibbles(codes))
    nb = np.asarray(scales).shape[-1]
    vb = v.reshape(v.shape[:-1] + (nb, BLOCK))
    e = np.asarray(scales).astype(np.int64) - E8M0_BIAS
    out = np.ldexp(vb, e[..., None]).reshape(v.shape)
    return out if C is None else out[..., :C]


def quantize_transposed(x, mode: int):
    """Quantize a [..., R, C] matrix in blocks of 32 along R (used for V along keys).

    Returns codes [..., C, ceil(R/32)*16] and scales [..., C, ceil(R/32)].
    """
    xt = np.swapaxes(np.asarray(x, dtype=np.float64), -1, -2)
    return quantize_rows(xt, mode)


def rel_frobenius(x, ref) -> float:
    """||x - ref||_F / ||ref||_F (the "Quantization Error" page's first error metric)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / np.linalg.norm(ref))


def block_amax_ratio(x) -> np.ndarray:
    """Per-block amax / median|x| (the page's outlier-dominance diagnostic)."""
    x = _pad_last(np.asarray(x, dtype=np.float64), BLOCK)
    xb = np.abs(x.reshape(x.shape[:-1] + (x.shape[-1] // BLOCK, BLOCK)))
    med = np.median(xb, axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        return xb.max(axis=-1) / med

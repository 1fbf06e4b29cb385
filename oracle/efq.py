"""CPU oracle for exp-free generation of the P~ operand, as EFQ-Softmax describes it (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the library calls this module; only the test suite, the
package smoke check and the benchmark's CPU-baseline leg may import it. It shares no code with
the CUDA sources.

What it follows
---------------
EFQ-Softmax abstract: instead of evaluating the shifted-score exponentials and then quantizing
them, each microscaling block of P~ gets a power-of-two scale chosen from the block's own
maximum, the shifted scores are expressed relative to that scale, and the non-negative E2M1 codes
come straight from those residuals through one affine map. The operand built this way is the one
both the numerator P~V and the denominator P~1 use; the FlashAttention loop around it (running
max, history rescale, fp accumulation, final division) is unchanged.

The abstract prints no constants. The reading taken here (each item is also in the design notes):
  * a block is 32 consecutive keys at absolute key multiples of 32 (the MXFP4 block);
  * the shifted score of key j is u_j = (s_j - m') log2(e), the base-2 logarithm of P~_j, with
    s_j = sigma <q, k_j> and m' the running max in force for the tile;
  * the exponent-only scale is the MXFP4 scale exponent e of the block (the OCP or UOS rule of
    oracle/mxfp4.py) applied to the block's largest P~, 2^max_j u_j, taken in fp32 like every
    other decision of the oracle;
  * the residual is r_j = u_j - e, the base-2 logarithm of P~_j / 2^e (at most log2 7.25 under
    UOS, below 3 under OCP);
  * the affine rule is k_j = clamp(round_half_even(2 r_j + 2), 0, 7), and the code is k_j with
    the sign bit clear. It puts two codes on every binade of the E2M1 grid and lands exactly on
    the grid values 1, 2 and 4 at r = 0, 1 and 2; below 1 it assigns 0.5 to r in (-0.75, -0.25)
    and 0 below that (the exact grid would keep 0.5 down to r = -2), so it never exceeds the
    exp-then-quantize code by more than one step, and never undercuts it by more than one.
Masked keys (u = -inf) get code 0; an all-masked block gets scale byte 0x00, as for the other
P~ rules.
"""
from __future__ import annotations

import numpy as np

from . import mxfp4 as mx

SLOPE = 2.0        # codes per binade of the residual
OFFSET = 2.0       # code of residual 0 (the grid value 1.0)


def efq_block_exponent(u_blocks: np.ndarray, mode: int) -> np.ndarray:
    """Scale exponent of each block [..., nblk, 32] of base-2 shifted scores: the MXFP4 rule of
    `mode` on the block's largest P~ = 2^max(u), rounded to fp32 (0 for an all-masked block)."""
    umax = np.max(u_blocks, axis=-1)
    with np.errstate(over="ignore"):
        amax = np.where(np.isneginf(umax), 0.0, np.exp2(umax)).astype(np.float32).astype(np.float64)
    return mx.scale_exponent(amax, mode)


def efq_residual_codes(u_blocks: np.ndarray, e: np.ndarray):
    """Affine rule on the residuals r = u - e: returns (codes uint8, the pre-rounding argument
    z = 2 r + 2 with -inf for masked keys)."""
    with np.errstate(invalid="ignore"):
        z = SLOPE * (u_blocks - e[..., None]) + OFFSET
    k = np.clip(np.rint(np.where(np.isneginf(z), -1.0, z)), 0, 7)
    return k.astype(np.uint8), z


def efq_quantize_p(u: np.ndarray, mode: int):
    """The P~ operand of one tile from base-2 shifted scores u [R, T] (T a multiple of 32).

    Returns (dequantized operand fp64 [R, T], codes [R, T], scale bytes [R, T/32], z [R, T]).
    """
    R, T = u.shape
    ub = np.asarray(u, dtype=np.float64).reshape(R, T // mx.BLOCK, mx.BLOCK)
    e = efq_block_exponent(ub, mode)
    codes, z = efq_residual_codes(ub, e)
    deq = np.ldexp(mx.e2m1_decode(codes), e[..., None]).reshape(R, T)
    return deq, codes.reshape(R, T), (e + mx.E8M0_BIAS).astype(np.uint8), z.reshape(R, T)

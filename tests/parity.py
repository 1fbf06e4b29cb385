"""Helpers shared by the GPU parity tests: tolerances, the oracle side of a run, and the
tie-aware classification of P~ code mismatches.

Tolerances (fixed before measurement):
  * Q/K/V codes and scales: bit-exact (a pure function of the bf16 input).
  * P~ codes: mismatch rate <= 1e-4, and every mismatch must sit at a rounding tie the
    fp32 arithmetic can flip: the oracle's scaled value lies within TIE_REL of an E2M1
    rounding midpoint (for the exp-free rule: its argument 2 r + 2 lies within TIE_REL times
    the magnitude of its terms of a half-integer), or the block amax lies within TIE_REL of a
    scale-exponent boundary.
    TIE_REL = 2^-15 covers the GPU's independent error sources (fp32 score accumulation in
    the tensor core, the fp32 exponent argument, ex2.approx), each a few fp32 ulps of an
    argument of magnitude up to ~100.
  * Attention output (fp32): max |gpu - oracle| <= 5e-3 and relative Frobenius <= 1e-3.
"""
from __future__ import annotations

import numpy as np

from oracle import mxfp4 as mx
from oracle import nvfp4 as nv

OUT_MAX_ABS = 5e-3
OUT_REL_FRO = 1e-3
P_MISMATCH_RATE = 1e-4
TIE_REL = 2.0 ** -15
MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def near_midpoint(y: np.ndarray) -> np.ndarray:
    a = np.abs(y)[..., None]
    return (np.abs(a - MIDPOINTS) <= TIE_REL * MIDPOINTS).any(axis=-1)


_E4M3_VALS = nv.e4m3_decode(np.arange(0x7F))
_E4M3_MIDS = (_E4M3_VALS[1:] + _E4M3_VALS[:-1]) / 2


def near_scale_boundary(amax: np.ndarray, mode: int) -> np.ndarray:
    """MXFP4: amax within TIE_REL of a power of two (both rules) or of 1.8125 * 2^k (UOS).
    NVFP4: the recorded fp32(amax / 6) within TIE_REL of an E4M3 rounding midpoint."""
    a = np.asarray(amax, dtype=np.float64)
    if mode == nv.SCALE_NVFP4:
        return (np.abs(a[..., None] - _E4M3_MIDS) <= TIE_REL * _E4M3_MIDS).any(axis=-1)
    out = np.zeros(a.shape, dtype=bool)
    pos = a > 0
    frac, ex = np.frexp(a[pos])            # a = frac * 2^ex, frac in [0.5, 1)
    sig = frac * 2.0                       # significand in [1, 2)
    near = (np.abs(sig - 1.0) <= TIE_REL) | (np.abs(sig - 2.0) <= 2 * TIE_REL)
    if mode == mx.SCALE_UOS:
        near |= np.abs(sig - 1.8125) <= TIE_REL * 1.8125
    out[pos] = near
    return out


def near_half_integer(z: np.ndarray, zmag: np.ndarray) -> np.ndarray:
    """Exp-free rule: the argument 2 r + 2 lies within TIE_REL * (magnitude of its terms) of a
    rounding boundary n + 1/2, where the kernel's fp32 arithmetic can take the other side."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        d = np.abs(z - np.floor(z) - 0.5)
    return np.isfinite(z) & (d <= TIE_REL * np.asarray(zmag, dtype=np.float64))


def classify_p_mismatches(gpu_codes, gpu_scales, rec, mode, n_valid):
    """Compare GPU P~ dumps with the oracle's record for the same rows.

    gpu_codes [R, Npad/2] packed, gpu_scales [R, Npad/blk] (blk = 32, or 16 for NVFP4); rec from
    attention_rows(record_p=True). Returns dict(rate, n, mismatches, unexplained, scale_mismatch_blocks).
    """
    bs = nv.BLOCK if mode == nv.SCALE_NVFP4 else mx.BLOCK
    g = mx.unpack_nibbles(np.asarray(gpu_codes))[:, :n_valid]
    o = rec["codes"][:, :n_valid]
    nb_valid = -(-n_valid // bs)
    gs = np.asarray(gpu_scales)[:, :nb_valid]
    os_ = rec["scales"][:, :nb_valid]
    code_mis = g != o
    blk = np.repeat(np.arange(nb_valid), bs)[:n_valid]
    scale_mis_blk = gs != os_
    explained_blk = near_scale_boundary(rec["amax"][:, :nb_valid], mode)
    if rec.get("rule", 1) == 2:
        near = near_half_integer(rec["z"][:, :n_valid], rec["zmag"][:, :n_valid])
    else:
        near = near_midpoint(rec["y"][:, :n_valid])
    explained = near | explained_blk[:, blk]
    unexplained = (code_mis & ~explained) | (scale_mis_blk & ~explained_blk)[:, blk]
    return dict(rate=float(code_mis.mean()), n=int(code_mis.size), mismatches=int(code_mis.sum()),
                unexplained=int(unexplained.sum()), scale_mismatch_blocks=int(scale_mis_blk.sum()))


def out_errors(gpu_out, ref_out):
    g = np.asarray(gpu_out, dtype=np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    return float(np.max(np.abs(g - r))), mx.rel_frobenius(g, r)


def ws_offsets(B, Hq, Hkv, N, d):
    """Byte offsets of the workspace regions (mirrors the library's documented carving)."""
    up = lambda x, a: -(-x // a) * a  # noqa: E731
    npad = up(N, 128)
    t = npad // 128
    off = 1024
    names = ["qc", "qs", "kc", "ks", "vc", "vs"]
    qk_atoms = d // 64 if d >= 128 else 1
    sizes = [B * Hq * npad * d // 2, B * Hq * t * qk_atoms * 512, B * Hkv * npad * d // 2,
             B * Hkv * t * qk_atoms * 512, B * Hkv * d * npad // 2, B * Hkv * t * 1024]
    res = {}
    for n, s in zip(names, sizes):
        res[n] = (off, s)
        off = up(off + s, 1024)
    res["total"] = off
    res["npad"] = npad
    return res


def atom_to_rowmajor(atoms: np.ndarray, heads: int, rows_pad: int, nblk: int) -> np.ndarray:
    """Undo the tensor-core scale atom layout: [heads][rows_pad/128][512] -> [heads][rows_pad][nblk]."""
    a = np.asarray(atoms).reshape(heads, rows_pad // 128, 512)
    r = np.arange(128)
    out = np.empty((heads, rows_pad, nblk), dtype=np.uint8)
    for k in range(nblk):
        off = (r % 32) * 16 + (r // 32) * 4 + k
        out[:, :, k] = a[:, :, off].reshape(heads, rows_pad)
    return out

"""Reading R20: the attention kernel takes the E8M0 byte of each P~ block from the base-2
logarithm d of the block maximum (amax = 2^d <= 1) rather than from amax itself:
floor(d) - 2, plus one under UOS when the fraction d - floor(d) exceeds log2(1.8125) rounded to
fp32, clamped at 0. This file restates that rule in numpy (as the kernel evaluates it: floor(d)
exactly, the fraction exactly, one fp32 comparison) and checks it against the oracle's scale rule
(oracle/mxfp4.scale_exponent) applied to amax = fp32(2^d), the precision the P~ decisions are
taken in, over random d, every integer, the fp32 neighbours of every integer and of every UOS
boundary, and values far below the E8M0 range. No GPU involved.

The two can differ only where fp32(2^d) itself sits on a scale boundary (d just below 0, whose
2^d rounds up to 1.0; d within an ulp of a UOS boundary, whose 2^d rounds onto 1.8125 * 2^k):
every difference must lie in the band the GPU parity check treats as a scale tie
(tests/parity.near_scale_boundary), and differences must be rare.
"""
import numpy as np
import pytest

from oracle import mxfp4 as mx
from tests import parity

LOG2_UOS_LIMIT = np.float32(float.fromhex("0x1.b74948p-1"))   # log2(1.8125) rounded to fp32


def byte_from_log2(d: np.ndarray, mode: int) -> np.ndarray:
    """The kernel's rule on fp32 d <= 0 (d = -inf for an all-masked block)."""
    dc = np.maximum(np.asarray(d, dtype=np.float32), np.float32(-160.0))
    fl = np.floor(dc.astype(np.float64))                       # exact for |d| < 2^22
    frac = (dc.astype(np.float64) - fl).astype(np.float32)     # exact (Sterbenz)
    bump = (mode == mx.SCALE_UOS) & (frac > LOG2_UOS_LIMIT)
    return np.maximum(fl.astype(np.int64) + 125 + bump, 0)


def byte_from_oracle(d: np.ndarray, mode: int) -> np.ndarray:
    with np.errstate(under="ignore"):
        amax = np.exp2(np.asarray(d, dtype=np.float32).astype(np.float64)).astype(np.float32).astype(np.float64)
    return mx.scale_exponent(amax, mode) + mx.E8M0_BIAS


def sample_d() -> np.ndarray:
    rng = np.random.default_rng(11)
    ints = -np.arange(0, 150, dtype=np.float64)
    uos = ints - 1.0 + np.log2(1.8125)
    pts = np.concatenate([ints, uos])
    around = np.concatenate([np.nextafter(pts.astype(np.float32), np.float32(-np.inf)),
                             np.nextafter(pts.astype(np.float32), np.float32(np.inf)), pts.astype(np.float32)])
    d = np.concatenate([rng.uniform(-150.0, 0.0, 500_000).astype(np.float32), around,
                        np.float32([-200.0, -1e30, -np.inf, -0.0, 0.0])])
    return np.minimum(d, np.float32(0.0))


def _amax(d):
    with np.errstate(under="ignore"):
        return np.exp2(np.asarray(d, dtype=np.float32).astype(np.float64)).astype(np.float32).astype(np.float64)


def _unexplained(got, d, mode):
    want = byte_from_oracle(d, mode)
    diff = got != want
    return diff, diff & ~parity.near_scale_boundary(_amax(d), mode)


@pytest.mark.parametrize("mode", [mx.SCALE_OCP, mx.SCALE_UOS])
def test_log_domain_byte_matches_the_scale_rule(mode):
    d = sample_d()
    diff, unexplained = _unexplained(byte_from_log2(d, mode), d, mode)
    assert not unexplained.any(), d[unexplained][:10]
    assert diff.sum() <= 4, d[diff]


@pytest.mark.parametrize("name", ["offset_124", "threshold_log2_1.75", "floor_as_round"])
def test_planted_mistakes_are_caught(name):
    d = sample_d()
    dc = np.maximum(d, np.float32(-160.0))
    fl = np.floor(dc.astype(np.float64))
    frac = (dc.astype(np.float64) - fl).astype(np.float32)
    if name == "offset_124":
        wrong = np.maximum(fl.astype(np.int64) + 124 + (frac > LOG2_UOS_LIMIT), 0)
    elif name == "threshold_log2_1.75":
        wrong = np.maximum(fl.astype(np.int64) + 125 + (frac > np.float32(np.log2(1.75))), 0)
    else:
        r = np.round(dc.astype(np.float64))
        fr = (dc.astype(np.float64) - r).astype(np.float32)
        wrong = np.maximum(r.astype(np.int64) + 125 + (fr > LOG2_UOS_LIMIT), 0)
    _, unexplained = _unexplained(wrong, d, mx.SCALE_UOS)
    assert unexplained.any()

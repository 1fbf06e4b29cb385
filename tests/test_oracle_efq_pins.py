"""Pins of the exp-free P~ rule (oracle/efq.py, the reading of the EFQ-Softmax abstract).

What pins it, other than itself:
  * the E2M1 grid of the "Quantization Error" page through the already-pinned exp-then-quantize
    encoder (oracle/mxfp4.e2m1_encode): the exp-free code never differs from the code of
    exp-then-quantize by more than one grid step, agrees with it away from the two rules'
    thresholds, and reproduces P~ exactly where P~ / 2^e is 1, 2 or 4;
  * a brute-force search for the scale exponent (smallest e with amax / 2^e <= 7.25 under UOS);
  * monotonicity in the score, saturation at 6, underflow to 0, round-half-even ties;
  * inside the attention loop, the property the abstract asks of the operand: it feeds the
    numerator and the denominator alike, so V = 1 gives out = 1 to rounding, and all-equal
    scores give the mean of the values.
Planted mistakes (slope, offset, tie rule, missing clamp, scale from the wrong end, exponent off
by one) each fail at least one of these checks.
"""
import types

import numpy as np
import pytest

from oracle import attention as oa
from oracle import efq
from oracle import mxfp4 as mx


def _impl():
    return types.SimpleNamespace(block_exponent=efq.efq_block_exponent, residual_codes=efq.efq_residual_codes)


def _quantize(impl, u, mode):
    """One tile through an implementation: u [R, T] -> (dequantized, codes, exponents)."""
    R, T = u.shape
    ub = u.reshape(R, T // 32, 32)
    e = impl.block_exponent(ub, mode)
    codes, _ = impl.residual_codes(ub, e)
    deq = np.ldexp(mx.e2m1_decode(codes), np.asarray(e)[..., None]).reshape(R, T)
    return deq, np.asarray(codes).reshape(R, T), np.asarray(e)


def _block_with_max(umax, rest):
    """A 32-key block whose largest base-2 shifted score is umax, the others `rest` (<= umax)."""
    u = np.full(32, -np.inf)
    u[0] = umax
    u[1:1 + len(rest)] = rest
    return u


def check_grid_points(impl):
    # block max at e0 + 2 fixes the UOS (and OCP) exponent at e0; then r = 0, 1, 2 are exact
    for e0 in (-30, -5, -2, 0, 7):
        u = _block_with_max(e0 + 2.0, [e0 + 0.0, e0 + 1.0, e0 + 2.0])[None, :]
        for mode in (mx.SCALE_UOS, mx.SCALE_OCP):
            deq, codes, e = _quantize(impl, u, mode)
            assert int(e[0, 0]) == e0
            assert np.array_equal(deq[0, 1:4], np.exp2([e0, e0 + 1.0, e0 + 2.0]))
            assert list(codes[0, 1:4]) == [2, 4, 6]


def _uos_exponent_brute(amax):
    es = np.arange(-140, 141)
    ok = np.ldexp(amax, -es) <= 7.25
    return int(es[ok].min())


def check_scale_exponent_brute_force(impl):
    rng = np.random.default_rng(7)
    for umax in np.concatenate([rng.uniform(-60, 0, 200), [0.0, -1.0, -2.857, -2.858, np.log2(7.25) - 3]]):
        amax = float(np.float32(2.0 ** umax))
        u = _block_with_max(umax, rng.uniform(umax - 10, umax, 31))[None, None, :]
        assert int(impl.block_exponent(u, mx.SCALE_UOS)[0, 0]) == _uos_exponent_brute(amax), umax
        e_ocp = int(np.floor(np.log2(amax))) - 2
        assert int(impl.block_exponent(u, mx.SCALE_OCP)[0, 0]) == e_ocp, umax
    # an all-masked block: scale byte 0
    assert int(impl.block_exponent(np.full((1, 1, 32), -np.inf), mx.SCALE_UOS)[0, 0]) == -127


def _sweep(impl, r):
    """Codes of residuals r (one per element) with the block exponent pinned at 0."""
    n = len(r)
    nb = -(-n // 31)
    u = np.full((nb, 32), -np.inf)
    u[:, 0] = 2.0                      # block max -> e = 0 under UOS
    flat = np.full(nb * 31, -np.inf)
    flat[:n] = r
    u[:, 1:] = flat.reshape(nb, 31)
    _, codes, e = _quantize(impl, u.reshape(1, -1), mx.SCALE_UOS)
    assert np.all(e == 0)
    return codes.reshape(nb, 32)[:, 1:].reshape(-1)[:n]


def check_near_exp_then_quantize(impl):
    r = np.linspace(-3.0, np.log2(7.25), 20001)
    k_efq = _sweep(impl, r).astype(int)
    k_exp = (mx.e2m1_encode(np.exp2(r)) & 7).astype(int)
    assert np.max(np.abs(k_efq - k_exp)) <= 1
    # away from both rules' thresholds the two agree
    agree = ((r > 0.0) & (r < 0.25)) | ((r > 0.33) & (r < 0.74)) | ((r > 0.81) & (r < 1.24)) | \
            ((r > 1.33) & (r < 1.74)) | ((r > 1.81) & (r < 2.24)) | (r > 2.33)
    assert np.array_equal(k_efq[agree], k_exp[agree])


def check_monotone_saturating(impl):
    r = np.linspace(-8.0, np.log2(7.25), 40001)
    k = _sweep(impl, r).astype(int)
    assert np.all(np.diff(k) >= 0)
    assert k.min() == 0 and k.max() == 7
    assert np.all(k[r >= 2.26] == 7) and np.all(k[r < -0.76] == 0)


def check_ties_half_even(impl):
    r = np.array([-0.75, -0.25, 0.25, 0.75, 1.25, 1.75, 2.25])    # 2r + 2 = 0.5, 1.5, ..., 6.5
    assert list(_sweep(impl, r)) == [0, 2, 2, 4, 4, 6, 6]


def check_attention_normalisation(impl):
    rng = np.random.default_rng(3)
    N, d = 200, 64
    qd, kd = rng.standard_normal((N, d)) * 2, rng.standard_normal((N, d)) * 2
    vd = np.ones((N, d))
    with _patched(impl):
        out = oa.attention_rows(qd, np.arange(N), kd, vd, causal=True, mode=mx.SCALE_UOS, pnq=oa.P_EFQ)
        assert np.max(np.abs(out - 1.0)) <= 1e-12
        # all scores equal: P~ = 1 everywhere -> code 6 with e = -2, out = mean of the values
        v = rng.standard_normal((N, d))
        eq = oa.attention_rows(np.zeros((4, d)), np.arange(4), np.ones((N, d)), v, causal=False,
                               mode=mx.SCALE_UOS, pnq=oa.P_EFQ)
        assert np.allclose(eq, v.mean(axis=0)[None, :], rtol=0, atol=1e-12)


class _patched:
    """Route the attention oracle's exp-free step through `impl` for the duration."""

    def __init__(self, impl):
        self.impl = impl

    def __enter__(self):
        self.saved = (efq.efq_block_exponent, efq.efq_residual_codes)
        efq.efq_block_exponent = self.impl.block_exponent
        efq.efq_residual_codes = self.impl.residual_codes

    def __exit__(self, *a):
        efq.efq_block_exponent, efq.efq_residual_codes = self.saved


CHECKS = [check_grid_points, check_scale_exponent_brute_force, check_near_exp_then_quantize,
          check_monotone_saturating, check_ties_half_even, check_attention_normalisation]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_efq_pin(check):
    check(_impl())


# ---------------------------------------------------------------- planted mistakes

def _codes_with(slope=2.0, offset=2.0, ties="even", clamp_hi=7):
    def residual_codes(u_blocks, e):
        with np.errstate(invalid="ignore"):
            z = slope * (u_blocks - np.asarray(e)[..., None]) + offset
        z = np.where(np.isneginf(z), -1.0, z)
        k = np.rint(z) if ties == "even" else np.floor(z + 0.5)
        k = np.clip(k, 0, clamp_hi)
        return k.astype(np.uint8), z
    return residual_codes


def _exponent_from_block_min(u_blocks, mode):
    finite = np.where(np.isneginf(u_blocks), np.inf, u_blocks)
    umin = np.min(finite, axis=-1)
    amax = np.where(np.isinf(umin), 0.0, np.exp2(umin)).astype(np.float32).astype(np.float64)
    return mx.scale_exponent(amax, mode)


_ORIGINAL_EXPONENT = efq.efq_block_exponent


def _exponent_plus_one(u_blocks, mode):
    return _ORIGINAL_EXPONENT(u_blocks, mode) + 1


MUTANTS = {
    "slope_1.9": dict(residual_codes=_codes_with(slope=1.9)),
    "offset_2.5": dict(residual_codes=_codes_with(offset=2.5)),
    "ties_away": dict(residual_codes=_codes_with(ties="away")),
    "no_clamp_at_7": dict(residual_codes=_codes_with(clamp_hi=15)),
    "scale_from_block_min": dict(block_exponent=_exponent_from_block_min),
    "exponent_plus_one": dict(block_exponent=_exponent_plus_one),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_efq_mutant_is_caught(name):
    impl = types.SimpleNamespace(**{**vars(_impl()), **MUTANTS[name]})
    caught = []
    for check in CHECKS:
        try:
            check(impl)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"mutant {name} passed every pin"

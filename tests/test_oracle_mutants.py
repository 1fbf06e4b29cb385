"""Planted mistakes in copies of the oracle must be caught by the pins.

Each mutant is a plausible slip in the format code (a tie rule, a threshold, a bias,
a nibble order, a dropped sign). The pin checks of test_oracle_pins.py run against the
mutant and at least one of them must fail. Everything here runs on the CPU.
"""
import types

import numpy as np
import pytest

from oracle import mxfp4 as mx
from tests import test_oracle_pins as pins


def _encode_ties_away(y):
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), 6.0)
    d = np.abs(a[..., None] - mx.E2M1_MAGNITUDES)
    k = (7 - np.argmin(d[..., ::-1], axis=-1)).astype(np.uint8)   # last minimum: ties up
    return (np.signbit(y).astype(np.uint8) << 3) | k


def _encode_truncate(y):
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), 6.0)
    k = (np.searchsorted(mx.E2M1_MAGNITUDES, a, side="right") - 1).astype(np.uint8)
    return (np.signbit(y).astype(np.uint8) << 3) | k


def _encode_unsigned_zero(y):
    c = mx.e2m1_encode(y)
    return np.where((c & 7) == 0, 0, c).astype(np.uint8)


def _scale_uos_7(amax, mode):
    e = mx.scale_exponent(amax, mx.SCALE_OCP)
    if mode == mx.SCALE_UOS:
        e = np.where(np.ldexp(np.asarray(amax, float), -e) > 7.0, e + 1, e)
    return e


def _scale_ocp_minus3(amax, mode):
    return mx.scale_exponent(amax, mode) - 1


def _quantize_rows_swapped(x, mode):
    c, s = mx.quantize_rows(x, mode)
    return ((c >> 4) | (c << 4)).astype(np.uint8), s


def _dequant_bias128(codes, scales, C=None):
    return mx.dequantize_rows(codes, (np.asarray(scales).astype(np.int64) - 1).astype(np.uint8), C)


MUTANTS = {
    "ties_away": dict(encode=_encode_ties_away),
    "truncate": dict(encode=_encode_truncate),
    "unsigned_zero": dict(encode=_encode_unsigned_zero),
    "uos_threshold_7": dict(scale_exponent=_scale_uos_7),
    "exponent_off_by_one": dict(scale_exponent=_scale_ocp_minus3),
    "nibbles_swapped": dict(quantize_rows=_quantize_rows_swapped),
    "e8m0_bias_128": dict(dequantize_rows=_dequant_bias128),
}

CHECKS = [pins.check_grid, pins.check_page_values, pins.check_rtne_against_binade_rule,
          pins.check_small_values_underflow, pins.check_saturation_and_sign,
          pins.check_scale_exponents, pins.check_power_of_two_exactness,
          pins.check_block_order_independence, pins.check_partial_block_padding,
          pins.check_nibble_layout]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, golden_dir):
    impl = pins._impl()
    impl = types.SimpleNamespace(**{**vars(impl), **MUTANTS[name]})
    caught = []
    for check in CHECKS:
        try:
            if check is pins.check_page_values:
                check(impl, golden_dir)
            else:
                check(impl)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"mutant {name} passed every pin"

"""Planted mistakes in the NVFP4 and GEMM oracles must be caught by their pins.

Each mutant is a plausible slip (an E4M3 tie rule, an exponent bias, the amax divisor, the block
size, a dropped operand scale, an untransposed operand). It is patched into the oracle module and
the pins of test_oracle_nvfp4_pins.py / test_oracle_gemm_pins.py are run against it: at least one
must fail. Everything here runs on the CPU.
"""
import numpy as np
import pytest

from oracle import gemm as og
from oracle import mxfp4 as mx
from oracle import nvfp4 as nv
from tests import test_oracle_gemm_pins as gpins
from tests import test_oracle_nvfp4_pins as npins

_real_encode = nv.e4m3_encode
_real_decode = nv.e4m3_decode
_real_quantize_blocks = nv.quantize_blocks


def _e4m3_ties_up(v):
    v = np.asarray(v, dtype=np.float64)
    vals = _real_decode(np.arange(0x7F))
    d = np.abs(vals[None, :] - v.reshape(-1, 1))
    last_min = (d.shape[1] - 1 - np.argmin(d[:, ::-1], axis=1))      # ties go up
    return np.minimum(last_min, 0x7E).reshape(v.shape)


def _e4m3_decode_bias8(codes):
    return _real_decode(codes) / 2.0


def _quantize_blocks_amax_over_4(xb):
    return _real_quantize_blocks(np.asarray(xb) * (6.0 / 4.0))


def _quantize_rows_block32(x):
    x = np.asarray(x, dtype=np.float64)
    C = x.shape[-1]
    pad = (-C) % 32
    if pad:
        x = np.concatenate([x, np.zeros(x.shape[:-1] + (pad,))], axis=-1)
    xb = x.reshape(x.shape[:-1] + (x.shape[-1] // 32, 32))
    amax = np.abs(xb).max(axis=-1)
    sbyte = _real_encode((amax / 6.0).astype(np.float32).astype(np.float64))
    s = _real_decode(sbyte)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where((s > 0)[..., None], xb / s[..., None], 0.0)
    codes = mx.e2m1_encode(y).reshape(x.shape)
    return mx.pack_nibbles(codes), np.repeat(sbyte, 2, axis=-1).astype(np.uint8)


def _nvgemm_no_b_scale(ac, as_, bc, bs, K):
    return nv.dequantize_rows(ac, as_, K) @ mx.e2m1_decode(mx.unpack_nibbles(bc))[:, :K].T


def _mxgemm_no_b_scale(ac, as_, bc, bs, K):
    return mx.dequantize_rows(ac, as_, K) @ mx.e2m1_decode(mx.unpack_nibbles(bc))[:, :K].T


def _mxgemm_untransposed(ac, as_, bc, bs, K):
    ad = mx.dequantize_rows(ac, as_, K)
    bd = mx.dequantize_rows(bc, bs, K)
    return (ad.reshape(-1) @ bd.reshape(-1)) * np.ones((ad.shape[0], bd.shape[0]))


NV_PINS = [npins.test_e4m3_format_facts, npins.test_e4m3_round_trip, npins.test_e4m3_nearest_even_by_search,
           npins.test_nvfp4_exactly_representable_blocks, npins.test_nvfp4_error_bound_padding_and_zero_scale,
           npins.test_nvgemm_exact_on_representable_operands]
GEMM_PINS = [gpins.test_brute_force_small, gpins.test_all_ones_gives_k, gpins.test_exactly_representable_operands,
             gpins.test_transpose_symmetry_and_abs_bound]

MUTANTS = {
    "e4m3_ties_up": (nv, "e4m3_encode", _e4m3_ties_up, NV_PINS),
    "e4m3_bias_8": (nv, "e4m3_decode", _e4m3_decode_bias8, NV_PINS),
    "amax_over_4": (nv, "quantize_blocks", _quantize_blocks_amax_over_4, NV_PINS),
    "block_32": (nv, "quantize_rows", _quantize_rows_block32, NV_PINS),
    "nvgemm_no_b_scale": (og, "nvgemm", _nvgemm_no_b_scale, NV_PINS),
    "mxgemm_no_b_scale": (og, "mxgemm", _mxgemm_no_b_scale, GEMM_PINS),
    "mxgemm_untransposed": (og, "mxgemm", _mxgemm_untransposed, GEMM_PINS),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(monkeypatch, name):
    module, attr, fn, pins = MUTANTS[name]
    monkeypatch.setattr(module, attr, fn)
    failed = []
    for pin in pins:
        try:
            pin()
        except Exception:   # an assertion, or a shape error the slip provokes
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"

"""Pins for the CPU oracle of the MXFP4 format and block quantizer.

Each check ties the oracle to something other than itself: values printed on the
"Quantization Error" page, a rounding rule written as a different algorithm, brute-force
searches, and exact invariants. tests/test_oracle_mutants.py plants plausible mistakes
in copies of the oracle and asserts that these same checks catch them.
"""
import os
import types
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import mxfp4 as mx


def _impl():
    return types.SimpleNamespace(encode=mx.e2m1_encode, decode=mx.e2m1_decode,
                                 scale_exponent=mx.scale_exponent,
                                 quantize_rows=mx.quantize_rows,
                                 dequantize_rows=mx.dequantize_rows)


def all_bf16_magnitudes():
    """Every positive finite bf16 value, as float64."""
    bits = np.arange(1, 0x7F80, dtype=np.int32)             # 0x7F80 = +inf
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()


def read_golden(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append([float(t) for t in line.split()])
    return np.array(rows)


# ---------------------------------------------------------------- check functions

def check_grid(impl):
    vals = impl.decode(np.arange(16))
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    assert np.array_equal(vals[:8], mags)
    assert np.array_equal(vals[8:], -mags)
    # grid points encode to themselves (sign bit 3)
    assert np.array_equal(impl.encode(mags), np.arange(8))
    assert np.array_equal(impl.encode(-mags[1:]), np.arange(9, 16))


def check_page_values(impl, golden_dir):
    g = read_golden(os.path.join(golden_dir, "e2m1_page_values.txt"))
    deq = impl.decode(impl.encode(g[:, 0]))
    assert np.array_equal(deq, g[:, 1])
    assert np.allclose(np.abs(deq - g[:, 0]) / np.abs(g[:, 0]), g[:, 2], rtol=0, atol=1e-15)
    sp = read_golden(os.path.join(golden_dir, "e2m1_grid_spacing.txt"))
    grid = impl.decode(np.arange(8))
    for lo, hi, spacing in sp:
        i = int(np.where(grid == lo)[0][0])
        assert grid[i + 1] == hi and hi - lo == spacing
    # linear below 1.0, geometric above it
    assert np.allclose(np.diff(grid[:3]), 0.5)
    assert np.array_equal(grid[2::2], [1, 2, 4])
    assert grid[4] / grid[2] == 2 and grid[6] / grid[4] == 2 and grid[5] / grid[3] == 2


def binade_rne(y):
    """Independent rounding rule: within each binade of the E2M1 grid, round half-to-even
    onto that binade's step with numpy's round (IEEE style), then saturate at 6."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    out = np.where(a < 2.0, np.round(a * 2.0) / 2.0,
                   np.where(a < 4.0, np.round(a), np.round(a / 2.0) * 2.0))
    return np.minimum(out, 6.0)


def check_rtne_against_binade_rule(impl):
    rng = np.random.default_rng(123)
    ys = np.concatenate([
        rng.uniform(0, 8, 200_000),
        np.arange(0, 8.0, 0.125),                                # every tie and grid point
        all_bf16_magnitudes()[all_bf16_magnitudes() < 16],
    ])
    got = np.abs(impl.decode(impl.encode(ys)))
    assert np.array_equal(got, binade_rne(ys))


def check_small_values_underflow(impl):
    # anything at or below a quarter (half the 0.5 subnormal step) rounds to zero;
    # just above it rounds up to 0.5
    assert impl.decode(impl.encode(np.array([0.25, 0.1, 1e-30, 0.0]))).max() == 0.0
    assert impl.decode(impl.encode(np.array([np.nextafter(0.25, 1.0)])))[0] == 0.5


def check_saturation_and_sign(impl):
    assert np.array_equal(impl.decode(impl.encode(np.array([6.0, 7.0, 7.25, 1e6]))), [6, 6, 6, 6])
    assert np.array_equal(impl.decode(impl.encode(np.array([-7.0, -1e6]))), [-6, -6])
    codes = impl.encode(np.array([-0.1, -0.0, 0.1, 0.0]))
    assert list(codes) == [8, 8, 0, 0]


def check_scale_exponents(impl):
    a = all_bf16_magnitudes()
    eo = impl.scale_exponent(a, mx.SCALE_OCP)
    eu = impl.scale_exponent(a, mx.SCALE_UOS)
    ok = (eo > -127) & (eo < 127)
    r = np.ldexp(a, -eo)
    assert np.all((r[ok] >= 4.0) & (r[ok] < 8.0))            # floor(log2 amax) - 2 closed form
    # UOS by brute-force search: the smallest e with amax / 2^e <= 7.25
    e_bf = np.full(a.shape, 10_000, dtype=np.int64)
    for e in range(200, -300, -1):
        e_bf = np.where(np.ldexp(a, -e) <= 7.25, e, e_bf)
    e_bf = np.clip(e_bf, -127, 127)
    assert np.array_equal(eu, e_bf)
    ru = np.ldexp(a, -eu)
    oku = (eu > -127)
    assert np.all((ru[oku] > 3.625) & (ru[oku] <= 7.25))
    # zero block -> byte 0
    assert impl.scale_exponent(np.array([0.0]), mx.SCALE_UOS)[0] == -127
    assert impl.scale_exponent(np.array([0.0]), mx.SCALE_OCP)[0] == -127


def check_power_of_two_exactness(impl):
    rng = np.random.default_rng(7)
    x = torch.from_numpy(rng.standard_normal((64, 96)).astype(np.float32)).bfloat16().double().numpy()
    for mode in (mx.SCALE_OCP, mx.SCALE_UOS):
        c, s = impl.quantize_rows(x, mode)
        deq = impl.dequantize_rows(c, s, 96)
        # exact: every dequantized value equals code value times 2^(byte-127) in rationals
        nib = np.empty((64, 96), dtype=np.uint8)
        nib[:, 0::2] = c[:, :48] & 0xF
        nib[:, 1::2] = c[:, :48] >> 4
        for (i, j) in [(0, 0), (3, 17), (63, 95), (10, 33)]:
            val = Fraction(float(impl.decode(np.array([nib[i, j]]))[0]))
            want = val * Fraction(2) ** (int(s[i, j // 32]) - 127)
            assert Fraction(float(deq[i, j])) == want
        for k in (-5, 3, 20):
            c2, s2 = impl.quantize_rows(np.ldexp(x, k), mode)
            assert np.array_equal(c2, c)
            assert np.array_equal(s2.astype(int), s.astype(int) + k)


def check_block_order_independence(impl):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((8, 256)) * rng.uniform(0.01, 100, (8, 1))
    c, s = impl.quantize_rows(x, mx.SCALE_UOS)
    perm = rng.permutation(8)
    blocks = x.reshape(8, 8, 32)[:, ::-1].reshape(8, 256)      # reverse the block order
    c2, s2 = impl.quantize_rows(blocks[perm], mx.SCALE_UOS)
    assert np.array_equal(c2, c.reshape(8, 8, 16)[:, ::-1].reshape(8, 128)[perm])
    assert np.array_equal(s2, s[:, ::-1][perm])


def check_partial_block_padding(impl):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 40))
    xpad = np.concatenate([x, np.zeros((4, 24))], axis=1)
    c, s = impl.quantize_rows(x, mx.SCALE_UOS)
    c2, s2 = impl.quantize_rows(xpad, mx.SCALE_UOS)
    assert c.shape == (4, 32) and s.shape == (4, 2)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
    assert np.all(c[:, 20:] == 0)                              # padding encodes as +0


def check_nibble_layout(impl):
    # the library's stated packing: element 2i in the low nibble, 2i+1 in the high nibble
    x = np.zeros((1, 32))
    x[0, 0], x[0, 1], x[0, 31] = 4.0, 6.0, -1.0          # amax 6 -> e = 0 in both modes
    for mode in (mx.SCALE_OCP, mx.SCALE_UOS):
        c, s = impl.quantize_rows(x, mode)
        assert s[0, 0] == 127
        assert c[0, 0] == 0x76 and c[0, 15] == 0xA0


# ---------------------------------------------------------------- tests on the oracle

def test_grid():
    check_grid(_impl())


def test_page_values(golden_dir):
    check_page_values(_impl(), golden_dir)


def test_rtne_against_binade_rule():
    check_rtne_against_binade_rule(_impl())


def test_small_values_underflow():
    check_small_values_underflow(_impl())


def test_saturation_and_sign():
    check_saturation_and_sign(_impl())


def test_scale_exponents():
    check_scale_exponents(_impl())


def test_power_of_two_exactness():
    check_power_of_two_exactness(_impl())


def test_block_order_independence():
    check_block_order_independence(_impl())


def test_partial_block_padding():
    check_partial_block_padding(_impl())


def test_nibble_layout():
    check_nibble_layout(_impl())


def test_nibble_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert list(mx.pack_nibbles(codes)[0]) == [0x21, 0x43]
    assert np.array_equal(mx.unpack_nibbles(mx.pack_nibbles(codes)), codes)


def test_rel_frobenius_closed_form():
    x = np.array([3.0, 4.0])
    assert mx.rel_frobenius(np.array([3.0, 4.0 + 0.5]), x) == pytest.approx(0.1, abs=1e-15)


# ---------------------------------------------------------------- UOS optimality by brute force

def _block_sse(blocks, e):
    y = np.ldexp(blocks, -e[:, None])
    deq = np.ldexp(mx.e2m1_decode(mx.e2m1_encode(y)), e[:, None])
    return ((deq - blocks) ** 2).sum(axis=1)


def _distributions(n_blocks, rng):
    return {
        "normal": rng.standard_normal((n_blocks, 32)),
        "laplace": rng.laplace(size=(n_blocks, 32)),
        "uniform": rng.uniform(-1, 1, (n_blocks, 32)),
        "student_t3": rng.standard_t(3, size=(n_blocks, 32)),
    }


def test_uos_beats_ocp_by_exhaustive_exponent_search():
    """The MXAttention abstract claims Qmax = 7.25 is a distribution-independent optimal
    boundary. Brute force over each block's exponent: UOS's total squared error is below
    OCP's on every distribution, within a few percent of the per-block optimum, and the
    best threshold T of the rule 'smallest e with amax/2^e <= T' lies near 7.25."""
    rng = np.random.default_rng(2024)
    thresholds = np.round(np.arange(6.0, 8.0001, 0.1), 2)
    for name, blocks in _distributions(12_000, rng).items():
        amax = np.abs(blocks).max(axis=1)
        e_ocp = mx.scale_exponent(amax, mx.SCALE_OCP)
        e_uos = mx.scale_exponent(amax, mx.SCALE_UOS)
        cands = np.stack([_block_sse(blocks, e_ocp + de) for de in range(-2, 4)])
        best = cands.min(axis=0).sum()
        sse_ocp, sse_uos = _block_sse(blocks, e_ocp).sum(), _block_sse(blocks, e_uos).sum()
        assert sse_uos < sse_ocp, name
        assert sse_uos <= 1.05 * best, name
        sweep = []
        for T in thresholds:
            e_T = np.where(np.ldexp(amax, -e_ocp) > T, e_ocp + 1, e_ocp)
            sweep.append(_block_sse(blocks, e_T).sum())
        t_best = thresholds[int(np.argmin(sweep))]
        assert 6.9 <= t_best <= 7.6, (name, t_best)

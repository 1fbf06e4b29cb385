"""Pins for the NVFP4 oracle (oracle/nvfp4.py) and its GEMM (oracle/gemm.nvgemm).

E4M3 is pinned to the facts of the OCP FP8 format (largest finite 448 = 0x7E, smallest normal
2^-6 = 0x08, smallest subnormal 2^-9 = 0x01, 0x7F NaN) and to an exhaustive nearest-value search
with ties to the even mantissa, written independently of the frexp-based encoder. The block
quantizer is pinned by exactly representable blocks, the elementwise error bound of one E2M1
rounding step, zero padding and the all-zero-scale case. The NVFP4 GEMM by exactly representable
operands (quantize-then-multiply equals the fp64 product of the originals).
"""
import numpy as np
import torch

from oracle import gemm as og
from oracle import mxfp4 as mx
from oracle import nvfp4 as nv


def _finite_codes():
    return np.arange(0x7F)                       # 0x00 .. 0x7E


def test_e4m3_format_facts():
    d = nv.e4m3_decode(np.array([0x7E, 0x08, 0x01, 0x00, 0x38, 0x7F, 0xFF, 0xB8]))
    assert d[0] == 448.0 and d[1] == 2.0 ** -6 and d[2] == 2.0 ** -9 and d[3] == 0.0
    assert d[4] == 1.0 and np.isnan(d[5]) and np.isnan(d[6]) and d[7] == -1.0
    vals = nv.e4m3_decode(_finite_codes())
    assert np.all(np.diff(vals) > 0)              # strictly increasing over the finite codes


def test_e4m3_round_trip():
    c = _finite_codes()
    assert np.array_equal(nv.e4m3_encode(nv.e4m3_decode(c)), c)


def test_e4m3_nearest_even_by_search():
    vals = nv.e4m3_decode(_finite_codes())
    rng = np.random.default_rng(21)
    mids = (vals[1:] + vals[:-1]) / 2                                # every tie
    samples = np.concatenate([rng.uniform(0, 480, 20000), np.exp2(rng.uniform(-12, 9, 20000)), mids,
                              [448.0, 460.0, 500.0, 1e6]])
    got = nv.e4m3_encode(samples)
    for v, g in zip(samples, got):
        if v >= 448.0:
            assert g == 0x7E
            continue
        dist = np.abs(vals - v)
        best = np.flatnonzero(dist == dist.min())
        want = best[0] if best.size == 1 else best[(best & 1) == 0][0]   # tie: even mantissa bit
        assert g == want, (v, g, want)


def test_nvfp4_exactly_representable_blocks():
    rng = np.random.default_rng(22)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    s = nv.e4m3_decode(rng.integers(0x10, 0x70, size=(50, 4)))       # normal scales
    y = rng.choice(grid, size=(50, 4, 16)) * rng.choice([-1.0, 1.0], size=(50, 4, 16))
    y[..., 0] = 6.0                                                  # amax / 6 == s exactly
    x = (y * s[..., None]).reshape(50, 64)
    codes, sb = nv.quantize_rows(x)
    assert np.array_equal(nv.e4m3_decode(sb), s)
    assert np.array_equal(nv.dequantize_rows(codes, sb, 64), x)


def test_nvfp4_error_bound_padding_and_zero_scale():
    rng = np.random.default_rng(23)
    x = torch.from_numpy(rng.standard_normal((64, 100)).astype(np.float32)).bfloat16().double().numpy()
    codes, sb = nv.quantize_rows(x)
    assert codes.shape == (64, 56) and sb.shape == (64, 7)           # 100 -> 7 blocks of 16
    deq = nv.dequantize_rows(codes, sb, 100)
    s = np.repeat(nv.e4m3_decode(sb), 16, axis=1)[:, :100]
    y = np.abs(x) / s
    # one E2M1 rounding step: at most half the local grid spacing, plus saturation above 6
    half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0)) * s
    assert np.all(np.abs(deq - x) <= half_step + np.maximum(np.abs(x) - 6 * s, 0) + 1e-300)
    tiny = np.full((1, 16), 1e-4)                                    # amax / 6 < 2^-10: scale 0
    c0, s0 = nv.quantize_rows(tiny)
    assert s0[0, 0] == 0 and np.all(c0 == 0)


def test_nvgemm_exact_on_representable_operands():
    rng = np.random.default_rng(24)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])

    def make(rows, K):
        s = nv.e4m3_decode(rng.integers(0x20, 0x50, size=(rows, K // 16)))
        y = rng.choice(grid, size=(rows, K // 16, 16)) * rng.choice([-1.0, 1.0], size=(rows, K // 16, 16))
        y[..., 0] = 6.0
        return (y * s[..., None]).reshape(rows, K)
    a, b = make(6, 96), make(5, 96)
    qa, qb = nv.quantize_rows(a), nv.quantize_rows(b)
    assert np.array_equal(og.nvgemm(*qa, *qb, 96), a @ b.T)


def test_nvfp4_finer_than_mxfp4_on_gaussian_blocks():
    # a property of the formats, not a tuning target: 16-element blocks with 3-bit-mantissa scales
    # track the data more closely than 32-element power-of-two scales
    rng = np.random.default_rng(25)
    x = rng.standard_normal((256, 1024))
    e_nv = mx.rel_frobenius(nv.dequantize_rows(*nv.quantize_rows(x), 1024), x)
    e_mx = mx.rel_frobenius(mx.dequantize_rows(*mx.quantize_rows(x, mx.SCALE_OCP), 1024), x)
    assert e_nv < e_mx

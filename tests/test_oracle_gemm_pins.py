"""Pins for the MXFP4 GEMM oracle (oracle/gemm.py), each against something other than itself:

* brute force over blocks with the E2M1 values decoded bit by bit from the format's layout
  (sign bit 3, exponent bits 2..1 with bias 1, mantissa bit 0), not by the oracle's table, and
  plain Python loops instead of a matrix product;
* exact closed forms (all-ones operands give C = K);
* operands that MXFP4 represents exactly: quantizing them and multiplying must reproduce the
  fp64 product of the originals exactly (a transposed operand, a swapped nibble or a wrong scale
  index would not);
* transpose symmetry C(A, B) = C(B, A)^T.
"""
import numpy as np

from oracle import gemm as og
from oracle import mxfp4 as mx


def _e2m1_bits(code: int) -> float:
    sign = -1.0 if code & 0x8 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    mag = man * 0.5 if exp == 0 else (1.0 + 0.5 * man) * 2.0 ** (exp - 1)
    return sign * mag


def _brute(a_codes, a_scales, b_codes, b_scales, K):
    M, N = a_codes.shape[0], b_codes.shape[0]
    out = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            total = 0.0
            for blk in range(K // 32):
                ea = int(a_scales[m, blk]) - 127
                eb = int(b_scales[n, blk]) - 127
                part = 0.0
                for i in range(32):
                    k = blk * 32 + i
                    ca = (int(a_codes[m, k // 2]) >> (4 * (k % 2))) & 0xF
                    cb = (int(b_codes[n, k // 2]) >> (4 * (k % 2))) & 0xF
                    part += _e2m1_bits(ca) * _e2m1_bits(cb)
                total += part * 2.0 ** (ea + eb)
            out[m, n] = total
    return out


def test_brute_force_small():
    rng = np.random.default_rng(11)
    for (M, N, K) in [(3, 5, 64), (2, 2, 32), (4, 3, 96)]:
        a = rng.standard_normal((M, K)) * rng.choice([1e-3, 1.0, 40.0], size=(M, 1))
        b = rng.standard_normal((N, K)) * 3.0
        ac, as_ = mx.quantize_rows(a, mx.SCALE_UOS)
        bc, bs = mx.quantize_rows(b, mx.SCALE_OCP)
        ref = _brute(ac, as_, bc, bs, K)
        got = og.mxgemm(ac, as_, bc, bs, K)
        np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-300)


def test_all_ones_gives_k():
    for K in (32, 256, 4096):
        codes = np.full((4, K // 2), 0x22, dtype=np.uint8)     # code 0x2 = 1.0 in both nibbles
        scales = np.full((4, K // 32), 127, dtype=np.uint8)    # 2^0
        c = og.mxgemm(codes, scales, codes, scales, K)
        assert np.all(c == K)


def test_exactly_representable_operands():
    rng = np.random.default_rng(12)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    M, N, K = 7, 5, 160
    # per-block values g * 2^e with the block's largest magnitude 6 or 4 so UOS / OCP keep e
    def make(rows):
        x = rng.choice(grid, size=(rows, K)) * rng.choice([-1.0, 1.0], size=(rows, K))
        e = rng.integers(-6, 7, size=(rows, K // 32))
        x = x.reshape(rows, K // 32, 32)
        x[:, :, 0] = 6.0                                     # fixes the block exponent to e
        return (x * np.exp2(e)[..., None]).reshape(rows, K)
    a, b = make(M), make(N)
    for mode in (mx.SCALE_OCP, mx.SCALE_UOS):
        ac, as_ = mx.quantize_rows(a, mode)
        bc, bs = mx.quantize_rows(b, mode)
        assert np.array_equal(mx.dequantize_rows(ac, as_, K), a)
        assert np.array_equal(og.mxgemm(ac, as_, bc, bs, K), a @ b.T)


def test_transpose_symmetry_and_abs_bound():
    rng = np.random.default_rng(13)
    a = rng.standard_normal((6, 128))
    b = rng.laplace(size=(9, 128))
    ac, as_ = mx.quantize_rows(a, mx.SCALE_UOS)
    bc, bs = mx.quantize_rows(b, mx.SCALE_UOS)
    c = og.mxgemm(ac, as_, bc, bs, 128)
    assert np.array_equal(c, og.mxgemm(bc, bs, ac, as_, 128).T)
    assert np.all(np.abs(c) <= og.mxgemm_abs(ac, as_, bc, bs, 128) * (1 + 1e-15))

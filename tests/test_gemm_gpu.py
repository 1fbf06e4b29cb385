"""GPU parity of the block-scaled MXFP4 GEMM (mxattn_gemm) against the oracle.

Operands are quantized by the oracle (so only the product is under test), on shapes that span
several 128 x 256 tiles and 256-element K stages and leave ragged edges in M, N and K. The bar:
fp32 output within (K/32 + 8) * 2^-24 * sum_k |a_k b_k| of the exact product (at most one fp32
rounding per 32-element block accumulation, plus slack), bf16 output additionally within half a
bf16 ulp of the result. At the benchmark's size the check samples rows and columns, which the
oracle quantizes itself from the seeded generator.
"""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import api, build, synthetic
from oracle import gemm as og
from oracle import mxfp4 as mx

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return torch.device("cuda:0")


def _u8(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(dev)


def _bound(absum, K):
    return (K / 32 + 8) * 2.0 ** -24 * absum


SHAPES = [(128, 256, 256), (1, 8, 32), (100, 200, 96), (300, 520, 992), (257, 264, 4096), (129, 1024, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_vs_oracle(dev, M, N, K, out_dtype):
    rng = np.random.default_rng(M * 31 + N * 7 + K)
    a = rng.standard_normal((M, K)) * np.exp2(rng.integers(-8, 8, size=(M, 1)))
    b = rng.laplace(size=(N, K)) * 0.1
    ac, as_ = mx.quantize_rows(a, mx.SCALE_UOS)
    bc, bs = mx.quantize_rows(b, mx.SCALE_OCP)
    ws = api.gemm_workspace(M, N, K, dev)
    c = api.mxattn_gemm(_u8(ac, dev), _u8(as_, dev), _u8(bc, dev), _u8(bs, dev), K, out_dtype=out_dtype,
                        workspace=ws)
    assert api.mxattn_check_status(ws) == 0
    c = c.float().cpu().numpy().astype(np.float64)
    ref = og.mxgemm(ac, as_, bc, bs, K)
    tol = _bound(og.mxgemm_abs(ac, as_, bc, bs, K), K)
    if out_dtype == torch.bfloat16:
        tol = tol + np.abs(ref) * 2.0 ** -8
    err = np.abs(c - ref)
    assert np.all(err <= tol), (float(err.max()), float((err / np.maximum(tol, 1e-300)).max()))


def test_gemm_benchmark_size_sampled(dev):
    M, N, K = synthetic.GEMM_SHAPE
    a, b = synthetic.gemm_inputs(M, N, K)
    da, db = a.to(dev), b.to(dev)
    ac, as_ = api.mxattn_quantize(da, False, api.SCALE_UOS)
    bc, bs = api.mxattn_quantize(db, False, api.SCALE_UOS)
    ws = api.gemm_workspace(M, N, K, dev)
    c = api.mxattn_gemm(ac, as_, bc, bs, K, out_dtype=torch.bfloat16, workspace=ws)
    assert api.mxattn_check_status(ws) == 0
    rng = np.random.default_rng(7)
    rows = np.concatenate([[0, M - 1], rng.integers(0, M, 6)])
    cols = np.concatenate([[0, N - 1], rng.integers(0, N, 62)])
    # the oracle starts from the same bf16 values the GPU quantized
    a_bf = torch.from_numpy(synthetic.gemm_rows_f32("A", rows, K)).bfloat16().double().numpy()
    b_bf = torch.from_numpy(synthetic.gemm_rows_f32("B", cols, K)).bfloat16().double().numpy()
    qa = mx.quantize_rows(a_bf, mx.SCALE_UOS)
    qb = mx.quantize_rows(b_bf, mx.SCALE_UOS)
    ref = og.mxgemm(*qa, *qb, K)
    tol = _bound(og.mxgemm_abs(*qa, *qb, K), K) + np.abs(ref) * 2.0 ** -8
    got = c[torch.from_numpy(rows).to(dev)][:, torch.from_numpy(cols).to(dev)].float().cpu().numpy()
    err = np.abs(got - ref)
    assert np.all(err <= tol), float((err / tol).max())

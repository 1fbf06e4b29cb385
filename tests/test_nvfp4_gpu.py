"""GPU parity of the NVFP4 comparison path: the quantizer bit for bit against the oracle, the
NVFP4 GEMM (tcgen05 kind::mxf4nvf4, E4M3 scales per 16 elements) against the oracle's product,
and the two formats side by side on the same data."""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import api, build
from oracle import gemm as og
from oracle import mxfp4 as mx
from oracle import nvfp4 as nv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return torch.device("cuda:0")


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).bfloat16()


def _u8(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(dev)


@pytest.mark.parametrize("rows,cols", [(1, 16), (37, 100), (256, 1024), (3, 8), (1000, 72)])
def test_quantizer_bit_exact(dev, rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    x = rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-14, 12, size=(rows, 1)))
    x[rng.random((rows, cols)) < 0.01] *= 40.0
    x[0, :min(cols, 16)] = 1e-5                         # a block whose scale underflows to 0
    if rows > 1:
        x[1, :min(cols, 16)] = 3.0e4                    # a block that saturates the scale at 448
    xb = _bf16(x)
    codes, scales = api.mxattn_quantize_nvfp4(xb.to(dev))
    oc, os_ = nv.quantize_rows(xb.double().numpy())
    assert np.array_equal(scales.cpu().numpy(), os_)
    assert np.array_equal(codes.cpu().numpy(), oc)


def _bound(absum, K):
    return (K / 16 + 8) * 2.0 ** -24 * absum


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 8, 32), (100, 200, 96), (300, 520, 992), (257, 264, 4096)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_nvfp4_gemm_vs_oracle(dev, M, N, K, out_dtype):
    rng = np.random.default_rng(M + 3 * N + 5 * K)
    a = rng.standard_normal((M, K)) * np.exp2(rng.integers(-4, 4, size=(M, 1)))
    b = rng.laplace(size=(N, K)) * 0.1
    qa, qb = nv.quantize_rows(a), nv.quantize_rows(b)
    c = api.mxattn_gemm_nvfp4(*(_u8(t, dev) for t in (*qa, *qb)), K, out_dtype=out_dtype)
    c = c.float().cpu().numpy().astype(np.float64)
    ref = og.nvgemm(*qa, *qb, K)
    tol = _bound(og.nvgemm_abs(*qa, *qb, K), K)
    if out_dtype == torch.bfloat16:
        tol = tol + np.abs(ref) * 2.0 ** -8
    err = np.abs(c - ref)
    assert np.all(err <= tol), (float(err.max()), float((err / np.maximum(tol, 1e-300)).max()))


def test_formats_side_by_side(dev):
    """Same bf16 operands through the MXFP4 (UOS) and NVFP4 GEMMs on the GPU; each result must
    match its own oracle, and NVFP4's finer scales must land closer to the exact product."""
    M, N, K = 512, 512, 2048
    rng = np.random.default_rng(31)
    a = _bf16(rng.standard_normal((M, K)))
    b = _bf16(rng.standard_normal((N, K)) * 0.05)
    exact = a.double().numpy() @ b.double().numpy().T
    da, db = a.to(dev), b.to(dev)
    c_mx = api.mxattn_gemm(*api.mxattn_quantize(da, False, api.SCALE_UOS),
                           *api.mxattn_quantize(db, False, api.SCALE_UOS), K).double().cpu().numpy()
    c_nv = api.mxattn_gemm_nvfp4(*api.mxattn_quantize_nvfp4(da), *api.mxattn_quantize_nvfp4(db), K)
    c_nv = c_nv.double().cpu().numpy()
    e_mx = mx.rel_frobenius(c_mx, exact)
    e_nv = mx.rel_frobenius(c_nv, exact)
    assert e_nv < e_mx, (e_nv, e_mx)

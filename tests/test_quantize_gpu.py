"""GPU parity of the MXFP4 quantizer kernels against the oracle: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import api, build, synthetic
from oracle import mxfp4 as mx
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return torch.device("cuda:0")


def _rand_bf16(shape, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape) * np.exp(rng.uniform(-6, 6, shape[:-1] + (1,)))
    x[rng.random(shape) < 0.01] *= 40
    x[rng.random(shape) < 0.01] = 0.0
    return torch.from_numpy(x.astype(np.float32)).bfloat16()


def _check_rows(xc, dev, mode):
    codes, scales = api.mxattn_quantize(xc.to(dev), transpose=False, scale_mode=mode)
    oc, os_ = mx.quantize_rows(xc.double().numpy(), mode)
    assert np.array_equal(scales.cpu().numpy(), os_)
    assert np.array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("mode", [mx.SCALE_OCP, mx.SCALE_UOS])
@pytest.mark.parametrize("shape", [(1, 32), (5, 40), (2, 7, 1000), (64, 1024), (33, 31), (4, 129, 128),
                                   (3, 1, 1), (2, 3, 64)])
def test_rows_bitexact(dev, mode, shape):
    _check_rows(_rand_bf16(shape, seed=sum(shape)), dev, mode)


@pytest.mark.parametrize("mode", [mx.SCALE_OCP, mx.SCALE_UOS])
@pytest.mark.parametrize("shape", [(2, 100, 64), (1, 257, 128), (3, 31, 10), (1, 1000, 72), (1, 300, 128),
                                   (1, 1, 8)])
def test_cols_bitexact(dev, mode, shape):
    x = _rand_bf16(shape, seed=7 + sum(shape))
    codes, scales = api.mxattn_quantize(x.to(dev), transpose=True, scale_mode=mode)
    oc, os_ = mx.quantize_transposed(x.double().numpy(), mode)
    assert np.array_equal(scales.cpu().numpy(), os_)
    assert np.array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("mode", [mx.SCALE_OCP, mx.SCALE_UOS])
def test_special_values(dev, mode):
    rows = []
    # every rounding tie of the E2M1 grid with block exponent 0 (amax 4 -> e = 0 in both rules)
    ties = [4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, 0.1, -0.1, -0.0]
    rows.append(ties + [0.0] * 16)
    rows.append([5.0, 6.0, 7.0, 7.25, 7.5, -5.0] + [1.0] * 26)                  # saturation region
    rows.append([0.0] * 32)                                                     # all zero -> byte 0
    rows.append([1e-40, -2e-40, 3e-39] + [0.0] * 29)                            # bf16 subnormals
    rows.append([3.0e38, -1.0e38] + [1.0] * 30)                                 # near bf16 max
    rows.append([7.25 * 2 ** 3, 7.26 * 2 ** 3] + [0.5] * 30)                    # UOS boundary region
    x = torch.tensor(rows, dtype=torch.float32).bfloat16()
    _check_rows(x, dev, mode)


@pytest.mark.parametrize("mode", [mx.SCALE_OCP, mx.SCALE_UOS])
def test_quantizer_workload_sampled(dev, mode):
    x = synthetic.quant_input()
    codes, scales = api.mxattn_quantize(x.to(dev), transpose=False, scale_mode=mode)
    rng = np.random.default_rng(mode)
    rows = np.unique(np.concatenate([[0, x.shape[0] - 1], rng.choice(x.shape[0], 2046, replace=False)]))
    oc, os_ = mx.quantize_rows(x[rows].double().numpy(), mode)
    assert np.array_equal(scales[rows].cpu().numpy(), os_)
    assert np.array_equal(codes[rows].cpu().numpy(), oc)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", [mx.SCALE_OCP, mx.SCALE_UOS])
def test_forward_prepare_layouts(dev, d, mode):
    B, Hq, Hkv, N = 2, 4, 2, 300
    q = _rand_bf16((B, Hq, N, d), 1)
    k = _rand_bf16((B, Hkv, N, d), 2)
    v = _rand_bf16((B, Hkv, N, d), 3)
    ws = api.alloc_workspace(B, Hq, Hkv, N, d, dev)
    api.mxattn_forward_prepare(q.to(dev), k.to(dev), v.to(dev), mode, ws)
    torch.cuda.synchronize()
    w = ws.cpu().numpy()
    L = parity.ws_offsets(B, Hq, Hkv, N, d)
    npad = L["npad"]
    region = lambda n: w[L[n][0]:L[n][0] + L[n][1]]  # noqa: E731

    def pad_rows(a):
        out = np.zeros(a.shape[:-2] + (npad, a.shape[-1]), dtype=np.float64)
        out[..., :N, :] = a
        return out

    for name, t, H in (("q", q, Hq), ("k", k, Hkv)):
        oc, os_ = mx.quantize_rows(pad_rows(t.double().numpy()), mode)
        assert np.array_equal(region(name + "c").reshape(B * H, npad, d // 2), oc.reshape(B * H, npad, d // 2))
        # MXFP4 packs one atom per 128 rows at the front of a region sized for NVFP4
        sf = parity.atom_to_rowmajor(region(name + "s")[:B * H * (npad // 128) * 512], B * H, npad, d // 32)
        assert np.array_equal(sf, os_.reshape(B * H, npad, d // 32))
    oc, os_ = mx.quantize_transposed(pad_rows(v.double().numpy()), mode)      # [B,Hkv,d,npad/2]
    assert np.array_equal(region("vc").reshape(B * Hkv, d, npad // 2), oc.reshape(B * Hkv, d, npad // 2))
    # V scale atoms: MN index = channel, K index = key block inside each 128-key tile
    a = region("vs")[:B * Hkv * (npad // 128) * 512].reshape(B * Hkv, npad // 128, 512)
    ch = np.arange(d)
    for kb in range(npad // 32):
        got = a[:, kb // 4, (ch % 32) * 16 + (ch // 32) * 4 + kb % 4]
        assert np.array_equal(got, os_.reshape(B * Hkv, d, npad // 32)[:, :, kb])

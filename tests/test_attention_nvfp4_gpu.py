"""GPU parity of the attention kernel's NVFP4 comparison mode (MXATTN_SCALE_NVFP4: blocks of 16
with E4M3 scales for Q, K, V and P~) against the oracle's NVFP4 mode: the quantized operands in
the workspace bit for bit, P~ codes with the tie-aware classification, and the outputs."""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import api, build, synthetic
from oracle import attention as oa
from oracle import nvfp4 as nv
from tests import parity
from tests.test_attention_gpu import _rand_qkv, _run_and_check, _sample_rows

pytestmark = pytest.mark.gpu
NV = nv.SCALE_NVFP4


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return torch.device("cuda:0")


def _rows_atoms(atoms, heads, rows_pad, nblk):
    """[heads][rows_pad/128][ceil(nblk/4)][512] -> [heads][rows_pad][nblk]."""
    ksteps = -(-nblk // 4)
    a = np.asarray(atoms).reshape(heads, rows_pad // 128, ksteps, 512)
    n = np.arange(rows_pad)
    out = np.empty((heads, rows_pad, nblk), dtype=np.uint8)
    for b in range(nblk):
        off = (n % 32) * 16 + ((n % 128) // 32) * 4 + b % 4
        out[:, :, b] = a[:, n // 128, b // 4, off]
    return out


def _cols_atoms(atoms, heads, d, npad):
    """[heads][npad/64][512] (MN index = channel) -> [heads][d][npad/16]."""
    a = np.asarray(atoms).reshape(heads, npad // 64, 512)
    c = np.arange(d)
    out = np.empty((heads, d, npad // 16), dtype=np.uint8)
    for b in range(npad // 16):
        out[:, :, b] = a[:, b // 4, (c % 32) * 16 + (c // 32) * 4 + b % 4]
    return out


@pytest.mark.parametrize("d", [64, 128])
def test_prepare_layouts_bit_exact(dev, d):
    B, Hq, Hkv, N = 1, 2, 1, 300
    q, k, v = _rand_qkv(B, Hq, Hkv, N, d, seed=40 + d, qk_scale=2.0)
    ws = api.alloc_workspace(B, Hq, Hkv, N, d, dev)
    api.mxattn_forward_prepare(q.to(dev), k.to(dev), v.to(dev), NV, ws)
    w = ws.cpu().numpy()
    o = parity.ws_offsets(B, Hq, Hkv, N, d)
    npad = o["npad"]

    def region(name, shape):
        off, _ = o[name]
        return w[off:off + int(np.prod(shape))].reshape(shape)
    for name, x, heads in (("q", q, B * Hq), ("k", k, B * Hkv)):
        oc, os_ = nv.quantize_rows(x.double().numpy().reshape(heads, N, d))
        codes = region(name + "c", (heads, npad, d // 2))
        assert np.array_equal(codes[:, :N], oc) and not codes[:, N:].any(), name
        scales = _rows_atoms(region(name + "s", (heads, npad // 128, max(1, d // 64), 512)), heads, npad, d // 16)
        assert np.array_equal(scales[:, :N], os_) and not scales[:, N:].any(), name
    vt = np.swapaxes(v.double().numpy().reshape(B * Hkv, N, d), -1, -2)
    vt = np.concatenate([vt, np.zeros(vt.shape[:-1] + (npad - N,))], axis=-1)
    oc, os_ = nv.quantize_rows(vt)
    assert np.array_equal(region("vc", (B * Hkv, d, npad // 2)), oc)
    assert np.array_equal(_cols_atoms(region("vs", (B * Hkv, npad // 64, 512)), B * Hkv, d, npad), os_)


@pytest.mark.parametrize("pnq", [True, False])
def test_tiny_workload(dev, pnq):
    cfg = synthetic.ATTN_CONFIGS["tiny"]
    q, k, v = synthetic.attn_inputs(cfg)
    _run_and_check(dev, q, k, v, cfg.causal, NV, pnq, [(0, 0), (0, 1)])


@pytest.mark.parametrize("N", [1, 100, 129, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes(dev, N, d, causal):
    q, k, v = _rand_qkv(1, 4, 2, N, d, seed=500 + N + d + causal, qk_scale=1.5)
    _run_and_check(dev, q, k, v, causal, NV, True, [(0, 0), (0, 3)])


def test_gqa_and_batches(dev):
    q, k, v = _rand_qkv(2, 8, 2, 200, 128, seed=41)
    _run_and_check(dev, q, k, v, True, NV, True, [(0, 0), (0, 5), (1, 3), (1, 7)])


def test_llm_gqa_full_size_sampled(dev):
    cfg = synthetic.ATTN_CONFIGS["llm_gqa"]
    q, k, v = synthetic.attn_inputs(cfg)
    B, Hq, Hkv, N = cfg.B, cfg.Hq, cfg.Hkv, cfg.N
    ws = api.alloc_workspace(B, Hq, Hkv, N, cfg.d, dev)
    out = api.mxattn_forward(q.to(dev), k.to(dev), v.to(dev), causal=cfg.causal, scale_mode=NV, pnq=True,
                             workspace=ws)
    assert api.mxattn_check_status(ws) == 0
    rng = np.random.default_rng(98)
    for (b, h) in [(0, 0), (B - 1, Hq - 1)]:
        rows = _sample_rows(cfg, rng)
        g = h // (Hq // Hkv)
        (qd, kd, vd), _ = oa.dequantized_qkv(q[b, h].double().numpy(), k[b, g].double().numpy(),
                                             v[b, g].double().numpy(), NV)
        ref = oa.attention_rows(qd[rows], rows, kd, vd, causal=cfg.causal, mode=NV, pnq=True)
        mabs, rfro = parity.out_errors(out[b, h, rows].cpu().numpy(), ref)
        assert mabs <= parity.OUT_MAX_ABS and rfro <= parity.OUT_REL_FRO, (b, h, mabs, rfro)

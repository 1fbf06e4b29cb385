"""GPU parity of mxattn_forward_quantized, the attention kernel on operands already in MXFP4.

* Operands quantized by the oracle (from fp64 values, so the check does not pass through the GPU
  quantizer at all) against the oracle's tiled attention on the same dequantized operands.
* Operands from mxattn_quantize against mxattn_forward: the same codes must give the same output
  bit for bit, which checks the canonical-layout plumbing (per-head row stride N instead of the
  padded one, scale repacking, zero-filled tails) at full size as well.
"""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import api, build, synthetic
from oracle import attention as oa
from oracle import mxfp4 as mx
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return torch.device("cuda:0")


def _u8(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(dev)


SHAPES = [(1, 2, 2, 256, 64, False), (1, 2, 1, 100, 128, True), (2, 4, 2, 129, 64, True),
          (1, 1, 1, 1, 128, False), (1, 2, 2, 300, 128, False), (1, 2, 2, 200, 64, True)]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", SHAPES)
@pytest.mark.parametrize("mode,pnq", [(mx.SCALE_UOS, True), (mx.SCALE_OCP, False), (mx.SCALE_UOS, False)])
def test_oracle_quantized_operands(dev, B, Hq, Hkv, N, d, causal, mode, pnq):
    rng = np.random.default_rng(1000 * N + d + 7 * causal)
    q = rng.standard_normal((B, Hq, N, d)) * 1.5
    k = rng.standard_normal((B, Hkv, N, d)) * 1.5
    v = rng.standard_normal((B, Hkv, N, d))
    qc, qs = mx.quantize_rows(q, mode)
    kc, ks = mx.quantize_rows(k, mode)
    vc, vs = mx.quantize_transposed(v, mode)
    out = api.mxattn_forward_quantized(*(_u8(a, dev) for a in (qc, qs, kc, ks, vc, vs)), N=N, d=d,
                                       causal=causal, p_scale_mode=mode, pnq=pnq).cpu().numpy()
    assert np.isfinite(out).all()
    group = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            g = h // group
            qd = mx.dequantize_rows(qc[b, h], qs[b, h], d)
            kd = mx.dequantize_rows(kc[b, g], ks[b, g], d)
            vd = np.swapaxes(mx.dequantize_rows(vc[b, g], vs[b, g], N), -1, -2)
            ref = oa.attention_rows(qd, np.arange(N), kd, vd, causal=causal, mode=mode, pnq=pnq)
            mabs, rfro = parity.out_errors(out[b, h], ref)
            assert mabs <= parity.OUT_MAX_ABS and rfro <= parity.OUT_REL_FRO, (b, h, mabs, rfro)


@pytest.mark.parametrize("name", ["tiny", "llm_gqa", "video_dit"])
def test_same_codes_same_output(dev, name):
    cfg = synthetic.ATTN_CONFIGS[name]
    q, k, v = (t.to(dev) for t in synthetic.attn_inputs(cfg))
    mode, pnq = mx.SCALE_UOS, True
    qc, qs = api.mxattn_quantize(q, False, mode)
    kc, ks = api.mxattn_quantize(k, False, mode)
    vc, vs = api.mxattn_quantize(v, True, mode)
    ws = api.alloc_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.d, dev)
    ref = api.mxattn_forward(q, k, v, causal=cfg.causal, scale_mode=mode, pnq=pnq, workspace=ws)
    assert api.mxattn_check_status(ws) == 0
    out = api.mxattn_forward_quantized(qc, qs, kc, ks, vc, vs, N=cfg.N, d=cfg.d, causal=cfg.causal,
                                       p_scale_mode=mode, pnq=pnq, workspace=ws)
    assert api.mxattn_check_status(ws) == 0
    assert torch.equal(out, ref)

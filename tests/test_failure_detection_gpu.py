"""The bounded-wait failure detection on the GPU, without a fault: a kernel waits on an mbarrier
phase that nothing completes (mxattn_selftest_wait_timeout). The wait must give up after its
bound, report its code through the status word that mxattn_check_status reads, raise the abort
flag that releases the CTA's other waiters, and leave a context that still computes correctly."""
import time

import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import _lib, api, build, synthetic
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


def test_wait_timeout_is_reported_and_context_survives(dev):
    ws = torch.zeros(1024, dtype=torch.uint8, device=dev)
    lib = _lib.load()
    t0 = time.time()
    assert lib.mxattn_selftest_wait_timeout(ws.data_ptr(), api._stream(dev)) == 0
    detail = api.mxattn_check_status(ws)              # synchronises
    elapsed = time.time() - t0
    assert detail == 0x701, hex(detail)
    assert 1.5 < elapsed < 30.0, elapsed               # the 2 s device-time bound, not a hang
    seen = int(ws[4:8].view(torch.int32).item())
    assert seen == 3, seen                             # both warps left their wait
    assert api.mxattn_check_status(ws) == 0            # the status word was cleared
    # the context still runs the real pipeline correctly
    cfg = synthetic.ATTN_CONFIGS["tiny"]
    q, k, v = synthetic.attn_inputs(cfg)
    out = api.mxattn_forward(q.to(dev), k.to(dev), v.to(dev), causal=cfg.causal).cpu().numpy()
    (qd, kd, vd), _ = oa.dequantized_qkv(q[0, 0].double().numpy(), k[0, 0].double().numpy(),
                                         v[0, 0].double().numpy(), mx.SCALE_UOS)
    ref = oa.attention_rows(qd, np.arange(cfg.N), kd, vd, causal=cfg.causal, mode=mx.SCALE_UOS, pnq=True)
    mabs, rfro = parity.out_errors(out[0, 0], ref)
    assert mabs <= parity.OUT_MAX_ABS and rfro <= parity.OUT_REL_FRO

"""mxattn_forward_noalloc: the attention forward for callers that cannot allocate device memory
(a host or framework that owns all device memory, or a loop where an allocation call is not
allowed). It takes the workspace from a static device array inside the library instead of a
caller buffer. This file is collected last on purpose.

Checks, through the C ABI: two calls in a row each reproduce mxattn_forward (the entry point with
a caller-provided workspace) bit for bit -- both run the same kernels on the same inputs, so any
difference would be a bug such as stale bytes left in the shared array by the previous call -- and
a rejected call gets the same status code from both entry points.
"""
import ctypes

import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import _lib, api, build, synthetic
from oracle import mxfp4 as mx

pytestmark = pytest.mark.gpu

MAX_WORKSPACE = 16 << 20       # MXATTN_NOALLOC_MAX_WORKSPACE in include/mxattn.h
INVALID_ARG, UNSUPPORTED, WORKSPACE_ERR = 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return _lib.load()


def _noalloc(lib, q, k, v, out, causal, mode, pnq):
    B, Hq, N, d = q.shape
    stream = torch.cuda.current_stream(q.device).cuda_stream
    return lib.mxattn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq,
                                      k.shape[1], N, d, int(causal), mode, int(pnq), 0, stream)


@pytest.mark.parametrize("mode,pnq,causal", [(mx.SCALE_UOS, True, False), (mx.SCALE_OCP, False, True)])
def test_noalloc_matches_forward_twice(lib, mode, pnq, causal):
    dev = torch.device("cuda:0")
    cfg = synthetic.ATTN_CONFIGS["tiny"]
    q, k, v = (t.to(dev) for t in synthetic.attn_inputs(cfg))
    assert lib.mxattn_forward_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.d) <= MAX_WORKSPACE
    ref = api.mxattn_forward(q, k, v, causal=causal, scale_mode=mode, pnq=pnq)
    for _ in range(2):
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev)
        assert _noalloc(lib, q, k, v, out, causal, mode, pnq) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def test_noalloc_other_shape_after_first(lib):
    # a second shape through the same static array (d = 128, GQA, ragged N), twice
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 4, 300, 128, generator=g).bfloat16().to(dev)
    k = torch.randn(1, 2, 300, 128, generator=g).bfloat16().to(dev)
    v = torch.randn(1, 2, 300, 128, generator=g).bfloat16().to(dev)
    ref = api.mxattn_forward(q, k, v, causal=True)
    for _ in range(2):
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev)
        assert _noalloc(lib, q, k, v, out, True, mx.SCALE_UOS, True) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


@pytest.mark.parametrize("shape,expected", [
    ((1, 40, 40, 32760, 128), WORKSPACE_ERR),      # video-DiT: ~267 MB of workspace
    ((1, 4, 2, 256, 96), UNSUPPORTED),             # head dimension
    ((1, 4, 3, 256, 64), INVALID_ARG),             # Hq not a multiple of Hkv
    ((1, 1 << 24, 1, 128 * 128, 64), UNSUPPORTED),  # B * Hq * query tiles >= 2^31
])
def test_noalloc_rejects_like_forward(lib, shape, expected):
    # rejected on the host before anything runs: the pointers are never read
    B, Hq, Hkv, N, d = shape
    fake = ctypes.c_void_p(0x100000)
    r = lib.mxattn_forward_noalloc(fake, fake, fake, fake, B, Hq, Hkv, N, d, 0, 1, 1, 0, None)
    assert r == expected
    ws_bytes = min(lib.mxattn_forward_workspace_size(B, Hq, Hkv, N, d), MAX_WORKSPACE) or MAX_WORKSPACE
    r_fwd = lib.mxattn_forward(fake, fake, fake, fake, B, Hq, Hkv, N, d, 0, 1, 1, 0, fake, ws_bytes, None)
    assert r_fwd == expected


def test_noalloc_status_word_reads_clean(lib):
    """After good noalloc calls the static array's status word reads 0, and reading clears it."""
    dev = torch.device("cuda:0")
    cfg = synthetic.ATTN_CONFIGS["tiny"]
    q, k, v = (t.to(dev) for t in synthetic.attn_inputs(cfg))
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    assert _noalloc(lib, q, k, v, out, False, mx.SCALE_UOS, True) == 0
    stream = torch.cuda.current_stream(dev).cuda_stream
    for _ in range(2):
        detail = ctypes.c_uint(123)
        assert lib.mxattn_check_status_noalloc(stream, ctypes.byref(detail)) == 0
        assert detail.value == 0

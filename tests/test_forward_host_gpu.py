"""GPU test of mxattn_forward_host: the host-buffer entry point pipelines copies and kernels over
groups of KV heads; heads are independent, so its output must equal mxattn_forward's bit for bit
(several groups, a partial last group, GQA, causal, both output types, both formats)."""
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import api, build, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return torch.device("cuda:0")


@pytest.mark.parametrize("name,mode,out_dtype", [("video_dit", api.SCALE_UOS, torch.float32),
                                                 ("llm_gqa", api.SCALE_UOS, torch.bfloat16),
                                                 ("tiny", api.SCALE_OCP, torch.float32),
                                                 ("llm_gqa", api.SCALE_NVFP4, torch.float32)])
def test_host_pipeline_matches_forward(dev, name, mode, out_dtype):
    cfg = synthetic.ATTN_CONFIGS[name]
    q, k, v = synthetic.attn_inputs(cfg)
    if name == "video_dit":       # 13 heads: several groups and a partial last one, still quick
        q, k, v = q[:, :13].contiguous(), k[:, :13].contiguous(), v[:, :13].contiguous()
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    out_h = torch.empty(q.shape, dtype=out_dtype).pin_memory()
    n = api._lib.load().mxattn_forward_host_workspace_size(
        *q.shape[:2], k.shape[1], *q.shape[2:], 0 if out_dtype == torch.float32 else 1)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    api.mxattn_forward_host(qh, kh, vh, out_h, causal=cfg.causal, scale_mode=mode, workspace=ws, device=dev)
    assert api.mxattn_check_status(ws) == 0          # synchronises the stream
    ref = api.mxattn_forward(q.to(dev), k.to(dev), v.to(dev), causal=cfg.causal, scale_mode=mode,
                             out_dtype=out_dtype).cpu()
    assert torch.equal(out_h, ref)


def test_host_pipeline_is_ordered_on_the_callers_stream(dev):
    """The call runs on side streams of its own, but it must start after, and finish before, the
    work around it on the caller's stream. Here the pinned inputs are filled by copies queued on a
    non-default stream just before each call, two calls with different inputs share one
    workspace, and the outputs are read after that stream alone has been synchronised."""
    cfg = synthetic.ATTN_CONFIGS["llm_gqa"].scaled(B=2, N=4096)       # chunks of 2, 4, 4, 4, 2 KV heads
    q, k, v = synthetic.attn_inputs(cfg)
    q2, k2, v2 = (-t for t in (q, k, v))
    n = api._lib.load().mxattn_forward_host_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.d, 0)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    dev_inputs = [tuple(t.to(dev) for t in x) for x in ((q, k, v), (q2, k2, v2))]
    pinned = [tuple(torch.zeros(t.shape, dtype=t.dtype).pin_memory() for t in (q, k, v)) for _ in range(2)]
    outs = [torch.zeros(q.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    side = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(side):
        for i in range(2):
            for h, d_ in zip(pinned[i], dev_inputs[i]):
                h.copy_(d_, non_blocking=True)
            api.mxattn_forward_host(*pinned[i], outs[i], causal=cfg.causal, workspace=ws, device=dev)
    side.synchronize()
    for i in range(2):
        ref = api.mxattn_forward(*dev_inputs[i], causal=cfg.causal).cpu()
        assert torch.equal(outs[i], ref), i
    assert api.mxattn_check_status(ws) == 0

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

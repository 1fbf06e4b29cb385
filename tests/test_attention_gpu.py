"""GPU parity of the fused MXFP4 attention kernel against the oracle.

Small shapes are compared on every row (outputs) and on whole heads (P~ codes); the full-size
workloads are run in the benchmark's launch configuration and compared on sampled rows, which
the oracle computes exactly (rows are independent under the online softmax).
"""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import api, build, synthetic
from oracle import attention as oa
from oracle import mxfp4 as mx
from tests import parity

pytestmark = pytest.mark.gpu
MODES = [(mx.SCALE_UOS, True), (mx.SCALE_OCP, False), (mx.SCALE_UOS, False), (mx.SCALE_OCP, True),
         (mx.SCALE_UOS, oa.P_EFQ), (mx.SCALE_OCP, oa.P_EFQ)]


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return torch.device("cuda:0")


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).bfloat16()


def _rand_qkv(B, Hq, Hkv, N, d, seed, qk_scale=1.0):
    rng = np.random.default_rng(seed)
    return (_bf16(rng.standard_normal((B, Hq, N, d)) * qk_scale),
            _bf16(rng.standard_normal((B, Hkv, N, d)) * qk_scale),
            _bf16(rng.standard_normal((B, Hkv, N, d))))


def _oracle_head(q, k, v, b, h, rows, causal, mode, pnq):
    """Oracle rows (and their P~ record) of query head h of batch b."""
    Hq, Hkv = q.shape[1], k.shape[1]
    g = h // (Hq // Hkv)
    (qd, kd, vd), _ = oa.dequantized_qkv(q[b, h].double().numpy(), k[b, g].double().numpy(),
                                         v[b, g].double().numpy(), mode)
    return oa.attention_rows(qd[rows], rows, kd, vd, causal=causal, mode=mode, pnq=pnq, record_p=True)


def _run_and_check(dev, q, k, v, causal, mode, pnq, check_heads, rows_of=None, full_out=True):
    B, Hq, N, d = q.shape
    qd_, kd_, vd_ = q.to(dev), k.to(dev), v.to(dev)
    ws = api.alloc_workspace(B, Hq, k.shape[1], N, d, dev)
    out = api.mxattn_forward(qd_, kd_, vd_, causal=causal, scale_mode=mode, pnq=pnq, workspace=ws)
    assert api.mxattn_check_status(ws) == 0
    out = out.cpu().numpy()
    assert np.isfinite(out).all()
    stats = []
    for (b, h) in check_heads:
        rows = np.arange(N) if rows_of is None else rows_of(b, h)
        r0, r1 = int(rows.min()), int(rows.max()) + 1
        ref, rec = _oracle_head(q, k, v, b, h, np.arange(r0, r1), causal, mode, pnq)
        _, pc, ps = api.mxattn_forward_debug(qd_, kd_, vd_, b * Hq + h, r0, r1, causal=causal,
                                             scale_mode=mode, pnq=pnq, workspace=ws)
        assert api.mxattn_check_status(ws) == 0
        cls = parity.classify_p_mismatches(pc.cpu().numpy(), ps.cpu().numpy(), rec, mode, N)
        stats.append(cls)
        assert cls["unexplained"] == 0, cls
        assert cls["rate"] <= parity.P_MISMATCH_RATE, cls
        sel = rows - r0
        mabs, rfro = parity.out_errors(out[b, h, rows], ref[sel])
        assert mabs <= parity.OUT_MAX_ABS, (b, h, mabs, rfro, cls)
        assert rfro <= parity.OUT_REL_FRO, (b, h, mabs, rfro, cls)
    return out, stats


@pytest.mark.parametrize("mode,pnq", MODES)
def test_tiny_workload_all_modes(dev, mode, pnq):
    cfg = synthetic.ATTN_CONFIGS["tiny"]
    q, k, v = synthetic.attn_inputs(cfg)
    _run_and_check(dev, q, k, v, cfg.causal, mode, pnq, [(0, 0), (0, 1)])


@pytest.mark.parametrize("N", [1, 31, 100, 128, 129, 300, 511])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes(dev, N, d, causal):
    q, k, v = _rand_qkv(1, 4, 2, N, d, seed=N + d + causal, qk_scale=1.5)
    _run_and_check(dev, q, k, v, causal, mx.SCALE_UOS, True, [(0, 0), (0, 3)])


@pytest.mark.parametrize("N", [1, 100, 129, 300, 511])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_exp_free(dev, N, d, causal):
    q, k, v = _rand_qkv(1, 4, 2, N, d, seed=1000 + N + d + causal, qk_scale=1.5)
    _run_and_check(dev, q, k, v, causal, mx.SCALE_UOS, oa.P_EFQ, [(0, 0), (0, 3)])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_odd_tile_count_long_rows(dev, d, causal):
    """An odd number of query tiles (the last tile pair of each head has no tile B, so one P~V
    issuer has no product at any key tile) with more key tiles than pipeline stages (6 for
    d = 128, 8 for d = 64), and more tile pairs than SMs."""
    N = 1100                                       # 9 query tiles, 9 key tiles
    q, k, v = _rand_qkv(1, 72, 18, N, d, seed=2000 + d + causal, qk_scale=1.5)
    _run_and_check(dev, q, k, v, causal, mx.SCALE_UOS, True, [(0, 0), (0, 37), (0, 71)])


@pytest.mark.parametrize("mode,pnq", [(mx.SCALE_OCP, oa.P_EFQ), (mx.SCALE_UOS, False)])
def test_odd_tile_count_other_rules(dev, mode, pnq):
    q, k, v = _rand_qkv(2, 40, 8, 1100, 128, seed=2100 + int(pnq), qk_scale=1.5)
    _run_and_check(dev, q, k, v, True, mode, pnq, [(0, 5), (1, 39)])


def test_bf16_output_ragged_odd_tiles(dev):
    q, k, v = _rand_qkv(1, 64, 16, 1100, 64, seed=2200)
    o32 = api.mxattn_forward(q.to(dev), k.to(dev), v.to(dev), causal=True)
    o16 = api.mxattn_forward(q.to(dev), k.to(dev), v.to(dev), causal=True, out_dtype=torch.bfloat16)
    assert torch.equal(o16.float(), o32.bfloat16().float())


def test_gqa_and_batches(dev):
    q, k, v = _rand_qkv(2, 8, 2, 200, 128, seed=11)
    _run_and_check(dev, q, k, v, True, mx.SCALE_UOS, True, [(0, 0), (0, 5), (1, 3), (1, 7)])


def test_bf16_output_matches_fp32(dev):
    q, k, v = _rand_qkv(1, 2, 2, 256, 128, seed=12)
    o32 = api.mxattn_forward(q.to(dev), k.to(dev), v.to(dev), causal=False)
    o16 = api.mxattn_forward(q.to(dev), k.to(dev), v.to(dev), causal=False, out_dtype=torch.bfloat16)
    assert torch.equal(o16.float(), o32.bfloat16().float())


def _sample_rows(cfg, rng, n_per_head=24):
    N = cfg.N
    last_tile = (N - 1) // 128 * 128
    fixed = np.array([0, 1, 127, 128, last_tile, N - 1])
    extra = rng.choice(N, n_per_head - fixed.size, replace=False)
    return np.unique(np.concatenate([fixed, extra]))


def _p_slabs(cfg, rng):
    """Row slabs for the full-size P~ comparison: 64 rows each from the first query tile, a middle
    one, the last (partial) one and a random one -- 256 rows per head. For the causal workload the
    middle and random slabs straddle a tile's diagonal block."""
    N = cfg.N
    last = (N - 1) // 128 * 128
    mid = (N // 2) // 128 * 128
    rnd = int(rng.integers(1, max(2, N // 128 - 1))) * 128
    return [(0, 64), (mid + 32, mid + 96), (max(0, N - 64), N), (rnd, rnd + 64)]


FULL_SIZE_CASES = [("video_dit", mx.SCALE_UOS, True), ("video_dit_long", mx.SCALE_UOS, True),
                   ("video_dit_long", mx.SCALE_OCP, False), ("llm_gqa", mx.SCALE_UOS, True)]


@pytest.mark.parametrize("name,mode,pnq", FULL_SIZE_CASES)
def test_full_size_sampled(dev, name, mode, pnq):
    cfg = synthetic.ATTN_CONFIGS[name]
    q, k, v = synthetic.attn_inputs(cfg)
    B, Hq, Hkv, N, d = cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.d
    dq, dk, dv = q.to(dev), k.to(dev), v.to(dev)
    ws = api.alloc_workspace(B, Hq, Hkv, N, d, dev)
    out = api.mxattn_forward(dq, dk, dv, causal=cfg.causal, scale_mode=mode, pnq=pnq, workspace=ws)
    assert api.mxattn_check_status(ws) == 0
    rng = np.random.default_rng(99)
    heads = [(0, 0), (B - 1, Hq - 1), (int(rng.integers(B)), int(rng.integers(1, Hq - 1)))]
    n_p = n_mis = 0
    for (b, h) in heads:
        g = h // (Hq // Hkv)
        (qd, kd, vd), _ = oa.dequantized_qkv(q[b, h].double().numpy(), k[b, g].double().numpy(),
                                             v[b, g].double().numpy(), mode)
        # outputs of sampled rows
        rows = _sample_rows(cfg, rng)
        ref = oa.attention_rows(qd[rows], rows, kd, vd, causal=cfg.causal, mode=mode, pnq=pnq)
        mabs, rfro = parity.out_errors(out[b, h, rows].cpu().numpy(), ref)
        assert mabs <= parity.OUT_MAX_ABS and rfro <= parity.OUT_REL_FRO, (name, b, h, mabs, rfro)
        # P~ codes and scales of 256 rows in four slabs, through the debug dump
        for (r0, r1) in _p_slabs(cfg, rng):
            _, pc, ps = api.mxattn_forward_debug(dq, dk, dv, b * Hq + h, r0, r1, causal=cfg.causal,
                                                 scale_mode=mode, pnq=pnq, workspace=ws)
            assert api.mxattn_check_status(ws) == 0
            srows = np.arange(r0, r1)
            _, rec = oa.attention_rows(qd[srows], srows, kd, vd, causal=cfg.causal, mode=mode, pnq=pnq,
                                       record_p=True)
            cls = parity.classify_p_mismatches(pc.cpu().numpy(), ps.cpu().numpy(), rec, mode, N)
            assert cls["unexplained"] == 0, (name, b, h, r0, cls)
            n_p += cls["n"]
            n_mis += cls["mismatches"]
    assert n_mis <= parity.P_MISMATCH_RATE * n_p, (name, n_mis, n_p)

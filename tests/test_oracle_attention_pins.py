"""Pins for the CPU oracle of MXFP4 attention (tiled online softmax, UOS/OCP, PNQ).

* With every MXFP4 step off, the tiled loop must equal plain fp64 softmax attention
  (the EFQ-Softmax abstract: row-max update, history rescale, accumulation and final
  normalisation are the FlashAttention ones, unchanged), for any tile width.
* PNQ preserves normalisation by construction (MXAttention abstract): with V = 1 every
  output is exactly the sum of the final weights, which must be 1 to fp64 rounding;
  the exp-then-quantize path (pnq=0) must visibly miss it.
* A case solvable by hand: identical keys make every score equal, so P~ = 1 everywhere,
  which encodes as 4.0 with scale 2^-2, and the output is the mean of dequantized V.
* The paper's quality claim, as an expectation: on the tiny seeded workload UOS+PNQ
  against fp64 attention versus the OCP rule with the conventional row sum. Measured, it
  does not hold on seed 0 (kept as a strict xfail with the numbers); isolated to the
  softmax stage, the ordering holds with a wide margin.
"""
import numpy as np
import pytest
import torch

from mxfp4_microscaled_bit_quantize_b200 import synthetic
from oracle import attention as oa
from oracle import mxfp4 as mx


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).bfloat16().double().numpy()


def _rand_qkv(B, Hq, Hkv, N, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    q = _bf16(rng.standard_normal((B, Hq, N, d)) * scale)
    k = _bf16(rng.standard_normal((B, Hkv, N, d)) * scale)
    v = _bf16(rng.standard_normal((B, Hkv, N, d)))
    return q, k, v


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 31, 129, 200])
def test_loop_equals_softmax_without_quantization(causal, N):
    q, k, v = _rand_qkv(1, 4, 2, N, 64, seed=N, scale=2.0)
    ref = oa.softmax_attention_fp64(q, k, v, causal=causal)
    for tile in (32, 64, 128):
        got = oa.mxattention(q, k, v, causal=causal, mode=mx.SCALE_UOS, pnq=True,
                             kv_tile=tile, quantize=False)
        assert np.max(np.abs(got - ref)) <= 1e-12


@pytest.mark.parametrize("mode", [mx.SCALE_OCP, mx.SCALE_UOS, 2])
def test_pnq_preserves_normalisation(mode):
    rng = np.random.default_rng(3)
    N, d = 300, 64
    q = _bf16(rng.standard_normal((1, 2, N, d)) * 3.0)    # sharp rows
    k = _bf16(rng.standard_normal((1, 2, N, d)) * 3.0)
    v = np.ones((1, 2, N, d))
    # every V entry dequantizes to one constant: 1 in MXFP4 (code 1.0, scale 2^-2 ... exact), and
    # 6 * E4M3(1/6) = 1.03125 in NVFP4; a normalised softmax must return exactly that constant
    (_, _, vd), _ = oa.dequantized_qkv(q[0, 0], k[0, 0], v[0, 0], mode)
    vconst = vd[0, 0]
    assert np.all(vd == vconst)
    out_pnq = oa.mxattention(q, k, v, causal=False, mode=mode, pnq=True)
    out_conv = oa.mxattention(q, k, v, causal=False, mode=mode, pnq=False)
    assert np.max(np.abs(out_pnq - vconst)) <= 1e-12
    assert np.max(np.abs(out_conv - vconst)) > 1e-3       # numerator/denominator mismatch
    out_causal = oa.mxattention(q, k, v, causal=True, mode=mode, pnq=True)
    assert np.max(np.abs(out_causal - vconst)) <= 1e-12


def test_uniform_scores_by_hand():
    N, d = 96, 64
    q = np.full((1, 1, N, d), 0.5)
    k = np.full((1, 1, N, d), 0.25)
    rng = np.random.default_rng(9)
    v = _bf16(rng.standard_normal((1, 1, N, d)))
    out, rec = None, None
    (qd, kd, vd), _ = oa.dequantized_qkv(q[0, 0], k[0, 0], v[0, 0], mx.SCALE_UOS)
    out, rec = oa.attention_rows(qd, np.arange(N), kd, vd, causal=False, mode=mx.SCALE_UOS,
                                 pnq=True, record_p=True)
    # every P~ = 1 -> code 4 (magnitude 4.0) with scale byte 127 - 2
    valid = np.arange(rec["codes"].shape[1]) < N
    assert np.all(rec["codes"][:, valid] == 6)
    nb = -(-N // 32)
    assert np.all(rec["scales"][:, :nb] == 125)
    assert np.all(rec["scales"][:, nb:] == 0)              # all-masked padded blocks
    want = vd.mean(axis=0)
    assert np.max(np.abs(out - want[None, :])) <= 1e-15


def test_causal_first_row_is_first_value():
    # row 0 under a causal mask sees only key 0: P~ = 1, out = dq(V)_0 exactly
    q, k, v = _rand_qkv(1, 2, 1, 64, 64, seed=4)
    out = oa.mxattention(q, k, v, causal=True, mode=mx.SCALE_UOS, pnq=True)
    (_, _, vd), _ = oa.dequantized_qkv(q[0, 0], k[0, 0], v[0, 0], mx.SCALE_UOS)
    assert np.array_equal(out[0, 0, 0], vd[0])
    assert np.array_equal(out[0, 1, 0], vd[0])


def test_row_sample_equals_full():
    q, k, v = _rand_qkv(1, 2, 2, 200, 64, seed=5)
    full = oa.mxattention(q, k, v, causal=True, mode=mx.SCALE_UOS, pnq=True)
    rows = {(0, 1): np.array([0, 17, 128, 199])}
    part = oa.mxattention(q, k, v, causal=True, mode=mx.SCALE_UOS, pnq=True, rows=rows)
    assert np.array_equal(part[0, 1, rows[(0, 1)]], full[0, 1, rows[(0, 1)]])
    assert np.isnan(part[0, 0]).all()


def test_gqa_head_mapping():
    # query heads 0,1 share KV head 0; heads 2,3 share KV head 1 (contiguous groups)
    q, k, v = _rand_qkv(1, 4, 2, 64, 64, seed=6)
    got = oa.mxattention(q, k, v, causal=False, mode=mx.SCALE_UOS, pnq=True, quantize=False)
    kk = np.repeat(k, 2, axis=1)
    vv = np.repeat(v, 2, axis=1)
    ref = oa.softmax_attention_fp64(q, kk, vv, causal=False)
    assert np.max(np.abs(got - ref)) <= 1e-12


def _tiny_inputs(seed=0, v_offset=0.0):
    cfg = synthetic.ATTN_CONFIGS["tiny"].scaled(seed=seed)
    q, k, v = (t.double().numpy() for t in synthetic.attn_inputs(cfg))
    return q, k, v + v_offset


@pytest.mark.xfail(strict=True, reason=(
    "measured, not tuned: on the tiny workload (zero-mean V, x20 outliers in Q/K) the output "
    "error is dominated by Q/K quantization in near one-hot rows, and PNQ's renormalisation "
    "noise is visible while the normalisation error it removes is not; seed 0 gives "
    "UOS+PNQ 0.546 vs OCP exp-then-quantize 0.523 relative Frobenius error"))
def test_mode_ordering_on_tiny_workload():
    q, k, v = _tiny_inputs()
    ref = oa.softmax_attention_fp64(q, k, v, causal=False)
    uos = oa.mxattention(q, k, v, causal=False, mode=mx.SCALE_UOS, pnq=True)
    ocp = oa.mxattention(q, k, v, causal=False, mode=mx.SCALE_OCP, pnq=False)
    e_uos, e_ocp = mx.rel_frobenius(uos, ref), mx.rel_frobenius(ocp, ref)
    assert e_uos <= e_ocp, (e_uos, e_ocp)


def _p_only(q, k, v, mode, pnq):
    """Quantize only P~ (Q, K, V kept exact): isolates the softmax-loop error."""
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        out[0, h] = oa.attention_rows(q[0, h], np.arange(q.shape[2]), k[0, h], v[0, h],
                                      causal=False, mode=mode, pnq=pnq)
    return out


def test_softmax_stage_error_ordering():
    """The softmax-stage error the two components target, isolated from Q/K/V quantization:
    UOS beats OCP at either PNQ setting, and when V rows share a common component (the
    case where a wrong row sum visibly rescales the output) UOS+PNQ beats OCP with the
    exp-then-quantize row sum by a wide margin."""
    q, k, v = _tiny_inputs()
    ref = oa.softmax_attention_fp64(q, k, v, causal=False)
    for pnq in (False, True):
        e_u = mx.rel_frobenius(_p_only(q, k, v, mx.SCALE_UOS, pnq), ref)
        e_o = mx.rel_frobenius(_p_only(q, k, v, mx.SCALE_OCP, pnq), ref)
        assert e_u < e_o, (pnq, e_u, e_o)
    v2 = v + 2.0
    ref2 = oa.softmax_attention_fp64(q, k, v2, causal=False)
    e_best = mx.rel_frobenius(_p_only(q, k, v2, mx.SCALE_UOS, True), ref2)
    e_base = mx.rel_frobenius(_p_only(q, k, v2, mx.SCALE_OCP, False), ref2)
    assert e_best * 1.5 < e_base, (e_best, e_base)


def test_uniform_scores_by_hand_nvfp4():
    """NVFP4 mode: every P~ = 1 -> fp32(1/6) rounds to the E4M3 scale 1.375 * 2^-3 = 0.171875
    (byte 0x23: exponent field 4, mantissa 3), 1 / 0.171875 = 5.82 rounds to the top E2M1 value 6
    (code 7); all weights equal, so the output is the mean of the dequantized V rows."""
    from oracle import nvfp4 as nv
    N, d = 80, 64
    q = np.full((1, 1, N, d), 0.5)
    k = np.full((1, 1, N, d), 0.25)
    rng = np.random.default_rng(10)
    v = _bf16(rng.standard_normal((1, 1, N, d)))
    (qd, kd, vd), _ = oa.dequantized_qkv(q[0, 0], k[0, 0], v[0, 0], nv.SCALE_NVFP4)
    out, rec = oa.attention_rows(qd, np.arange(N), kd, vd, causal=False, mode=nv.SCALE_NVFP4,
                                 pnq=True, record_p=True)
    valid = np.arange(rec["codes"].shape[1]) < N
    assert np.all(rec["codes"][:, valid] == 7)
    nb = N // 16
    assert np.all(rec["scales"][:, :nb] == 0x23)
    assert np.all(rec["scales"][:, nb:] == 0)              # all-masked padded blocks
    assert np.max(np.abs(out - vd.mean(axis=0)[None, :])) <= 1e-14

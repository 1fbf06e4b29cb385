"""CPU oracle for MXFP4 attention forward with UOS / OCP scaling and PNQ (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the library calls this module; only the test
suite, the package smoke check and the benchmark's CPU-baseline leg may import it.
It shares no code with the CUDA sources.

What it follows
---------------
MXAttention abstract (the UOS and PNQ sentences) and the EFQ-Softmax abstract (the
FlashAttention loop it keeps: "row-maximum update, historical rescaling,
high-precision accumulation, and final normalization remain unchanged"; the low-bit
probability operand "used consistently in both the P~V numerator update and the P~1
denominator update"):

For one query row i of query head h (KV head g = h // (Hq/Hkv)), softmax scale
sigma = 1/sqrt(d), keys visited in tiles of ``kv_tile`` keys in increasing key order:

  m = -inf, l = 0, acc = 0
  for each tile:
      s_j  = sigma * <dq(Q)_i, dq(K)_j>                 (fp64; -inf if masked)
      m'   = max(m, max_j s_j);   alpha = exp(m - m')    (alpha = 0 while m = -inf)
      p_j  = exp(s_j - m')                               (masked -> 0)
      q_j  = dq(MXFP4(p)_j), blocks of 32 keys            (PNQ operand)
      l    = alpha * l + sum_j (q_j if pnq else p_j)
      acc  = alpha * acc + sum_j q_j * dq(V)_j
      m    = m'
  out_i = acc / l

With pnq=1 the same dequantized operand q feeds the numerator and the denominator
(Pre-Normalization Quantization). With pnq=0 the denominator sums the unquantized p:
the "exp-then-quantize" path whose numerator/denominator mismatch the EFQ-Softmax
abstract describes.

Readings taken where the pages are silent (each also listed in the design notes):
* Q, K are quantized along the head dimension, V and P~ along keys, all with the
  same scale rule; raw Q is quantized (sigma is applied to the fp32/fp64 scores).
* The running max includes the current tile and every change of it rescales the
  history (no lazy rescale): P~ codes depend on the max in force when a tile is
  quantized, so tile width and key order are part of the definition.
* Decision precision: a quantised code is an integer decided by floating point, so
  the oracle takes it in the kernel's precision: each p_j is rounded to fp32 before
  its block amax, scale exponent and code are chosen. Everything else stays fp64.
* Keys >= N and (causal) keys > i are masked: p = 0, code +0; an all-masked 32-key
  block gets scale byte 0x00.
* pnq = 2 (P_EFQ) replaces exp-then-quantize by the exp-free rule of oracle/efq.py (EFQ-Softmax
  abstract): the codes come from the base-2 shifted scores through one affine map, and that
  operand feeds both the numerator and the denominator, as under PNQ. MXFP4 modes only.
* mode = 2 (nvfp4.SCALE_NVFP4) is the NVFP4 comparison format of oracle/nvfp4.py for all four
  operands: blocks of 16 with E4M3 scales; P~ blocks are 16 keys, each decision again taken on
  the fp32-rounded P~ (scale byte from fp32(amax / 6), element from fp32(p / s)).
"""
from __future__ import annotations

import numpy as np

from . import efq
from . import mxfp4 as mx
from . import nvfp4 as nv

KV_TILE = 128         # the library's documented tile width (MXATTN_KV_TILE)
P_CONVENTIONAL, P_PNQ, P_EFQ = 0, 1, 2     # the `pnq` argument: rule of the P~ operand and row sum
LOG2E = 1.0 / np.log(2.0)


def dequantized_qkv(q, k, v, mode: int):
    """Quantize bf16-valued Q [..,N,d], K [..,N,d] along d and V along keys; return fp64
    dequantized copies (V as [.., N, d]) and the raw codes/scales for bit-exact checks."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = q.shape[-2], q.shape[-1]
    if mode == nv.SCALE_NVFP4:
        qc, qs = nv.quantize_rows(q)
        kc, ks = nv.quantize_rows(k)
        vc, vs = nv.quantize_rows(np.swapaxes(v, -1, -2))  # [.., d, ceil(N/16)*8], [.., d, ceil(N/16)]
        qd = nv.dequantize_rows(qc, qs, d)
        kd = nv.dequantize_rows(kc, ks, d)
        vd = np.swapaxes(nv.dequantize_rows(vc, vs, N), -1, -2)
        return (qd, kd, vd), dict(qc=qc, qs=qs, kc=kc, ks=ks, vc=vc, vs=vs)
    qc, qs = mx.quantize_rows(q, mode)
    kc, ks = mx.quantize_rows(k, mode)
    vc, vs = mx.quantize_transposed(v, mode)            # [.., d, Npad/2], [.., d, Npad/32]
    qd = mx.dequantize_rows(qc, qs, d)
    kd = mx.dequantize_rows(kc, ks, d)
    vd = np.swapaxes(mx.dequantize_rows(vc, vs, N), -1, -2)
    return (qd, kd, vd), dict(qc=qc, qs=qs, kc=kc, ks=ks, vc=vc, vs=vs)


def block_size(mode: int) -> int:
    return nv.BLOCK if mode == nv.SCALE_NVFP4 else mx.BLOCK


def _quantize_p(p32: np.ndarray, mode: int):
    """PNQ step: round trip of P~ rows along keys in the mode's format (MXFP4: blocks of 32
    absolute keys; NVFP4: blocks of 16). p32: [R, T] with T a multiple of the block.
    Returns (dequantized fp64, codes, scale bytes)."""
    R, T = p32.shape
    if mode == nv.SCALE_NVFP4:
        pb = p32.astype(np.float64).reshape(R, T // nv.BLOCK, nv.BLOCK)
        codes, sbytes = nv.quantize_blocks(pb)
        deq = mx.e2m1_decode(codes) * nv.e4m3_decode(sbytes)[..., None]
        return deq.reshape(R, T), codes.reshape(R, T), sbytes
    pb = p32.astype(np.float64).reshape(R, T // mx.BLOCK, mx.BLOCK)
    codes, e = mx.quantize_blocks(pb, mode)
    deq = np.ldexp(mx.e2m1_decode(codes), e[..., None]).reshape(R, T)
    return deq, codes.reshape(R, T), (e + mx.E8M0_BIAS).astype(np.uint8)


def attention_rows(qd_rows, row_idx, kd, vd, *, causal: bool, mode: int, pnq: bool,
                   kv_tile: int = KV_TILE, quantize_p: bool = True, record_p: bool = False):
    """Tiled online-softmax MXFP4 attention for selected query rows of one head.

    qd_rows: [R, d] dequantized query rows; row_idx: [R] their positions (for causal).
    kd, vd:  [N, d] dequantized keys / values of the matching KV head.
    quantize_p=False turns the PNQ step off (a check of the loop: the result is then
    plain softmax attention on the given operands).
    Returns out [R, d] (and, with record_p, the P~ codes/scales/margins per row).
    """
    qd_rows = np.asarray(qd_rows, dtype=np.float64)
    row_idx = np.asarray(row_idx, dtype=np.int64)
    N, d = kd.shape
    blk = block_size(mode)
    rule = int(pnq)
    if rule == P_EFQ and mode == nv.SCALE_NVFP4:
        raise ValueError("the exp-free P~ rule is defined for MXFP4 (power-of-two block scales) only")
    assert kv_tile % mx.BLOCK == 0
    R = qd_rows.shape[0]
    sigma = 1.0 / np.sqrt(d)
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    acc = np.zeros((R, d))
    n_tiles = -(-N // kv_tile)
    if record_p:
        npad = n_tiles * kv_tile
        rec_codes = np.zeros((R, npad), dtype=np.uint8)
        rec_scales = np.zeros((R, npad // blk), dtype=np.uint8)
        rec_y = np.zeros((R, npad))
        rec_amax = np.zeros((R, npad // blk))
        rec_z = np.full((R, npad), -np.inf)
        rec_zmag = np.zeros((R, npad))
    for t in range(n_tiles):
        j0 = t * kv_tile
        keys = np.arange(j0, j0 + kv_tile)
        valid = keys < N
        kj = np.zeros((kv_tile, d))
        vj = np.zeros((kv_tile, d))
        kj[valid] = kd[keys[valid]]
        vj[valid] = vd[keys[valid]]
        s = sigma * (qd_rows @ kj.T)                       # [R, kv_tile]
        mask = np.broadcast_to(~valid[None, :], s.shape).copy()
        if causal:
            mask |= keys[None, :] > row_idx[:, None]
        s[mask] = -np.inf
        m_new = np.maximum(m, s.max(axis=1))
        with np.errstate(invalid="ignore"):
            alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))
            p = np.where(mask, 0.0, np.exp(s - m_new[:, None]))
        if quantize_p and rule == P_EFQ:
            with np.errstate(invalid="ignore"):
                u = np.where(mask, -np.inf, (s - m_new[:, None]) * LOG2E)   # log2 P~
            qv, codes, sbytes, z = efq.efq_quantize_p(u, mode)
            denom = qv
            if record_p:
                rec_codes[:, j0:j0 + kv_tile] = codes
                nb0 = j0 // blk
                rec_scales[:, nb0:nb0 + kv_tile // blk] = sbytes
                rec_z[:, j0:j0 + kv_tile] = z
                # magnitude of the terms that form 2 r + 2 (scores, running max, block exponent):
                # the scale of the fp32 rounding a kernel makes in it
                e_el = np.repeat(sbytes.astype(np.float64) - mx.E8M0_BIAS, blk, axis=1)
                with np.errstate(invalid="ignore"):
                    rec_zmag[:, j0:j0 + kv_tile] = 2.0 * (np.abs(np.where(mask, 0.0, s)) + np.abs(m_new)[:, None]) \
                        * LOG2E + 2.0 * np.abs(e_el) + 2.0
                with np.errstate(over="ignore"):
                    rec_amax[:, nb0:nb0 + kv_tile // blk] = np.exp2(u.reshape(R, -1, blk).max(axis=-1)).astype(
                        np.float32)
        elif quantize_p:
            p32 = p.astype(np.float32)                     # decision precision: fp32
            qv, codes, sbytes = _quantize_p(p32, mode)
            denom = qv if rule != P_CONVENTIONAL else p32.astype(np.float64)
            if record_p:
                rec_codes[:, j0:j0 + kv_tile] = codes
                nb0 = j0 // blk
                rec_scales[:, nb0:nb0 + kv_tile // blk] = sbytes
                pbk = p32.astype(np.float64).reshape(R, -1, blk)
                if mode == nv.SCALE_NVFP4:   # y = fp32(p / s), amax recorded as fp32(amax / 6)
                    s_ = nv.e4m3_decode(sbytes)[..., None]
                    with np.errstate(divide="ignore", invalid="ignore"):
                        yv = np.where(s_ > 0, (pbk / s_).astype(np.float32), 0.0)
                    rec_y[:, j0:j0 + kv_tile] = yv.reshape(R, -1)
                    rec_amax[:, nb0:nb0 + kv_tile // blk] = (pbk.max(axis=-1) / 6.0).astype(np.float32)
                else:
                    e = sbytes.astype(np.int64) - mx.E8M0_BIAS
                    rec_y[:, j0:j0 + kv_tile] = np.ldexp(pbk, -e[..., None]).reshape(R, -1)
                    rec_amax[:, nb0:nb0 + kv_tile // blk] = pbk.max(axis=-1)
        else:
            qv = p
            denom = p
        l = alpha * l + denom.sum(axis=1)
        acc = alpha[:, None] * acc + qv @ vj
        m = m_new
    out = acc / l[:, None]
    if record_p:
        return out, dict(codes=rec_codes, scales=rec_scales, y=rec_y, amax=rec_amax, z=rec_z, zmag=rec_zmag,
                         rule=rule)
    return out


def mxattention(q, k, v, *, causal: bool, mode: int, pnq: bool, kv_tile: int = KV_TILE,
                rows=None, quantize=True):
    """MXFP4 attention forward for [B, Hq, N, d] Q and [B, Hkv, N, d] K/V (bf16 values).

    rows: None for every row, or a dict {(b, h): row index array} to compute only those
    rows (rows are independent under the online softmax, so a sample is exact for them).
    quantize=False skips every MXFP4 step (fp64 tiled softmax attention on raw inputs).
    Returns out [B, Hq, N, d] (NaN where a row was not computed).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    assert Hq % Hkv == 0
    group = Hq // Hkv
    out = np.full(q.shape, np.nan)
    for b in range(B):
        for g in range(Hkv):
            if quantize:
                (qd_g, kd, vd), _ = dequantized_qkv(q[b, g * group:(g + 1) * group], k[b, g],
                                                    v[b, g], mode)
            else:
                qd_g, kd, vd = q[b, g * group:(g + 1) * group], k[b, g], v[b, g]
            for hh in range(group):
                h = g * group + hh
                idx = np.arange(N) if rows is None else np.asarray(rows.get((b, h), []))
                if idx.size == 0:
                    continue
                out[b, h, idx] = attention_rows(qd_g[hh][idx], idx, kd, vd, causal=causal,
                                                mode=mode, pnq=pnq, kv_tile=kv_tile,
                                                quantize_p=quantize)
    return out


def softmax_attention_fp64(q, k, v, *, causal: bool):
    """Plain softmax(sigma Q K^T) V in fp64 on the given operands (no tiling, no quantization)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, N, d = q.shape
    group = Hq // k.shape[1]
    out = np.empty_like(q)
    for b in range(B):
        for h in range(Hq):
            s = (q[b, h] @ k[b, h // group].T) / np.sqrt(d)
            if causal:
                s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            w = np.exp(s)
            out[b, h] = (w / w.sum(axis=1, keepdims=True)) @ v[b, h // group]
    return out

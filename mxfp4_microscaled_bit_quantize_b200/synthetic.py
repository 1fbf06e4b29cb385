"""Seeded synthetic workloads for MXFP4 attention and the standalone quantizer.

This module only draws random numbers and shapes them into bf16 tensors; it holds
none of the MXFP4 arithmetic. Both the CUDA path and the CPU oracle consume the
same tensors produced here, so neither side depends on the other.

Every random stream is keyed by (seed, tensor id, batch, head) or (seed, tensor id,
row chunk), so one head (or one row chunk) can be regenerated on its own: the
oracle re-creates just the heads it samples without materialising a full
video-sized tensor.

Workload recipes (shapes follow the workloads named by the MXAttention abstract:
video diffusion transformers such as Wan2.2 and HunyuanVideo, and the LLM prefill
setting of the EFQ-Softmax abstract; the numbers themselves are synthetic):

* ``tiny``: B=1, H=2, N=256, d=64. Q, K, V iid N(0,1); each entry is independently
  multiplied by 20 with probability 0.005 (an outlier mask per tensor).
* ``quantizer``: a 65536 x 1024 matrix. Each element is N(0,1) with probability 0.9,
  else Laplace(0, b=3); then 0.1% of the entries are multiplied by 50.
* ``video_dit``: B=1, H=40, N=32760 (21x39x40 latent tokens), d=128. Q, K ~ N(0,1)
  with 4 seeded channels per head scaled by 8 (the same channels in Q and K); V ~ N(0,1).
* ``video_dit_long``: B=1, H=24, N=76800, d=128. As ``video_dit``, and K also gets a
  per-(head, token) bias drawn from N(0, 0.5^2) added to all of its channels.
* ``llm_gqa``: B=4, Hq=32, Hkv=8, N=8192, d=128, causal. Q/K channels 0..15 scaled
  by 6, then rotary position embedding (base 1e6, rotate-half pairs (c, c+d/2),
  positions 0..N-1) applied in fp32; V ~ N(0,1).

All tensors are produced as fp32 and rounded to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

_Q, _K, _V, _CHAN, _KBIAS = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class AttnConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    seed: int
    recipe: str  # "iid_outlier" | "channel_outlier" | "channel_outlier_kbias" | "rope"

    def scaled(self, **kw) -> "AttnConfig":
        """Same recipe at another size (used for parity cases that the oracle finishes quickly)."""
        return dataclasses.replace(self, **kw)

    @property
    def flops(self) -> float:
        f = 4.0 * self.B * self.Hq * float(self.N) * float(self.N) * self.d
        return f / 2.0 if self.causal else f

    def describe(self) -> dict:
        return {"B": self.B, "Hq": self.Hq, "Hkv": self.Hkv, "N": self.N, "d": self.d,
                "causal": self.causal, "seed": self.seed, "recipe": self.recipe}


ATTN_CONFIGS = {
    "tiny": AttnConfig("tiny", 1, 2, 2, 256, 64, False, 0, "iid_outlier"),
    "video_dit": AttnConfig("video_dit", 1, 40, 40, 32760, 128, False, 2, "channel_outlier"),
    "video_dit_long": AttnConfig("video_dit_long", 1, 24, 24, 76800, 128, False, 3,
                                 "channel_outlier_kbias"),
    "llm_gqa": AttnConfig("llm_gqa", 4, 32, 8, 8192, 128, True, 4, "rope"),
}

QUANT_ROWS, QUANT_COLS, QUANT_SEED = 65536, 1024, 1


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(k) for k in key])


def _to_bf16(a32: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a32, dtype=np.float32)).to(torch.bfloat16)


def _rope_tables(N: int, d: int, base: float = 1.0e6):
    half = d // 2
    inv = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = np.arange(N, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def _apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    half = x.shape[1] // 2
    lo, hi = x[:, :half], x[:, half:]
    out = np.empty_like(x)
    out[:, :half] = lo * cos - hi * sin
    out[:, half:] = hi * cos + lo * sin
    return out


def _outlier_channels(cfg: AttnConfig, b: int, h_kv: int) -> np.ndarray:
    return _rng(cfg.seed, _CHAN, b, h_kv).choice(cfg.d, size=4, replace=False)


def head_f32(cfg: AttnConfig, which: str, b: int, h: int) -> np.ndarray:
    """fp32 values (before the bf16 rounding) of one head: which in {'q','k','v'}.

    ``h`` is a query head for 'q' and a KV head for 'k'/'v'.
    """
    tid = {"q": _Q, "k": _K, "v": _V}[which]
    rng = _rng(cfg.seed, tid, b, h)
    x = rng.standard_normal((cfg.N, cfg.d), dtype=np.float32)
    if which == "v":
        if cfg.recipe == "iid_outlier":
            mask = rng.random((cfg.N, cfg.d)) < 0.005
            x[mask] *= 20.0
        return x
    if cfg.recipe == "iid_outlier":
        mask = rng.random((cfg.N, cfg.d)) < 0.005
        x[mask] *= 20.0
    elif cfg.recipe in ("channel_outlier", "channel_outlier_kbias"):
        # Q head h and KV head h share their outlier channels (Hq == Hkv for these recipes).
        h_kv = h if which == "k" else h * cfg.Hkv // cfg.Hq
        ch = _outlier_channels(cfg, b, h_kv)
        x[:, ch] *= 8.0
        if which == "k" and cfg.recipe == "channel_outlier_kbias":
            bias = _rng(cfg.seed, _KBIAS, b, h).normal(0.0, 0.5, size=cfg.N).astype(np.float32)
            x += bias[:, None]
    elif cfg.recipe == "rope":
        x[:, :16] *= 6.0
        cos, sin = _rope_tables(cfg.N, cfg.d)
        x = _apply_rope(x, cos, sin)
    else:
        raise ValueError(cfg.recipe)
    return x


def head_bf16(cfg: AttnConfig, which: str, b: int, h: int) -> torch.Tensor:
    return _to_bf16(head_f32(cfg, which, b, h))


def attn_inputs(cfg: AttnConfig, threads: int = 8):
    """Full Q [B,Hq,N,d], K/V [B,Hkv,N,d] as contiguous CPU bf16 tensors."""
    q = torch.empty((cfg.B, cfg.Hq, cfg.N, cfg.d), dtype=torch.bfloat16)
    k = torch.empty((cfg.B, cfg.Hkv, cfg.N, cfg.d), dtype=torch.bfloat16)
    v = torch.empty((cfg.B, cfg.Hkv, cfg.N, cfg.d), dtype=torch.bfloat16)
    jobs = [(q, "q", b, h) for b in range(cfg.B) for h in range(cfg.Hq)]
    jobs += [(t, w, b, h) for (t, w) in ((k, "k"), (v, "v"))
             for b in range(cfg.B) for h in range(cfg.Hkv)]

    def run(job):
        t, w, b, h = job
        t[b, h].copy_(head_bf16(cfg, w, b, h))

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(run, jobs))
    return q, k, v


def quant_chunk_f32(row0: int, rows: int, cols: int = QUANT_COLS, seed: int = QUANT_SEED,
                    chunk: int = 4096) -> np.ndarray:
    """Rows [row0, row0+rows) of the quantizer workload (row0 and rows multiples of ``chunk``)."""
    assert row0 % chunk == 0 and rows % chunk == 0
    out = np.empty((rows, cols), dtype=np.float32)
    for c in range(rows // chunk):
        rng = _rng(seed, _Q, (row0 // chunk) + c)
        n = rng.standard_normal((chunk, cols), dtype=np.float32)
        lap = rng.laplace(0.0, 3.0, size=(chunk, cols)).astype(np.float32)
        pick = rng.random((chunk, cols)) < 0.9
        x = np.where(pick, n, lap)
        spike = rng.random((chunk, cols)) < 0.001
        x[spike] *= 50.0
        out[c * chunk:(c + 1) * chunk] = x
    return out


def quant_input(rows: int = QUANT_ROWS, cols: int = QUANT_COLS, seed: int = QUANT_SEED,
                threads: int = 8) -> torch.Tensor:
    """The standalone quantizer workload as a contiguous CPU bf16 [rows, cols] tensor."""
    chunk = 4096 if rows % 4096 == 0 else rows
    out = torch.empty((rows, cols), dtype=torch.bfloat16)

    def run(c):
        out[c * chunk:(c + 1) * chunk].copy_(
            _to_bf16(quant_chunk_f32(c * chunk, chunk, cols, seed, chunk)))

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(run, range(rows // chunk)))
    return out


# ---------------------------------------------------------------- W4A4 GEMM operands
# A (activations): N(0,1) rows with a per-row gain, log-uniform in [0.1, 10]; B (weights):
# N(0, 0.05^2). In both, 0.1% of the entries are multiplied by 20 (outliers that set their
# block's scale). Every row has its own stream, so the oracle regenerates only sampled rows.
GEMM_SHAPE = (16384, 16384, 8192)       # M, N, K of the benchmark's product
GEMM_SEED = 5
_GEMM_TAG = {"A": 21, "B": 22}


def gemm_rows_f32(which: str, rows, K: int, seed: int = GEMM_SEED) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    out = np.empty((rows.size, K), dtype=np.float32)
    for i, r in enumerate(rows):
        rng = _rng(seed, _GEMM_TAG[which], int(r))
        x = rng.standard_normal(K, dtype=np.float32)
        if which == "A":
            x *= np.float32(10.0 ** rng.uniform(-1.0, 1.0))
        else:
            x *= np.float32(0.05)
        x[rng.random(K) < 0.001] *= 20.0
        out[i] = x
    return out


def gemm_inputs(M: int, N: int, K: int, seed: int = GEMM_SEED, threads: int = 8):
    """(A bf16 [M, K], B bf16 [N, K]) as contiguous CPU tensors."""
    a = torch.empty((M, K), dtype=torch.bfloat16)
    b = torch.empty((N, K), dtype=torch.bfloat16)
    step = 1024

    def run(job):
        which, r0, dst, rows = job
        r1 = min(r0 + step, rows)
        dst[r0:r1].copy_(_to_bf16(gemm_rows_f32(which, np.arange(r0, r1), K, seed)))

    jobs = [("A", r0, a, M) for r0 in range(0, M, step)] + [("B", r0, b, N) for r0 in range(0, N, step)]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(run, jobs))
    return a, b

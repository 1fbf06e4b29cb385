"""Torch-facing wrappers of the C ABI: they only check tensors, allocate outputs with torch and
marshal pointers, sizes and the current CUDA stream. Every step of the computation runs in the
library's kernels; there is no CPU path."""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib

SCALE_OCP, SCALE_UOS, SCALE_NVFP4 = 0, 1, 2
P_CONVENTIONAL, P_PNQ, P_EFQ = 0, 1, 2   # the `pnq` argument (MXATTN_P_*): rule of the P~ operand
OUT_F32, OUT_BF16 = 0, 1
KV_TILE = 128         # keys per online-softmax tile (MXATTN_KV_TILE)
NPAD_ALIGN = 128      # the workspace pads N to a multiple of this


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def _need(t: torch.Tensor, name: str, dtype=torch.bfloat16) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def npad(N: int) -> int:
    return -(-N // NPAD_ALIGN) * NPAD_ALIGN


def mxattn_quantize(x: torch.Tensor, transpose: bool = False, scale_mode: int = SCALE_UOS, out=None):
    """MXFP4-quantize the last two axes [rows, cols] of a bf16 CUDA tensor.

    transpose=False: blocks of 32 along cols -> codes [..., rows, ceil(cols/32)*16], scales [..., rows, ceil(cols/32)].
    transpose=True:  blocks of 32 along rows -> codes [..., cols, ceil(rows/32)*16], scales [..., cols, ceil(rows/32)].
    out: optional (codes, scales) uint8 CUDA tensors of exactly those shapes, written in place.
    """
    _need(x, "x")
    if x.dim() < 2:
        raise ValueError("x must have at least 2 dimensions")
    lead = tuple(x.shape[:-2])
    rows, cols = int(x.shape[-2]), int(x.shape[-1])
    batch = math.prod(lead) if lead else 1
    nb = -(-(rows if transpose else cols) // 32)
    outer = cols if transpose else rows
    if out is None:
        codes = torch.empty(lead + (outer, nb * 16), dtype=torch.uint8, device=x.device)
        scales = torch.empty(lead + (outer, nb), dtype=torch.uint8, device=x.device)
    else:
        codes, scales = out
        for t, shape, name in ((codes, lead + (outer, nb * 16), "codes"), (scales, lead + (outer, nb), "scales")):
            _need(t, name, torch.uint8)
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    lib = _lib.load()
    st = lib.mxattn_quantize(x.data_ptr(), batch, rows, cols, int(bool(transpose)), int(scale_mode),
                             codes.data_ptr(), scales.data_ptr(), _stream(x.device))
    _lib.check(st, "mxattn_quantize")
    return codes, scales


def workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(_lib.load().mxattn_forward_workspace_size(B, Hq, Hkv, N, d))


def alloc_workspace(B: int, Hq: int, Hkv: int, N: int, d: int, device) -> torch.Tensor:
    n = workspace_size(B, Hq, Hkv, N, d)
    if n == 0:
        raise ValueError("unsupported attention shape")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _shapes(q, k, v):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
        if t.dim() != 4:
            raise ValueError(f"{n} must be [B, H, N, d]")
    B, Hq, N, d = (int(s) for s in q.shape)
    if tuple(k.shape) != tuple(v.shape) or k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    return B, Hq, int(k.shape[1]), N, d


def _out(q, out_dtype, out):
    dt = torch.float32 if out_dtype in (OUT_F32, torch.float32) else torch.bfloat16
    if out is None:
        out = torch.empty(q.shape, dtype=dt, device=q.device)
    else:
        _need(out, "out", dt)
    return out, (OUT_F32 if dt == torch.float32 else OUT_BF16)


def mxattn_forward(q, k, v, causal: bool = False, scale_mode: int = SCALE_UOS, pnq: bool = True,
                   out_dtype=torch.float32, workspace: torch.Tensor | None = None,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """MXFP4 attention forward (UOS / OCP scaling, PNQ on / off). q [B,Hq,N,d], k/v [B,Hkv,N,d] bf16."""
    B, Hq, Hkv, N, d = _shapes(q, k, v)
    out, od = _out(q, out_dtype, out)
    if workspace is None:
        workspace = alloc_workspace(B, Hq, Hkv, N, d, q.device)
    lib = _lib.load()
    st = lib.mxattn_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, N, d,
                            int(bool(causal)), int(scale_mode), int(pnq), od, workspace.data_ptr(),
                            workspace.numel(), _stream(q.device))
    _lib.check(st, "mxattn_forward")
    return out


def mxattn_forward_host(q, k, v, out, causal: bool = False, scale_mode: int = SCALE_UOS, pnq: bool = True,
                        workspace: torch.Tensor | None = None, device=None) -> torch.Tensor:
    """mxattn_forward on host (CPU, ideally pinned) bf16 tensors q [B,Hq,N,d], k/v [B,Hkv,N,d] and a host
    output tensor out [B,Hq,N,d] (fp32 or bf16): copies and kernels are pipelined over groups of
    KV heads. Asynchronous on the device's current stream; synchronise before reading `out`."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous bf16 host tensor")
    if out.is_cuda or not out.is_contiguous() or out.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out must be a contiguous fp32 or bf16 host tensor")
    B, Hq, N, d = (int(x) for x in q.shape)
    Hkv = int(k.shape[1])
    if tuple(k.shape) != tuple(v.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shapes must be q/out [B,Hq,N,d], k/v [B,Hkv,N,d]")
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    lib = _lib.load()
    if workspace is None:
        n = int(lib.mxattn_forward_host_workspace_size(B, Hq, Hkv, N, d, od))
        if n == 0:
            raise ValueError("unsupported attention shape")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    st = lib.mxattn_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, N, d,
                                 int(bool(causal)), int(scale_mode), int(pnq), od, workspace.data_ptr(),
                                 workspace.numel(), _stream(dev))
    _lib.check(st, "mxattn_forward_host")
    return out


def mxattn_forward_quantized(qc, qs, kc, ks, vtc, vts, N: int, d: int, causal: bool = False,
                             p_scale_mode: int = SCALE_UOS, pnq: bool = True, out_dtype=torch.float32,
                             workspace: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """The attention kernel on operands already in MXFP4 (the layout mxattn_quantize writes):
    qc [B,Hq,N,d/2] / qs [B,Hq,N,d/32], kc / ks [B,Hkv,N,..], vtc [B,Hkv,d,ceil(N/32)*16] /
    vts [B,Hkv,d,ceil(N/32)], all uint8 CUDA tensors. Returns out [B,Hq,N,d]."""
    for t, n in ((qc, "qc"), (qs, "qs"), (kc, "kc"), (ks, "ks"), (vtc, "vtc"), (vts, "vts")):
        _need(t, n, torch.uint8)
    nb = -(-N // 32)
    B, Hq = int(qc.shape[0]), int(qc.shape[1])
    Hkv = int(kc.shape[1])
    shapes = {"qc": (B, Hq, N, d // 2), "qs": (B, Hq, N, d // 32), "kc": (B, Hkv, N, d // 2),
              "ks": (B, Hkv, N, d // 32), "vtc": (B, Hkv, d, nb * 16), "vts": (B, Hkv, d, nb)}
    for t, n in ((qc, "qc"), (qs, "qs"), (kc, "kc"), (ks, "ks"), (vtc, "vtc"), (vts, "vts")):
        if tuple(t.shape) != shapes[n]:
            raise ValueError(f"{n} must have shape {shapes[n]}, got {tuple(t.shape)}")
    dt = torch.float32 if out_dtype in (OUT_F32, torch.float32) else torch.bfloat16
    if out is None:
        out = torch.empty((B, Hq, N, d), dtype=dt, device=qc.device)
    else:
        _need(out, "out", dt)
    od = OUT_F32 if dt == torch.float32 else OUT_BF16
    if workspace is None:
        workspace = alloc_workspace(B, Hq, Hkv, N, d, qc.device)
    st = _lib.load().mxattn_forward_quantized(qc.data_ptr(), qs.data_ptr(), kc.data_ptr(), ks.data_ptr(),
                                              vtc.data_ptr(), vts.data_ptr(), out.data_ptr(), B, Hq, Hkv, N, d,
                                              int(bool(causal)), int(p_scale_mode), int(pnq), od,
                                              workspace.data_ptr(), workspace.numel(), _stream(qc.device))
    _lib.check(st, "mxattn_forward_quantized")
    return out


def gemm_workspace(M: int, N: int, K: int, device) -> torch.Tensor:
    n = int(_lib.load().mxattn_gemm_workspace_size(M, N, K))
    if n == 0:
        raise ValueError("unsupported GEMM shape (needs K % 32 == 0, N % 8 == 0)")
    return torch.empty(n, dtype=torch.uint8, device=device)


def mxattn_gemm(a_codes, a_scales, b_codes, b_scales, K: int, out_dtype=torch.float32,
                workspace: torch.Tensor | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """C [M, N] = dq(A) dq(B)^T for A, B in MXFP4 (codes [R, K/2], scales [R, K/32], uint8 CUDA)."""
    for t, n in ((a_codes, "a_codes"), (a_scales, "a_scales"), (b_codes, "b_codes"), (b_scales, "b_scales")):
        _need(t, n, torch.uint8)
    M, N = int(a_codes.shape[0]), int(b_codes.shape[0])
    for t, n, r, c in ((a_codes, "a_codes", M, K // 2), (a_scales, "a_scales", M, K // 32),
                       (b_codes, "b_codes", N, K // 2), (b_scales, "b_scales", N, K // 32)):
        if tuple(t.shape) != (r, c):
            raise ValueError(f"{n} must have shape {(r, c)}, got {tuple(t.shape)}")
    dt = torch.float32 if out_dtype in (OUT_F32, torch.float32) else torch.bfloat16
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=a_codes.device)
    else:
        _need(out, "out", dt)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, a_codes.device)
    st = _lib.load().mxattn_gemm(a_codes.data_ptr(), a_scales.data_ptr(), b_codes.data_ptr(), b_scales.data_ptr(),
                                 out.data_ptr(), M, N, K, OUT_F32 if dt == torch.float32 else OUT_BF16,
                                 workspace.data_ptr(), workspace.numel(), _stream(a_codes.device))
    _lib.check(st, "mxattn_gemm")
    return out


def mxattn_quantize_nvfp4(x: torch.Tensor):
    """NVFP4-quantize a bf16 CUDA matrix [rows, cols] (blocks of 16, E4M3 scales):
    codes [rows, ceil(cols/16)*8], scales [rows, ceil(cols/16)]."""
    _need(x, "x")
    if x.dim() != 2:
        raise ValueError("x must be [rows, cols]")
    rows, cols = int(x.shape[0]), int(x.shape[1])
    nb = -(-cols // 16)
    codes = torch.empty((rows, nb * 8), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, nb), dtype=torch.uint8, device=x.device)
    st = _lib.load().mxattn_quantize_nvfp4(x.data_ptr(), rows, cols, codes.data_ptr(), scales.data_ptr(),
                                           _stream(x.device))
    _lib.check(st, "mxattn_quantize_nvfp4")
    return codes, scales


def mxattn_gemm_nvfp4(a_codes, a_scales, b_codes, b_scales, K: int, out_dtype=torch.float32,
                      workspace: torch.Tensor | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """C [M, N] = dq(A) dq(B)^T for A, B in NVFP4 (codes [R, K/2], E4M3 scales [R, K/16])."""
    for t, n in ((a_codes, "a_codes"), (a_scales, "a_scales"), (b_codes, "b_codes"), (b_scales, "b_scales")):
        _need(t, n, torch.uint8)
    M, N = int(a_codes.shape[0]), int(b_codes.shape[0])
    for t, n, r, c in ((a_codes, "a_codes", M, K // 2), (a_scales, "a_scales", M, K // 16),
                       (b_codes, "b_codes", N, K // 2), (b_scales, "b_scales", N, K // 16)):
        if tuple(t.shape) != (r, c):
            raise ValueError(f"{n} must have shape {(r, c)}, got {tuple(t.shape)}")
    dt = torch.float32 if out_dtype in (OUT_F32, torch.float32) else torch.bfloat16
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=a_codes.device)
    else:
        _need(out, "out", dt)
    lib = _lib.load()
    if workspace is None:
        n = int(lib.mxattn_gemm_nvfp4_workspace_size(M, N, K))
        if n == 0:
            raise ValueError("unsupported GEMM shape (needs K % 32 == 0, N % 8 == 0)")
        workspace = torch.empty(n, dtype=torch.uint8, device=a_codes.device)
    st = lib.mxattn_gemm_nvfp4(a_codes.data_ptr(), a_scales.data_ptr(), b_codes.data_ptr(), b_scales.data_ptr(),
                               out.data_ptr(), M, N, K, OUT_F32 if dt == torch.float32 else OUT_BF16,
                               workspace.data_ptr(), workspace.numel(), _stream(a_codes.device))
    _lib.check(st, "mxattn_gemm_nvfp4")
    return out


def mxattn_forward_prepare(q, k, v, scale_mode: int, workspace: torch.Tensor) -> None:
    B, Hq, Hkv, N, d = _shapes(q, k, v)
    st = _lib.load().mxattn_forward_prepare(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv, N, d,
                                            int(scale_mode), workspace.data_ptr(), workspace.numel(),
                                            _stream(q.device))
    _lib.check(st, "mxattn_forward_prepare")


def mxattn_forward_attend(out: torch.Tensor, B: int, Hq: int, Hkv: int, N: int, d: int, causal: bool,
                          scale_mode: int, pnq: bool, workspace: torch.Tensor) -> torch.Tensor:
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    st = _lib.load().mxattn_forward_attend(out.data_ptr(), B, Hq, Hkv, N, d, int(bool(causal)),
                                           int(scale_mode), int(pnq), od, workspace.data_ptr(),
                                           workspace.numel(), _stream(out.device))
    _lib.check(st, "mxattn_forward_attend")
    return out


def mxattn_forward_debug(q, k, v, dbg_bh: int, r0: int, r1: int, causal: bool = False,
                         scale_mode: int = SCALE_UOS, pnq: bool = True, out_dtype=torch.float32,
                         workspace: torch.Tensor | None = None):
    """mxattn_forward plus the quantized P~ of rows [r0, r1) of head dbg_bh (= b*Hq + h):
    returns (out, p_codes [r1-r0, Npad/2], p_scales [r1-r0, Npad/32], or Npad/16 for NVFP4)."""
    B, Hq, Hkv, N, d = _shapes(q, k, v)
    out, od = _out(q, out_dtype, None)
    if workspace is None:
        workspace = alloc_workspace(B, Hq, Hkv, N, d, q.device)
    npd = npad(N)
    pc = torch.zeros((r1 - r0, npd // 2), dtype=torch.uint8, device=q.device)
    ps = torch.zeros((r1 - r0, npd // (16 if scale_mode == SCALE_NVFP4 else 32)), dtype=torch.uint8, device=q.device)
    st = _lib.load().mxattn_forward_debug(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq,
                                          Hkv, N, d, int(bool(causal)), int(scale_mode), int(pnq), od,
                                          workspace.data_ptr(), workspace.numel(), _stream(q.device),
                                          dbg_bh, r0, r1, pc.data_ptr(), ps.data_ptr())
    _lib.check(st, "mxattn_forward_debug")
    return out, pc, ps


def mxattn_check_status(workspace: torch.Tensor) -> int:
    """Synchronises the current stream; returns the device status word (0 = ok)."""
    detail = ctypes.c_uint(0)
    st = _lib.load().mxattn_check_status(workspace.data_ptr(), _stream(workspace.device),
                                         ctypes.byref(detail))
    if st not in (0, 5):
        _lib.check(st, "mxattn_check_status")
    return int(detail.value)

"""Benchmark: MXFP4 attention forward (UOS + PNQ) on the video-DiT-shaped workload.

One step = one full pass of the hot path through the library's public C-ABI call
mxattn_forward: quantize Q and K along d and V along keys (one quantizer launch for all three),
then the fused tcgen05 attention kernel, on B=1, H=40, N=32760, d=128, non-causal, seeded synthetic
inputs resident in HBM. Inputs (3 x 335 MB of bf16) exceed the 126 MB L2, so no flush is needed.

Multi-GPU (torchrun): every rank runs its own independent problem of the same shape (weak
scaling, no data-path collective); the step time is the max over ranks.

--impl reference runs the CPU oracle (numpy fp64) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "video_dit"
# also timed, quantizers + attention per step, PNQ: (key, workload, scale mode); the long video DiT
# runs under both MXFP4 scale rules, UOS against the OCP baseline
OTHER_CONFIGS = (("video_dit_long", "video_dit_long", "uos"), ("video_dit_long_ocp", "video_dit_long", "ocp"),
                 ("llm_gqa", "llm_gqa", "uos"))
METRIC = "MXFP4 attention fwd TFLOP/s (video-DiT 1x40x32760x128, UOS+PNQ)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
FP4_PER_BF16 = 4.0          # nominal dense ratio: 9 PFLOP/s fp4 vs 2.25 PFLOP/s bf16
ATTN_SOURCES = ["mxfp4_microscaled_bit_quantize_b200/csrc/attn_fwd_sm100.cu",
                "mxfp4_microscaled_bit_quantize_b200/csrc/sm100_ptx.cuh"]
GEMM_SOURCES = ["mxfp4_microscaled_bit_quantize_b200/csrc/gemm_sm100.cu",
                "mxfp4_microscaled_bit_quantize_b200/csrc/sm100_ptx.cuh"]
QUANT_SOURCES = ["mxfp4_microscaled_bit_quantize_b200/csrc/quantize.cu",
                 "mxfp4_microscaled_bit_quantize_b200/csrc/sm100_ptx.cuh"]


def sources_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def profile_traffic(name: str, src_hash: str):
    """DRAM bytes per launch from the committed ncu summary, if it still matches the source."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_hash") != src_hash:
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms during the timed region. The
    sampler starts first; entering returns once its first sample has arrived (or after 3 s), and
    only the samples that arrive between entry and exit are summarised (all of them if none do)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.samples = []        # (arrival time, line)
        self.lines = []
        self.in_region = False

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.samples.append((time.monotonic(), ln))

    def __enter__(self):
        import shutil
        import threading
        cmd = ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "50"]
        if shutil.which("stdbuf"):
            cmd = ["stdbuf", "-oL"] + cmd      # one line per sample as it is taken
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        if self.proc is not None:
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            deadline = time.monotonic() + 3.0
            while not self.samples and self.proc.poll() is None and time.monotonic() < deadline:
                time.sleep(0.01)
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *a):
        t1 = time.monotonic()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)
        inside = [ln for t, ln in self.samples if self.t0 <= t <= t1]
        self.in_region = bool(inside)
        self.lines = inside or [ln for _, ln in self.samples]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "window": "timed region" if self.in_region else "around the timed region"}


def reduce_max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tflops(flops_per_rank: float, world: int, step_ms: float) -> float:
    """Whole-job throughput: every rank processed its own problem in at most step_ms."""
    return world * flops_per_rank / (step_ms * 1e-3) / 1e12


def oracle_sample(cfg, rows: int, head: int = 0):
    """CPU oracle on a bounded sample: quantize one head's Q/K/V, then attend `rows` query rows of it
    over all keys. Returns (algorithmic FLOP of those rows, seconds)."""
    from mxfp4_microscaled_bit_quantize_b200 import synthetic
    from oracle import attention as oa
    from oracle import mxfp4 as mx

    q = synthetic.head_bf16(cfg, "q", 0, head).double().numpy()
    g = head * cfg.Hkv // cfg.Hq
    k = synthetic.head_bf16(cfg, "k", 0, g).double().numpy()
    v = synthetic.head_bf16(cfg, "v", 0, g).double().numpy()
    t0 = time.perf_counter()
    (qd, kd, vd), _ = oa.dequantized_qkv(q, k, v, mx.SCALE_UOS)
    idx = np.arange(rows)
    oa.attention_rows(qd[:rows], idx, kd, vd, causal=cfg.causal, mode=mx.SCALE_UOS, pnq=True)
    dt = time.perf_counter() - t0
    flops = 4.0 * rows * cfg.N * cfg.d / (2.0 if cfg.causal else 1.0)
    return flops, dt


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_tiny_full():
    """The whole tiny workload (1x2x256x64, UOS + PNQ) through the oracle: (FLOP, seconds)."""
    from mxfp4_microscaled_bit_quantize_b200 import synthetic
    from oracle import attention as oa
    from oracle import mxfp4 as mx
    cfg = synthetic.ATTN_CONFIGS["tiny"]
    q, k, v = (t.double().numpy() for t in synthetic.attn_inputs(cfg))
    t0 = time.perf_counter()
    oa.mxattention(q, k, v, causal=cfg.causal, mode=mx.SCALE_UOS, pnq=True)
    return cfg.flops, time.perf_counter() - t0


def cpu_baseline(cfg, rows: int) -> dict:
    """The CPU oracle as it stands on this host: a bounded row sample of the workload (rows are
    independent under the online softmax, so the sample is exact for those rows), its linear
    extrapolation to the whole workload, the tiny workload in full, and one thread on a smaller
    sample."""
    f, dt = oracle_sample(cfg, rows)
    threads = blas_threads()
    out = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
           "sample": f"{rows} query rows of head 0 (that head's Q/K/V quantized, attention over all "
                     f"{cfg.N} keys), {dt:.1f} s",
           "cpu_model": cpu_model(), "nproc": os.cpu_count(), "blas_threads": threads,
           "extrapolated": {"seconds": cfg.flops / (f / dt),
                            "note": f"the sample's rate scaled to all {cfg.B * cfg.Hq * cfg.N} query rows "
                                    f"of {cfg.name} (extrapolated, not run)"}}
    tf, tdt = oracle_tiny_full()
    out["tiny_full"] = {"seconds": tdt, "value": tf / tdt / 1e12, "unit": "TFLOP/s",
                        "workload": "tiny 1x2x256x64, UOS+PNQ, every row (run in full)"}
    try:   # the same oracle on one thread (BLAS limited to 1), on an eighth of the rows
        from threadpoolctl import threadpool_limits
        rows1 = max(64, rows // 8)
        with threadpool_limits(limits=1):
            f1, dt1 = oracle_sample(cfg, rows1)
        out["single_thread"] = {"value": f1 / dt1 / 1e12, "unit": "TFLOP/s", "rows": rows1, "seconds": dt1}
    except ImportError:
        pass
    return out


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def run_reference(args, rank: int) -> None:
    from mxfp4_microscaled_bit_quantize_b200 import synthetic
    if rank != 0:
        return
    cfg = synthetic.ATTN_CONFIGS[WORKLOAD]
    # query rows per step: 10240 over the timed steps (512 a step at 20 steps, at least 128), so
    # that more steps take fewer rows each; each step also quantizes the head's Q/K/V (a fixed cost)
    rows = args.ref_rows if args.ref_rows else max(128, min(512, 10240 // max(1, args.steps)))
    for _ in range(args.warmup):
        oracle_sample(cfg, rows)
    flops = secs = 0.0
    for _ in range(args.steps):
        f, dt = oracle_sample(cfg, rows)
        flops += f
        secs += dt
    value = flops / secs / 1e12
    sample = (f"{rows} query rows of head 0 (Q/K/V of that head quantized, then online-softmax attention "
              f"over all {cfg.N} keys) per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, **cfg.describe(), "scale_mode": "UOS",
                                            "pnq": True, "sample_rows": rows},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                             "extrapolated": {"seconds": cfg.flops / (flops / secs),
                                              "note": "the sample's rate scaled to the whole workload "
                                                      "(extrapolated, not run)"}},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_gpu(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    from mxfp4_microscaled_bit_quantize_b200 import api, build, synthetic

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = synthetic.ATTN_CONFIGS[args.workload]
    if args.heads:
        cfg = cfg.scaled(Hq=args.heads, Hkv=args.heads)
    B, Hq, Hkv, N, d = cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.d
    if args.mode == "quantizer":
        run_quantizer_only(args, dev)
        return
    if args.mode == "gemm":
        run_gemm_only(args, dev)
        return
    q, k, v = synthetic.attn_inputs(cfg)
    q_h, k_h, v_h = (t.pin_memory() for t in (q, k, v))
    dq, dk, dv = (t.to(dev) for t in (q_h, k_h, v_h))
    ws = api.alloc_workspace(B, Hq, Hkv, N, d, dev)
    out = torch.empty((B, Hq, N, d), dtype=torch.float32, device=dev)
    out_h = torch.empty(out.shape, dtype=torch.float32, pin_memory=True)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    mode = {"uos": api.SCALE_UOS, "ocp": api.SCALE_OCP, "nvfp4": api.SCALE_NVFP4}[args.scale]
    p_rule = {"conventional": api.P_CONVENTIONAL, "pnq": api.P_PNQ, "efq": api.P_EFQ}[args.p_rule]

    def step():
        api.mxattn_forward_prepare(dq, dk, dv, mode, ws)
        api.mxattn_forward_attend(out, B, Hq, Hkv, N, d, cfg.causal, mode, p_rule, ws)

    for _ in range(args.warmup):
        step()
    if api.mxattn_check_status(ws) != 0:
        raise RuntimeError("device pipeline timeout during warm-up")
    barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        barrier()
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            api.mxattn_forward_prepare(dq, dk, dv, mode, ws)
            ev[i][1].record(stream)
            api.mxattn_forward_attend(out, B, Hq, Hkv, N, d, cfg.causal, mode, p_rule, ws)
            ev[i][2].record(stream)
        stop.record(stream)
        barrier()
    if api.mxattn_check_status(ws) != 0:
        raise RuntimeError("device pipeline timeout in the timed region")
    total_ms = start.elapsed_time(stop)
    quant_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    attn_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    if args.mode == "attention":
        print(json.dumps({"mode": "attention", "scale": args.scale, "p_rule": args.p_rule, "config": cfg.describe(),
                          "attn_ms": attn_ms,
                          "quant_ms": quant_ms, "tflops": cfg.flops / (attn_ms * 1e-3) / 1e12}), flush=True)
        return

    # end to end through the public host-buffer call: every step copies its inputs from pinned
    # host memory and its output back, pipelined with the kernels over groups of KV heads
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    d2h = out.numel() * out.element_size()
    e2e_steps = max(1, min(args.steps, 5))
    host_ws = torch.empty(api._lib.load().mxattn_forward_host_workspace_size(B, Hq, Hkv, N, d, api.OUT_F32),
                          dtype=torch.uint8, device=dev)
    api.mxattn_forward_host(q_h, k_h, v_h, out_h, causal=cfg.causal, workspace=host_ws, device=dev)   # warm-up
    barrier()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(e2e_steps):
        api.mxattn_forward_host(q_h, k_h, v_h, out_h, causal=cfg.causal, workspace=host_ws, device=dev)
    e_stop.record(stream)
    barrier()
    if api.mxattn_check_status(host_ws) != 0:
        raise RuntimeError("device pipeline timeout in the host-buffer forward")
    e2e_ms = e_start.elapsed_time(e_stop) / e2e_steps
    del host_ws

    # the floor for any pipeline over this host link: the same bytes copied both ways at once
    # (inputs in, output out, on two streams), with no kernels
    link_in, link_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    staging = torch.empty(h2d, dtype=torch.uint8, device=dev)

    def both_ways():
        link_in.wait_stream(stream)
        link_out.wait_stream(stream)
        with torch.cuda.stream(link_in):
            o = 0
            for t in (q_h, k_h, v_h):
                nb = t.numel() * t.element_size()
                staging[o:o + nb].copy_(t.view(-1).view(torch.uint8), non_blocking=True)
                o += nb
        with torch.cuda.stream(link_out):
            out_h.copy_(out, non_blocking=True)
        stream.wait_stream(link_in)
        stream.wait_stream(link_out)

    both_ways()
    barrier()
    c_start, c_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c_start.record(stream)
    for _ in range(3):
        both_ways()
    c_stop.record(stream)
    barrier()
    copy_ms = c_start.elapsed_time(c_stop) / 3
    del staging

    # the attention kernel on caller-owned MXFP4 operands (mxattn_forward_quantized): scale
    # repacking + the fused kernel, with the codes quantized once outside the timed loop
    fq_ops = (*api.mxattn_quantize(dq, False, api.SCALE_UOS), *api.mxattn_quantize(dk, False, api.SCALE_UOS),
              *api.mxattn_quantize(dv, True, api.SCALE_UOS))
    fq_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        api.mxattn_forward_quantized(*fq_ops, N=N, d=d, causal=cfg.causal, p_scale_mode=api.SCALE_UOS,
                                     pnq=True, workspace=ws, out=out)
    barrier()
    f_start, f_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f_start.record(stream)
    for _ in range(fq_steps):
        api.mxattn_forward_quantized(*fq_ops, N=N, d=d, causal=cfg.causal, p_scale_mode=api.SCALE_UOS,
                                     pnq=True, workspace=ws, out=out)
    f_stop.record(stream)
    barrier()
    fq_ms = f_start.elapsed_time(f_stop) / fq_steps
    del fq_ops

    # the NVFP4 comparison mode of the same kernel on the same workload (attention kernel alone)
    api.mxattn_forward_prepare(dq, dk, dv, api.SCALE_NVFP4, ws)
    for _ in range(2):
        api.mxattn_forward_attend(out, B, Hq, Hkv, N, d, cfg.causal, api.SCALE_NVFP4, True, ws)
    barrier()
    n_start, n_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_start.record(stream)
    for _ in range(fq_steps):
        api.mxattn_forward_attend(out, B, Hq, Hkv, N, d, cfg.causal, api.SCALE_NVFP4, True, ws)
    n_stop.record(stream)
    barrier()
    if api.mxattn_check_status(ws) != 0:
        raise RuntimeError("device pipeline timeout in the NVFP4 attention")
    nv_attn_ms = n_start.elapsed_time(n_stop) / fq_steps

    # the exp-free P~ rule (EFQ-Softmax reading) in the same kernel, UOS scales, attention alone
    api.mxattn_forward_prepare(dq, dk, dv, api.SCALE_UOS, ws)
    for _ in range(2):
        api.mxattn_forward_attend(out, B, Hq, Hkv, N, d, cfg.causal, api.SCALE_UOS, api.P_EFQ, ws)
    barrier()
    n_start.record(stream)
    for _ in range(fq_steps):
        api.mxattn_forward_attend(out, B, Hq, Hkv, N, d, cfg.causal, api.SCALE_UOS, api.P_EFQ, ws)
    n_stop.record(stream)
    barrier()
    if api.mxattn_check_status(ws) != 0:
        raise RuntimeError("device pipeline timeout in the exp-free attention")
    efq_attn_ms = n_start.elapsed_time(n_stop) / fq_steps

    # the other full-size attention workloads: the long video DiT and the causal GQA prefill
    # (quantizers + attention kernel per step, timed per phase as in the main loop)
    other = {}
    for name, wl, scale in OTHER_CONFIGS:
        ocfg = synthetic.ATTN_CONFIGS[wl]
        o_mode = {"uos": api.SCALE_UOS, "ocp": api.SCALE_OCP}[scale]
        oq, ok_, ov = (t.to(dev) for t in synthetic.attn_inputs(ocfg))
        o_ws = api.alloc_workspace(ocfg.B, ocfg.Hq, ocfg.Hkv, ocfg.N, ocfg.d, dev)
        o_out = torch.empty((ocfg.B, ocfg.Hq, ocfg.N, ocfg.d), dtype=torch.float32, device=dev)

        def o_step(e=None):
            if e is not None:
                e[0].record(stream)
            api.mxattn_forward_prepare(oq, ok_, ov, o_mode, o_ws)
            if e is not None:
                e[1].record(stream)
            api.mxattn_forward_attend(o_out, ocfg.B, ocfg.Hq, ocfg.Hkv, ocfg.N, ocfg.d, ocfg.causal, o_mode,
                                      True, o_ws)
            if e is not None:
                e[2].record(stream)

        for _ in range(3):
            o_step()
        barrier()
        o_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(fq_steps)]
        for e in o_ev:
            o_step(e)
        barrier()
        if api.mxattn_check_status(o_ws) != 0:
            raise RuntimeError(f"device pipeline timeout on {name}")
        other[name] = (ocfg, float(np.mean([e[1].elapsed_time(e[2]) for e in o_ev])),
                       float(np.mean([e[0].elapsed_time(e[2]) for e in o_ev])))
        del oq, ok_, ov, o_ws, o_out

    # block-scaled MXFP4 GEMM (W4A4) on its own seeded workload (the one its parity test samples):
    # A [M, K] activations with per-row gains, B [N, K] weights, quantized once outside the timing
    gm, gn, gk = synthetic.GEMM_SHAPE
    ga, gb = (t.to(dev) for t in synthetic.gemm_inputs(gm, gn, gk))
    g_ops = (*api.mxattn_quantize(ga, False, api.SCALE_UOS), *api.mxattn_quantize(gb, False, api.SCALE_UOS))
    nv_ops = (*api.mxattn_quantize_nvfp4(ga), *api.mxattn_quantize_nvfp4(gb))
    del ga, gb
    g_ws = api.gemm_workspace(gm, gn, gk, dev)
    g_out = torch.empty((gm, gn), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        api.mxattn_gemm(*g_ops, gk, out_dtype=torch.bfloat16, workspace=g_ws, out=g_out)
    barrier()
    g_start, g_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g_iters = 10
    g_start.record(stream)
    for _ in range(g_iters):
        api.mxattn_gemm(*g_ops, gk, out_dtype=torch.bfloat16, workspace=g_ws, out=g_out)
    g_stop.record(stream)
    barrier()
    if api.mxattn_check_status(g_ws) != 0:
        raise RuntimeError("device pipeline timeout in the GEMM")
    gemm_ms = g_start.elapsed_time(g_stop) / g_iters
    # the NVFP4 comparison format on the same shape (blocks of 16, E4M3 scales)
    for _ in range(3):
        api.mxattn_gemm_nvfp4(*nv_ops, gk, out_dtype=torch.bfloat16, out=g_out)
    barrier()
    g_start.record(stream)
    for _ in range(g_iters):
        api.mxattn_gemm_nvfp4(*nv_ops, gk, out_dtype=torch.bfloat16, out=g_out)
    g_stop.record(stream)
    barrier()
    gemm_nv_ms = g_start.elapsed_time(g_stop) / g_iters
    del g_ops, nv_ops, g_ws, g_out

    # standalone quantizer on its own workload (65536 x 1024 bf16)
    quant_alone_ms, xq0_numel = time_quantizer_rotating(dev, stream, barrier, iters=50)

    # max over ranks
    other_ms = [x for name, _, _ in OTHER_CONFIGS for x in other[name][1:]]
    (step_ms, attn_ms, quant_ms, e2e_ms, copy_ms, quant_alone_ms, fq_ms, gemm_ms, gemm_nv_ms,
     nv_attn_ms, efq_attn_ms, *other_ms) = reduce_max_over_ranks([total_ms / args.steps, attn_ms, quant_ms, e2e_ms,
                                                     copy_ms, quant_alone_ms, fq_ms, gemm_ms, gemm_nv_ms, nv_attn_ms,
                                                     efq_attn_ms,
                                                     *other_ms], world, dev)
    if rank != 0:
        return

    flops = cfg.flops
    peaks = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    elems = B * Hq * N * d + 2 * B * Hkv * N * d
    # algorithmic bytes of the quantization pass (Q, K, V): bf16 in, packed codes + scales out
    quant_bytes = elems * 2 + elems // 2 + elems // 32
    qa_elems = xq0_numel
    qa_bytes = qa_elems * 2 + qa_elems // 2 + qa_elems // 32
    line = {
        "metric": METRIC,
        "value": job_tflops(flops, world, step_ms),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1xe2m1->f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, **cfg.describe(), "scale_mode": "UOS", "pnq": True,
                   "out_dtype": "f32", "l2": "inputs 3x335 MB bf16 > 126 MB L2, no flush",
                   "parallelism": f"independent problem per GPU x{world}"},
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / fp4_peak, "kernel": "mxattn_fwd_kernel<128>",
                     "peak_note": f"{peaks['source']} bf16 burst x {FP4_PER_BF16:g} (nominal fp4/bf16 ratio)",
                     "traffic": profile_traffic("attn_fwd_video_dit.json", sources_hash(ATTN_SOURCES)),
                     "algorithmic_flops_per_launch": flops, "ms_per_launch": attn_ms},
        "quantizer": {"in_step_gbs": quant_bytes / (quant_ms * 1e-3) / 1e9, "in_step_ms": quant_ms,
                      "standalone_65536x1024_gbs": qa_bytes / (quant_alone_ms * 1e-3) / 1e9,
                      "standalone_ms": quant_alone_ms, "hbm_peak_gbs": peaks["hbm_gbs"],
                      "standalone_buffers": f"{QUANT_SETS} input/output sets rotated, "
                                            f"{QUANT_SETS * qa_bytes / 1e6:.0f} MB in all (> 2 x 126 MB L2)",
                      "standalone_frac": qa_bytes / (quant_alone_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                      "traffic": profile_traffic("quantize_rows_65536x1024.json", sources_hash(QUANT_SOURCES))},
        "exp_free_attention": {"ms": efq_attn_ms, "tflops": flops / (efq_attn_ms * 1e-3) / 1e12,
                               "frac": flops / (efq_attn_ms * 1e-3) / 1e12 / fp4_peak,
                               "note": "pnq = MXATTN_P_EFQ (exp-free P~ codes, EFQ-Softmax reading), UOS, "
                                       "attention kernel alone; a different P~ rule from the headline"},
        "nvfp4_attention": {"ms": nv_attn_ms, "tflops": flops / (nv_attn_ms * 1e-3) / 1e12,
                            "note": "MXATTN_SCALE_NVFP4 (Q, K, V, P~ in NVFP4), attention kernel alone",
                            "traffic": profile_traffic("attn_fwd_video_dit_nvfp4.json", sources_hash(ATTN_SOURCES))},
        "forward_quantized": {"ms": fq_ms, "tflops": flops / (fq_ms * 1e-3) / 1e12,
                              "note": "mxattn_forward_quantized on pre-quantized Q/K/V: scale repack + kernel"},
        "other_configs": {
            name: {"workload": other[name][0].describe(), "scale_mode": scale.upper(), "attn_ms": other_ms[2 * i],
                   "tflops": other[name][0].flops / (other_ms[2 * i] * 1e-3) / 1e12,
                   "frac": other[name][0].flops / (other_ms[2 * i] * 1e-3) / 1e12 / fp4_peak,
                   "step_ms": other_ms[2 * i + 1],
                   "step_tflops": other[name][0].flops / (other_ms[2 * i + 1] * 1e-3) / 1e12,
                   "traffic": profile_traffic(f"attn_fwd_{name}.json", sources_hash(ATTN_SOURCES))}
            for i, (name, _, scale) in enumerate(OTHER_CONFIGS)},
        "gemm": {"workload": f"mxattn_gemm W4A4 {gm}x{gn}x{gk}, bf16 out", "ms": gemm_ms,
                 "tflops": 2.0 * gm * gn * gk / (gemm_ms * 1e-3) / 1e12,
                 "frac": 2.0 * gm * gn * gk / (gemm_ms * 1e-3) / 1e12 / fp4_peak,
                 "nvfp4": {"ms": gemm_nv_ms, "tflops": 2.0 * gm * gn * gk / (gemm_nv_ms * 1e-3) / 1e12,
                           "frac": 2.0 * gm * gn * gk / (gemm_nv_ms * 1e-3) / 1e12 / fp4_peak},
                 "capture_traffic": {"workload": "2048x16384x8192 (M reduced for the ncu capture)",
                                     "dram_bytes": profile_traffic("mxgemm_2048x16384x8192.json",
                                                                   sources_hash(GEMM_SOURCES))}},
        "e2e": {"value": job_tflops(flops, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "api": "mxattn_forward_host (pinned host buffers in and out)",
                "copy_floor": {"ms": copy_ms, "gbs": (h2d + d2h) / (copy_ms * 1e-3) / 1e9,
                               "frac": copy_ms / e2e_ms,
                               "note": "the same H2D and D2H bytes copied concurrently, no kernels"}},
        "gpu_launches": 2 * args.steps,      # per step: the fused Q/K/V quantizer and the attention kernel
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_rows)
    print(json.dumps(line), flush=True)


def run_gemm_only(args, dev):
    """The W4A4 GEMM alone (used for its Nsight Compute capture); --heads scales M down."""
    import torch

    from mxfp4_microscaled_bit_quantize_b200 import api, synthetic
    gm, gn, gk = synthetic.GEMM_SHAPE
    if args.heads:
        gm = 128 * args.heads
    ga, gb = (t.to(dev) for t in synthetic.gemm_inputs(gm, gn, gk))
    ops = (*api.mxattn_quantize(ga, False, api.SCALE_UOS), *api.mxattn_quantize(gb, False, api.SCALE_UOS))
    ws = api.gemm_workspace(gm, gn, gk, dev)
    out = torch.empty((gm, gn), dtype=torch.bfloat16, device=dev)
    for _ in range(args.warmup):
        api.mxattn_gemm(*ops, gk, out_dtype=torch.bfloat16, workspace=ws, out=out)
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        api.mxattn_gemm(*ops, gk, out_dtype=torch.bfloat16, workspace=ws, out=out)
    e.record()
    torch.cuda.synchronize(dev)
    ms = s.elapsed_time(e) / args.steps
    print(json.dumps({"mode": "gemm", "M": gm, "N": gn, "K": gk, "ms": ms,
                      "tflops": 2.0 * gm * gn * gk / (ms * 1e-3) / 1e12}), flush=True)


QUANT_SETS = 4      # input/output buffer sets the standalone quantizer rotates through


def time_quantizer_rotating(dev, stream, barrier, iters: int, warmup: int = 5):
    """Mean ms per call of the standalone quantizer (65536 x 1024, UOS) on QUANT_SETS sets of input
    and output buffers used in turn, so that neither the bf16 input nor the codes and scales written
    by one call are still in L2 when their set comes round again (4 x 170 MB > 2 x 126 MB L2)."""
    import torch

    from mxfp4_microscaled_bit_quantize_b200 import api, synthetic
    x0 = synthetic.quant_input().to(dev)
    xs = [x0] + [x0.clone() for _ in range(QUANT_SETS - 1)]
    outs = [api.mxattn_quantize(x, False, api.SCALE_UOS) for x in xs]
    for i in range(warmup):
        api.mxattn_quantize(xs[i % QUANT_SETS], False, api.SCALE_UOS, out=outs[i % QUANT_SETS])
    barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for i in range(iters):
        api.mxattn_quantize(xs[i % QUANT_SETS], False, api.SCALE_UOS, out=outs[i % QUANT_SETS])
    e.record(stream)
    barrier()
    return s.elapsed_time(e) / iters, x0.numel()


def run_quantizer_only(args, dev):
    """The standalone quantizer workload alone (used for its Nsight Compute capture)."""
    import torch
    stream = torch.cuda.current_stream(dev)
    ms, n = time_quantizer_rotating(dev, stream, lambda: torch.cuda.synchronize(dev), iters=args.steps,
                                    warmup=args.warmup)
    gbs = (n * 2 + n // 2 + n // 32) / (ms * 1e-3) / 1e9
    print(json.dumps({"mode": "quantizer", "ms": ms, "gbs": gbs}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=4096)
    ap.add_argument("--ref-rows", type=int, default=0, help="query rows per reference step (0: 10240 / steps, 128..512)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", choices=["full", "attention", "quantizer", "gemm"], default="full",
                    help="attention / quantizer: time only that part (small cases for profiling)")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling only)")
    ap.add_argument("--workload", choices=[WORKLOAD, *sorted({wl for _, wl, _ in OTHER_CONFIGS})], default=WORKLOAD,
                    help="the attention workload of --mode attention (profiling only)")
    ap.add_argument("--p-rule", choices=["conventional", "pnq", "efq"], default="pnq",
                    help="the P~ rule of --mode attention (profiling only)")
    ap.add_argument("--scale", choices=["uos", "ocp", "nvfp4"], default="uos",
                    help="the scale mode of --mode attention (profiling only)")
    args = ap.parse_args()
    if args.workload != WORKLOAD and (args.mode != "attention" or args.heads):
        ap.error("--workload applies to --mode attention, without --heads")
    if args.p_rule != "pnq" and args.mode != "attention":
        ap.error("--p-rule applies to --mode attention")
    if args.scale != "uos" and args.mode != "attention":
        ap.error("--scale applies to --mode attention")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

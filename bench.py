"""Benchmark of the frozen-base NF4 + double-quant LoRA linear layer on B200.

One step = forward (Y, U) + input gradient (dX, G) + adapter gradients (dA, dB)
of the 7B attention projection: W0 4096x4096 NF4 (blocks of 64, 8-bit double
quant in groups of 256), 2048 bf16 tokens, LoRA r=8, alpha=16.  Metric:
algorithmic TFLOP/s = (4MNK + 2Mr(K+N) + 4Mr(N+K)) / step time (the frozen
base gets no weight gradient).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun as independent replicas (weak scaling, no data-path
collective); time is the max over ranks.  `--impl reference` times the CPU
oracle (float64 numpy) on the host cores on a bounded token sample.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused NF4-dequant LoRA linear TFLOP/s (fwd+bwd)"

# dram__bytes_read.sum + dram__bytes_write.sum per launch of each GEMM kernel on this
# workload, from one ncu capture each (profiles/); set to None when the kernel changes
KERNEL_TRAFFIC = {"dx": 25_606_400, "fwd": 25_710_592}
UNIT = "TFLOP/s"


def algo_flops(M, N, K, r):
    return 4 * M * N * K + 2 * M * r * (K + N) + 4 * M * r * (N + K)


def fwd_flops(M, N, K, r):
    return 2 * M * N * K + 2 * M * r * (K + N)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(backend):
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, local, ws


def dist_max(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Polls NVML (SM clock, max clock, throttle reasons) in a thread while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.stop_flag = threading.Event()
        self.thread = None
        self.err = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[0].isdigit() else self.gpu
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception as e:  # pragma: no cover
                self.err = str(e)
                return
            time.sleep(0.0005)

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"nvml unavailable: {self.err}"]}
        self.stop_flag.set()
        self.thread.join(timeout=5)
        nv = self.nv
        names = {"hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
                 "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                 "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                 "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4)}
        reasons = sorted({n for _, rs in self.samples for n, bit in names.items() if rs & bit})
        sm = [s for s, _ in self.samples]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle leg

def oracle_sample_step(state):
    """One oracle pass (fwd + dX + dA/dB in float64) over the sampled tokens."""
    from oracle import nf4_oracle as O
    Wd, X, A, B, dY, s = state
    Y, u = O.lora_linear_fwd(Wd, X, A, B, s)
    dX, g = O.lora_linear_bwd_dx(Wd, dY, A, B, s)
    dA, dB = O.lora_grad_ab(X, dY, u, g, s)
    return Y, dX, dA, dB


def oracle_state(case, m_sample):
    from oracle import nf4_oracle as O
    W = case.weight()
    ref = O.quantize_nf4_dq(W.numpy())
    Wd = O.dequant(ref["codes"], ref["scales"], ref["scales2"]).reshape(case.N, case.K).astype(np.float64)
    X = case.x()[:m_sample].float().numpy().astype(np.float64)
    dY = case.dy()[:m_sample].float().numpy().astype(np.float64)
    A = case.lora_a().float().numpy().astype(np.float64)
    B = case.lora_b().float().numpy().astype(np.float64)
    return Wd, X, A, B, dY, case.scaling


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline(case, m_sample=256, budget_s=10.0):
    st = oracle_state(case, m_sample)
    oracle_sample_step(st)                       # warm
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_sample_step(st)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    flops = algo_flops(m_sample, case.N, case.K, case.r) * n
    return {"value": flops / el / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{m_sample} of {case.M} tokens of {case.name}, fwd+dX+dA/dB in float64 numpy, "
                      f"{n} passes in {el:.1f} s"}


def run_reference(args, case):
    rank, local, ws = dist_setup("gloo")
    if rank != 0:
        return
    m_sample = 256
    st = oracle_state(case, m_sample)
    for _ in range(args.warmup):
        oracle_sample_step(st)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(st)
    el = time.perf_counter() - t0
    flops = algo_flops(m_sample, case.N, case.K, case.r) * args.steps
    value = flops / el / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(case, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{m_sample} of {case.M} tokens per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(case, n):
    return {"workload": f"{case.name}: W0 {case.N}x{case.K} NF4 block 64 + DQ 256, X {case.M}x{case.K} bf16, "
                        f"LoRA r={case.r} alpha={int(case.alpha)}, fwd + dX + dA/dB",
            "M": case.M, "N": case.N, "K": case.K, "r": case.r, "alpha": case.alpha,
            "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{n}"}


# ----------------------------------------------------------------------------- decode sweep

DECODE_LAYERS = 32
DECODE_MS = (1, 4, 16)
DECODE_R, DECODE_ALPHA = 8, 16.0


def decode_sweep(dev, steps, warmup, layers=DECODE_LAYERS, with_gate=False, ms=DECODE_MS):
    """Forward over the 32-layer 7B weight set (Q, K, V, O 4096x4096, up 11008x4096, down
    4096x11008; LoRA r=8 on Q/K/V/O) at M = 1, 4, 16 tokens, one library call per matrix,
    captured once in a CUDA graph per M.  Calls carry no data dependency on each other.
    with_gate adds a gate projection (11008x4096) per layer: 6.48e9 weights, the count the
    decode configuration quotes.  Returns algorithmic GB/s = (packed weights + X + Y + LoRA
    A/B bytes) / sweep time."""
    import torch
    import bit_quantized_base_nf4_b200 as q
    from bit_quantized_base_nf4_b200 import synthetic as syn
    shapes = syn.decode_layer_shapes(with_gate)
    r, s = DECODE_R, DECODE_ALPHA / DECODE_R
    mats = []
    for layer in range(layers):
        for i, (name, N, K, lora) in enumerate(shapes):
            w = q.NF4Weight.empty(N, K, device=dev)
            W = syn.decode_weight(layer, i, N, K, dev)
            q.qlora_quantize_nf4_dq(W, w)
            del W
            A = B = None
            if lora:
                A = syn.normal_bf16((r, K), 1.0 / K, 4500 + 16 * layer + i).to(dev)
                B = syn.normal_bf16((N, r), 0.01, 4700 + 16 * layer + i).to(dev)
            mats.append((w, N, K, A, B))
    q.qlora_sync_status()
    widths = sorted({K for _, _, K, _, _ in mats} | {N for _, N, _, _, _ in mats})
    out = {}
    for M in ms:
        X = {K: syn.decode_inputs(M, K, 4900 + K).to(dev) for K in widths}
        Y = {N: torch.empty(M, N, dtype=torch.bfloat16, device=dev) for N in widths}
        ws = torch.empty(max(q.qlora_workspace_bytes(M, N, K, r) for _, N, K, _, _ in mats), dtype=torch.uint8,
                         device=dev)
        nbytes = 0
        for w, N, K, A, B in mats:
            nbytes += q.qlora_packed_bytes(N * K) + 2 * M * K + 2 * M * N
            if A is not None:
                nbytes += 2 * r * K + 2 * N * r

        def sweep():
            for w, N, K, A, B in mats:
                rr = r if A is not None else 0
                q.qlora_lora_linear_fwd(w, X[K], A, B, rr, s if rr else 0.0, Y[N], None, ws)

        sweep()                                          # attributes and maps settle outside capture
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            sweep()
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            g.replay()
        b.record()
        torch.cuda.synchronize(dev)
        q.qlora_sync_status()
        ms = a.elapsed_time(b) / steps
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[f"M={M}"] = {"GB/s": gbs, "ms_per_sweep": ms, "bytes_per_sweep": nbytes,
                         "frac_of_hbm": gbs / peaks()["hbm_gbs"]}
        del g
    gate = " gate 11008x4096," if with_gate else ""
    out["workload"] = (f"7B decode sweep: {layers} layers x {{Q,K,V,O 4096x4096,{gate} up 11008x4096, down 4096x11008}} = "
                       f"{sum(N * K for _, N, K, _, _ in mats):.3e} NF4 weights, LoRA r=8 on Q/K/V/O; "
                       "one forward call per matrix, no inter-call dependency, CUDA graph per M; "
                       "working set >> L2 (no flush)")
    out["hbm_peak_gbs"] = peaks()["hbm_gbs"]
    return out


# ----------------------------------------------------------------------------- quantize pass

def quantize_pass(dev, steps, warmup):
    """One-shot encode (NF4 codes + double-quantized scales) of the 70B FFN up projection,
    28672 x 8192 fp32 ~N(0, 0.015) drawn on the device; GB/s = (4 + packed bytes per weight)
    x weights / time.  The 0.94 GB input is far larger than L2."""
    import torch
    import bit_quantized_base_nf4_b200 as q
    N, K = 28672, 8192
    g = torch.Generator(device=dev)
    g.manual_seed(5100)
    W = torch.randn(N, K, generator=g, device=dev, dtype=torch.float32) * 0.015
    w = q.NF4Weight.empty(N, K, device=dev)
    for _ in range(warmup):
        q.qlora_quantize_nf4_dq(W, w)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        q.qlora_quantize_nf4_dq(W, w)
    b.record()
    torch.cuda.synchronize(dev)
    q.qlora_sync_status()
    ms = a.elapsed_time(b) / steps
    nbytes = 4 * N * K + q.qlora_packed_bytes(N * K)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "70B FFN up 28672x8192 fp32 -> NF4 + DQ", "ms": ms, "bytes": nbytes, "GB/s": gbs,
            "frac_of_hbm": gbs / peaks()["hbm_gbs"]}


# ----------------------------------------------------------------------------- merge pass

def merge_pass(dev, steps, warmup):
    """LoRA merge + requantize (dequant to bf16, add s B A in float64, round to bf16,
    NF4 + DQ encode) of the 7B attention projection (4096 x 4096, r = 8) and the 70B FFN
    up projection (28672 x 8192, r = 64).  GB/s on the algorithmic bytes: packed weight
    in and out plus A and B; "moved" adds the float32 merged base the encode reads
    back (written once, read once)."""
    import torch
    import bit_quantized_base_nf4_b200 as q
    from bit_quantized_base_nf4_b200 import synthetic as syn
    out = {}
    for name, N, K, r, std in (("7B attn 4096x4096 r=8", 4096, 4096, 8, 0.02),
                               ("70B FFN up 28672x8192 r=64", 28672, 8192, 64, 0.015)):
        g = torch.Generator(device=dev)
        g.manual_seed(5200 + r)
        W = torch.randn(N, K, generator=g, device=dev, dtype=torch.float32) * std
        w = q.NF4Weight.empty(N, K, device=dev)
        q.qlora_quantize_nf4_dq(W, w)
        scratch = W   # the merged base overwrites the fp32 input, no longer needed
        A = syn.normal_bf16((r, K), 1.0 / K, 5300 + r).to(dev)
        B = syn.normal_bf16((N, r), 0.01, 5400 + r).to(dev)
        w_out = q.NF4Weight.empty(N, K, device=dev)
        for _ in range(warmup):
            q.qlora_lora_merge_requant(w, A, B, r, 16.0 / r, scratch, w_out)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            q.qlora_lora_merge_requant(w, A, B, r, 16.0 / r, scratch, w_out)
        b.record()
        torch.cuda.synchronize(dev)
        q.qlora_sync_status()
        ms = a.elapsed_time(b) / steps
        algo = 2 * q.qlora_packed_bytes(N * K) + 2 * r * (N + K)
        moved = algo + 8 * N * K
        out[name] = {"ms": ms, "GB/s": algo / (ms * 1e-3) / 1e9, "moved_GB/s": moved / (ms * 1e-3) / 1e9,
                     "moved_frac_of_hbm": moved / (ms * 1e-3) / 1e9 / peaks()["hbm_gbs"]}
        del W, scratch, w, w_out, A, B
        torch.cuda.empty_cache()
    return out


def _side_leg(fn):
    """Runs a measurement beside the headline step; a failure is reported in its key
    instead of losing the whole JSON line."""
    try:
        return fn()
    except Exception as e:  # noqa: BLE001 - any failure of a side measurement is reported, not raised
        return {"error": f"{type(e).__name__}: {e}"[:300]}


# ----------------------------------------------------------------------------- CUDA leg

def run_ours(args, case):
    import torch
    rank, local, ws = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import bit_quantized_base_nf4_b200 as q

    M, N, K, r, s = case.M, case.N, case.K, case.r, case.scaling
    w = q.NF4Weight.empty(N, K, device=dev)
    q.qlora_quantize_nf4_dq(case.weight().to(dev), w)
    X, A, B, dY = (t.to(dev) for t in (case.x(), case.lora_a(), case.lora_b(), case.dy()))
    wsb = torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    U = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    G = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = torch.empty(N, r, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 8   # fwd: rank product, finalize, fused GEMM; dX: same three; dA and dB products

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        q.qlora_lora_linear_fwd(w, X, A, B, r, s, Y, U, wsb, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        q.qlora_lora_linear_bwd_dx(w, dY, A, B, r, s, dX, G, wsb, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        q.qlora_lora_grad_AB(X, dY, U, G, r, s, dA, dB, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    q.qlora_sync_status(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    dist_barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)                         # evict the previous step's operands from L2 (untimed)
        step(evs[i])
    torch.cuda.synchronize(dev)
    dist_barrier()
    clk = clocks.stop()
    q.qlora_sync_status(stream)
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dx_ms = [e[1].elapsed_time(e[2]) for e in evs]
    grad_ms = [e[2].elapsed_time(e[3]) for e in evs]
    total_ms = dist_max(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    value = ws * algo_flops(M, N, K, r) / (ms_per_step * 1e-3) / 1e12

    # end to end through the same C ABI with host buffers: H2D of the step's inputs from
    # pinned memory, the three calls, D2H of the adapter gradients.
    hX, hdY = X.cpu().pin_memory(), dY.cpu().pin_memory()
    hdA, hdB = torch.empty_like(dA, device="cpu").pin_memory(), torch.empty_like(dB, device="cpu").pin_memory()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for i in range(args.warmup + args.steps):
        if i >= args.warmup:
            flush.fill_(i & 0xFF)
            e2e_ev[i - args.warmup][0].record(stream)
        X.copy_(hX, non_blocking=True)
        dY.copy_(hdY, non_blocking=True)
        step()
        hdA.copy_(dA, non_blocking=True)
        hdB.copy_(dB, non_blocking=True)
        if i >= args.warmup:
            e2e_ev[i - args.warmup][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = dist_max(sum(a.elapsed_time(b) for a, b in e2e_ev), dev) / args.steps
    h2d = (hX.numel() + hdY.numel()) * 2
    d2h = (hdA.numel() + hdB.numel()) * 4

    # the two GEMM kernels alone: with r = 0 each call is exactly one launch of the fused
    # kernel (dX: CTA-pair transposed-dequant GEMM; forward: CTA-pair dequant GEMM)
    kern = {"dx": [], "fwd": []}
    for i in range(args.warmup + args.steps):
        flush.fill_(i & 0xFF)
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        q.qlora_lora_linear_bwd_dx(w, dY, None, None, 0, 0.0, dX, None, wsb, stream=stream)
        b.record(stream)
        flush.fill_((i + 1) & 0xFF)
        b2 = torch.cuda.Event(enable_timing=True)
        b2.record(stream)
        q.qlora_lora_linear_fwd(w, X, None, None, 0, 0.0, Y, None, wsb, stream=stream)
        c.record(stream)
        if i >= args.warmup:
            kern["dx"].append((a, b))
            kern["fwd"].append((b2, c))
    torch.cuda.synchronize(dev)
    q.qlora_sync_status(stream)
    dx_k_ms = statistics.mean(x.elapsed_time(y) for x, y in kern["dx"])
    fwd_k_ms = statistics.mean(x.elapsed_time(y) for x, y in kern["fwd"])
    base_flops = 2 * M * N * K

    pk = peaks()

    def roofline(ms, name, traffic):
        achieved = base_flops / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"], "traffic": traffic, "kernel": name,
                "launch_ms": ms, "flops_per_launch": base_flops,
                "peak_source": f"{pk['source']} bf16 burst (MEASURED_PEAKS.json)",
                "frac_of_sustained": (achieved / pk["bf16_tflops_sustained"])
                if pk.get("bf16_tflops_sustained") else None}

    # dram bytes per launch from ncu captures of this workload (see profiles/), None once stale
    roof = roofline(dx_k_ms, "fused_bwd_pair_kernel (dX, dominant kernel of the step)", KERNEL_TRAFFIC.get("dx"))
    roof_fwd = roofline(fwd_k_ms, "fused_fwd_pair_kernel (forward base GEMM)", KERNEL_TRAFFIC.get("fwd"))

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(case, ws),
                "roofline": roof, "roofline_fwd": roof_fwd,
                "phases_ms": {"fwd": statistics.mean(fwd_ms), "bwd_dx": statistics.mean(dx_ms),
                              "grad_ab": statistics.mean(grad_ms)},
                "e2e": {"value": ws * algo_flops(M, N, K, r) / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": launches_per_step * args.steps, "clocks": clk}
        if not args.no_decode:
            k = max(5, args.steps // 2)
            line["quantize"] = _side_leg(lambda: quantize_pass(dev, k, args.warmup))
            line["decode"] = _side_leg(lambda: decode_sweep(dev, k, args.warmup, args.decode_layers))
            # the configuration's "~6.5e9 weights" counts a gate projection per layer as well
            line["decode_with_gate"] = _side_leg(lambda: decode_sweep(dev, k, args.warmup, args.decode_layers,
                                                                      with_gate=True, ms=(1,)))
            line["merge"] = _side_leg(lambda: merge_pass(dev, 5, args.warmup))
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = _side_leg(lambda: cpu_baseline(case))
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the quantize, decode-sweep and merge GB/s measurements")
    ap.add_argument("--decode-only", action="store_true", help="run only the decode sweep (prints its JSON)")
    ap.add_argument("--decode-layers", type=int, default=DECODE_LAYERS)
    ap.add_argument("--merge-only", action="store_true", help="run only the merge + requantize pass (prints its JSON)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from bit_quantized_base_nf4_b200 import synthetic as syn
    case = syn.attn7b_case()
    if args.impl == "reference":
        run_reference(args, case)
    elif args.merge_only:
        import torch
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps({"merge": merge_pass(dev, args.steps, args.warmup)}), flush=True)
    elif args.decode_only:
        import torch
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps({"decode": decode_sweep(dev, args.steps, args.warmup, args.decode_layers)}), flush=True)
    else:
        run_ours(args, case)


if __name__ == "__main__":
    main()

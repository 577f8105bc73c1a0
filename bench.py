"""Benchmark of the frozen-base NF4 + double-quant LoRA linear layer on B200.

One step = forward (Y, U) + input gradient (dX, G) + adapter gradients (dA, dB) of
every matrix of the 70B-shape layer: attention 8192x8192 and FFN 28672x8192 /
8192x28672, W0 NF4 (blocks of 64, 8-bit double quant in groups of 256), 4096 bf16
tokens, LoRA r=64, alpha=128 on every projection.  Metric: algorithmic TFLOP/s =
sum over the matrices of (4MNK + 2Mr(K+N) + 4Mr(N+K)) / step time (the frozen base
gets no weight gradient).  The 7B attention (2048 tokens, r=8) and 7B FFN pair
(4096 tokens, r=64, 0.1 % outliers) are measured the same way beside it, with the
decode sweep, the one-shot quantize, dequant and merge passes.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun as independent replicas (weak scaling, no data-path
collective); time is the max over ranks.  `--impl reference` times the CPU
oracle (float64 numpy) on the host cores on a bounded sample of the same layer.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused NF4-dequant LoRA linear TFLOP/s (fwd+bwd)"
UNIT = "TFLOP/s"
CSRC = os.path.join(ROOT, "bit_quantized_base_nf4_b200", "csrc")

# dram__bytes_read.sum + dram__bytes_write.sum of each GEMM kernel, summed over its three
# launches of one step of the 70B layer, from one ncu capture each (profiles/), with a
# hash of the kernel sources that capture ran; a source change makes the figure stale
# and the bench then reports null
KERNEL_TRAFFIC = {
    # attention 162.1 + 46.2 MB, FFN up 852.0 + 57.9 MB, FFN down 847.1 + 211.6 MB
    "dx": {"bytes": 2176886272, "src_sha": "8d831963ce15634a"},
    # attention 111.4 + 51.2 MB, FFN up 1952.1 + 222.3 MB, FFN down 1168.5 + 58.7 MB
    "fwd": {"bytes": 3564198400, "src_sha": "08e3f1cc905141cf"},
}


def kernel_src_hash(kind: str) -> str:
    # the kernel, its helpers, and the host code that picks its tiles and launch order
    common = ["ptx.cuh", "scale_src.cuh", "qlora_nf4.cu"]
    files = {"dx": ["fused_bwd_pair.cuh"] + common, "fwd": ["fused_fwd_pair.cuh"] + common}[kind]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def kernel_traffic(kind: str):
    t = KERNEL_TRAFFIC.get(kind)
    if not t or t.get("src_sha") != kernel_src_hash(kind):
        return None
    return t["bytes"]


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

ORACLE_TOKENS, ORACLE_ROWS = 256, 1024


def oracle_sample_step(states):
    """One oracle pass (fwd + dX + dA/dB in float64) over the sampled sub-layers."""
    from oracle import nf4_oracle as O
    for Wd, X, A, B, dY, s in states:
        Y, u = O.lora_linear_fwd(Wd, X, A, B, s)
        dX, g = O.lora_linear_bwd_dx(Wd, dY, A, B, s)
        O.lora_grad_ab(X, dY, u, g, s)


def oracle_states(cases, host):
    """The oracle's inputs for the bounded sample: for each matrix of the layer, its first
    ORACLE_ROWS output rows (whole double-quant groups of the row-major weight), encoded and
    dequantized by the oracle, and the first ORACLE_TOKENS tokens."""
    from oracle import nf4_oracle as O
    states, flops = [], 0
    for c in cases:
        W, X, A, B, dY = host[c.name]
        rows = min(ORACLE_ROWS, c.N)
        ref = O.quantize_nf4_dq(W[:rows].numpy())
        Wd = O.dequant(ref["codes"], ref["scales"], ref["scales2"]).reshape(rows, c.K).astype(np.float64)
        f64 = lambda t: t.float().numpy().astype(np.float64)
        states.append((Wd, f64(X[:ORACLE_TOKENS]), f64(A), f64(B[:rows]), f64(dY[:ORACLE_TOKENS, :rows]), c.scaling))
        flops += algo_flops(ORACLE_TOKENS, rows, c.K, c.r)
    return states, flops


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def oracle_sample_desc(cases):
    return (f"first {ORACLE_ROWS} output rows of each of the {len(cases)} matrices x first {ORACLE_TOKENS} of "
            f"{cases[0].M} tokens, fwd+dX+dA/dB in float64 numpy")


def cpu_baseline(cases, host, budget_s=10.0):
    states, flops_per_pass = oracle_states(cases, host)
    oracle_sample_step(states)                       # warm
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_sample_step(states)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": flops_per_pass * n / el / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{oracle_sample_desc(cases)}; {n} passes in {el:.1f} s"}


def host_tensors(cases):
    """The seeded synthetic inputs of each matrix, drawn on the host (the tests' bytes)."""
    return {c.name: (c.weight(), c.x(), c.lora_a(), c.lora_b(), c.dy()) for c in cases}


def run_reference(args, cases):
    rank, local, ws = dist_setup("gloo")
    if rank != 0:
        return
    host = host_tensors(cases)
    states, flops_per_pass = oracle_states(cases, host)
    for _ in range(args.warmup):
        oracle_sample_step(states)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(states)
    el = time.perf_counter() - t0
    value = flops_per_pass * args.steps / el / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cases, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": oracle_sample_desc(cases) + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(cases, n):
    mats = ", ".join(f"{c.N}x{c.K}" for c in cases)
    c0 = cases[0]
    return {"workload": f"70B-shape layer: W0 {{{mats}}} NF4 block 64 + DQ 256, X {c0.M} tokens bf16, "
                        f"LoRA r={c0.r} alpha={int(c0.alpha)} on every matrix, fwd + dX + dA/dB per matrix",
            "M": c0.M, "matrices": [[c.N, c.K] for c in cases], "r": c0.r, "alpha": c0.alpha,
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


def dequant_pass(dev, steps, warmup):
    """One-shot dequant (the "dequantize the whole matrix" route) of the 70B FFN up
    projection, 28672 x 8192, to bf16; GB/s = (packed bytes + 2 bytes per weight) / time."""
    import torch
    import bit_quantized_base_nf4_b200 as q
    N, K = 28672, 8192
    g = torch.Generator(device=dev)
    g.manual_seed(5150)
    W = torch.randn(N, K, generator=g, device=dev, dtype=torch.float32) * 0.015
    w = q.NF4Weight.empty(N, K, device=dev)
    q.qlora_quantize_nf4_dq(W, w)
    del W
    out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    for _ in range(warmup):
        q.qlora_dequant(w, out)
    a, b = _ev(), _ev()
    a.record()
    for _ in range(steps):
        q.qlora_dequant(w, out)
    b.record()
    torch.cuda.synchronize(dev)
    q.qlora_sync_status()
    ms = a.elapsed_time(b) / steps
    nbytes = q.qlora_packed_bytes(N * K) + 2 * N * K
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "70B FFN up 28672x8192 NF4 + DQ -> bf16", "ms": ms, "bytes": nbytes, "GB/s": gbs,
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

LAUNCHES_PER_MATRIX = 8   # fwd: rank product, finalize, fused GEMM; dX: the same three; dA and dB products


class MatrixRun:
    """Device buffers of one matrix of a layer and its three library calls (NF4 base, or
    the Q8_0 route with q8=True)."""

    def __init__(self, case, host, dev, q8=False):
        import torch
        import bit_quantized_base_nf4_b200 as q
        self.q, self.c, self.q8 = q, case, q8
        W, X, A, B, dY = host[case.name]
        M, N, K, r = case.M, case.N, case.K, case.r
        if q8:
            self.w = q.Q80Weight.empty(N, K, device=dev)
            q.qlora_quantize_q8_0(W.to(dev), self.w)
            self._fwd, self._dx = q.qlora_q8_0_lora_linear_fwd, q.qlora_q8_0_lora_linear_bwd_dx
        else:
            self.w = q.NF4Weight.empty(N, K, device=dev)
            q.qlora_quantize_nf4_dq(W.to(dev), self.w)
            self._fwd, self._dx = q.qlora_lora_linear_fwd, q.qlora_lora_linear_bwd_dx
        self.X, self.A, self.B, self.dY = (t.to(dev) for t in (X, A, B, dY))
        self.ws = torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
        bf = torch.bfloat16
        self.Y = torch.empty(M, N, dtype=bf, device=dev)
        self.U = torch.empty(M, r, dtype=bf, device=dev)
        self.dX = torch.empty(M, K, dtype=bf, device=dev)
        self.G = torch.empty(M, r, dtype=bf, device=dev)
        self.dA = torch.empty(r, K, dtype=torch.float32, device=dev)
        self.dB = torch.empty(N, r, dtype=torch.float32, device=dev)
        self.flops = algo_flops(M, N, K, r)
        self.base_flops = 2 * M * N * K

    def fwd(self, st, r=None):
        c = self.c
        if r == 0:
            self._fwd(self.w, self.X, None, None, 0, 0.0, self.Y, None, self.ws, stream=st)
        else:
            self._fwd(self.w, self.X, self.A, self.B, c.r, c.scaling, self.Y, self.U, self.ws, stream=st)

    def dx(self, st, r=None):
        c = self.c
        if r == 0:
            self._dx(self.w, self.dY, None, None, 0, 0.0, self.dX, None, self.ws, stream=st)
        else:
            self._dx(self.w, self.dY, self.A, self.B, c.r, c.scaling, self.dX, self.G, self.ws, stream=st)

    def grad(self, st):
        c = self.c
        self.q.qlora_lora_grad_AB(self.X, self.dY, self.U, self.G, c.r, c.scaling, self.dA, self.dB, stream=st)


def _ev():
    import torch
    return torch.cuda.Event(enable_timing=True)


def measure_layer(runs, dev, st, steps, warmup, flush, clocks=None, e2e=True, kernels=True):
    """Times `steps` steps (every matrix: fwd, dX, dA/dB) with L2 flushed between steps, then
    the same step end to end from pinned host memory, then each fused GEMM kernel alone
    (r = 0 calls: exactly one launch of the kernel).  Returns a dict of measurements."""
    import torch
    q = runs[0].q
    for _ in range(warmup):
        for m in runs:
            m.fwd(st); m.dx(st); m.grad(st)
    q.qlora_sync_status(st)
    flops = sum(m.flops for m in runs)
    evs = [[_ev() for _ in range(1 + 3 * len(runs))] for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize(dev)
    if clocks is not None:
        clocks.start()
    for i in range(steps):
        flush.fill_(i & 0xFF)                         # evict the previous step's operands from L2 (untimed)
        e = evs[i]
        e[0].record(st)
        for j, m in enumerate(runs):
            m.fwd(st); e[1 + 3 * j].record(st)
            m.dx(st); e[2 + 3 * j].record(st)
            m.grad(st); e[3 + 3 * j].record(st)
    torch.cuda.synchronize(dev)
    dist_barrier()
    clk = clocks.stop() if clocks is not None else None
    q.qlora_sync_status(st)
    step_ms = [e[0].elapsed_time(e[-1]) for e in evs]
    ph = {"fwd": 0.0, "bwd_dx": 0.0, "grad_ab": 0.0}
    per_matrix = {}
    for j, m in enumerate(runs):
        f = statistics.mean(e[3 * j].elapsed_time(e[1 + 3 * j]) for e in evs)
        d = statistics.mean(e[1 + 3 * j].elapsed_time(e[2 + 3 * j]) for e in evs)
        g = statistics.mean(e[2 + 3 * j].elapsed_time(e[3 + 3 * j]) for e in evs)
        ph["fwd"] += f; ph["bwd_dx"] += d; ph["grad_ab"] += g
        per_matrix[m.c.name] = {"fwd_ms": f, "bwd_dx_ms": d, "grad_ab_ms": g,
                                "TFLOP/s": m.flops / ((f + d + g) * 1e-3) / 1e12}
    total_ms = dist_max(sum(step_ms), dev)
    out = {"ms_per_step": total_ms / steps, "flops_per_step": flops,
           "TFLOP/s": flops / (total_ms / steps * 1e-3) / 1e12, "phases_ms": ph, "per_matrix": per_matrix,
           "clocks": clk}

    if e2e:
        # End to end through the same calls with host buffers: every step copies each
        # matrix's X and dY from pinned host memory and reads its dA and dB back.  The
        # copies run on two side streams (host to device, device to host) and overlap the
        # compute of the other matrices, as a training loop that prefetches its next inputs
        # would; events order every use of a buffer.  The timed region spans all the steps,
        # from the first copy to the last read-back, with the L2 flush of every step in it.
        hosts = [(m.X.cpu().pin_memory(), m.dY.cpu().pin_memory(),
                  torch.empty_like(m.dA, device="cpu").pin_memory(),
                  torch.empty_like(m.dB, device="cpu").pin_memory()) for m in runs]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in runs]   # this step's X and dY of matrix j are on the device
        used = [torch.cuda.Event() for _ in runs]     # matrix j's calls are done (inputs free, dA/dB written)
        read = [torch.cuda.Event() for _ in runs]     # matrix j's dA and dB are back on the host

        def e2e_step(i):
            flush.fill_(i & 0xFF)
            for j, (m, (hX, hdY, hdA, hdB)) in enumerate(zip(runs, hosts)):
                h2d.wait_event(used[j])               # the previous step's calls no longer read X, dY
                with torch.cuda.stream(h2d):
                    m.X.copy_(hX, non_blocking=True)
                    m.dY.copy_(hdY, non_blocking=True)
                copied[j].record(h2d)
                st.wait_event(copied[j])
                st.wait_event(read[j])                # the previous dA, dB are read before being rewritten
                m.fwd(st); m.dx(st); m.grad(st)
                used[j].record(st)
                d2h.wait_event(used[j])
                with torch.cuda.stream(d2h):
                    hdA.copy_(m.dA, non_blocking=True)
                    hdB.copy_(m.dB, non_blocking=True)
                read[j].record(d2h)

        for i in range(warmup):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        t0, t1 = _ev(), _ev()
        t0.record(st)
        h2d.wait_event(t0)
        d2h.wait_event(t0)
        for i in range(steps):
            e2e_step(warmup + i)
        for ev in read:
            st.wait_event(ev)
        t1.record(st)
        torch.cuda.synchronize(dev)
        q.qlora_sync_status(st)
        e2e_ms = dist_max(t0.elapsed_time(t1), dev) / steps
        out["e2e"] = {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                      "h2d_bytes_per_step": sum((h[0].numel() + h[1].numel()) * 2 for h in hosts),
                      "d2h_bytes_per_step": sum((h[2].numel() + h[3].numel()) * 4 for h in hosts),
                      "ms_per_step": e2e_ms,
                      "copies": "host-to-device and device-to-host on side streams, overlapping compute"}
        del hosts

    if kernels:
        # each fused GEMM kernel alone: an r = 0 call is exactly one launch of it
        kern = {"dx": [], "fwd": []}
        for i in range(warmup + steps):
            for m in runs:
                for kind, call in (("dx", m.dx), ("fwd", m.fwd)):
                    flush.fill_(i & 0xFF)
                    a, b = _ev(), _ev()
                    a.record(st)
                    call(st, r=0)
                    b.record(st)
                    if i >= warmup:
                        kern[kind].append((m, a, b))
        torch.cuda.synchronize(dev)
        q.qlora_sync_status(st)
        pk = peaks()
        roof = {}
        for kind, name in (("dx", "fused_bwd_pair_kernel (dX GEMM)"), ("fwd", "fused_fwd_pair_kernel (forward GEMM)")):
            ms = {}
            for m, a, b in kern[kind]:
                ms.setdefault(m.c.name, []).append(a.elapsed_time(b))
            launch_ms = sum(statistics.mean(v) for v in ms.values())
            fl = sum(m.base_flops for m in runs)
            achieved = fl / (launch_ms * 1e-3) / 1e12
            roof[kind] = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": achieved / pk["bf16_tflops"], "traffic": kernel_traffic(kind), "kernel": name,
                          "unit_of_work": f"its {len(runs)} launch(es) of one step, one per matrix (2MNK each)",
                          "launch_ms": launch_ms, "flops": fl,
                          "per_matrix_ms": {k: statistics.mean(v) for k, v in ms.items()},
                          "peak_source": f"{pk['source']} bf16 burst (MEASURED_PEAKS.json)",
                          "frac_of_sustained": (achieved / pk["bf16_tflops_sustained"])
                          if pk.get("bf16_tflops_sustained") else None}
        out["roofline"] = roof
    return out


def sustained_layer(runs, dev, st, seconds, gpu_index):
    """Back-to-back steps (no flush) for about `seconds`, with the SM clock sampled: the
    layer's throughput under the power cap, beside the burst figure."""
    import torch
    q = runs[0].q
    t_one = None
    clocks = ClockSampler(gpu_index)
    torch.cuda.synchronize(dev)
    a, b = _ev(), _ev()
    a.record(st)
    for m in runs:
        m.fwd(st); m.dx(st); m.grad(st)
    b.record(st)
    torch.cuda.synchronize(dev)
    t_one = a.elapsed_time(b)
    n = max(10, int(seconds * 1e3 / max(t_one, 1e-3)))
    clocks.start()
    a.record(st)
    for _ in range(n):
        for m in runs:
            m.fwd(st); m.dx(st); m.grad(st)
    b.record(st)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    q.qlora_sync_status(st)
    ms = a.elapsed_time(b) / n
    flops = sum(m.flops for m in runs)
    return {"TFLOP/s": flops / (ms * 1e-3) / 1e12, "ms_per_step": ms, "steps": n, "seconds": ms * n / 1e3,
            "clocks": clk}


def run_ours(args, cases):
    import torch
    rank, local, ws = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from bit_quantized_base_nf4_b200 import synthetic as syn
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    host = host_tensors(cases)
    runs = [MatrixRun(c, host, dev) for c in cases]
    clocks = ClockSampler(local)
    head = measure_layer(runs, dev, stream, args.steps, args.warmup, flush, clocks=clocks)
    value = ws * head["TFLOP/s"]
    sustained = _side_leg(lambda: sustained_layer(runs, dev, stream, args.sustained_s, local)) \
        if args.sustained_s > 0 else None
    del runs
    torch.cuda.empty_cache()

    # the other layer configurations, measured the same way (no e2e leg)
    others = {}
    if not args.headline_only:
        for label, cs in (("7b_attention_m2048_r8", [syn.attn7b_case()]), ("7b_ffn_pair_m4096_r64", syn.ffn7b_cases())):
            def leg(cs=cs):
                h = host_tensors(cs)
                rr = [MatrixRun(c, h, dev) for c in cs]
                res = measure_layer(rr, dev, stream, args.steps, args.warmup, flush, e2e=False)
                res["workload"] = config_dict(cs, ws)["workload"].replace("70B-shape layer", label)
                return res
            others[label] = _side_leg(leg)
            torch.cuda.empty_cache()

        # the Q8_0 route (int8 codes, fp16 scale per 32 weights) on the 70B attention matrix
        def q8_leg():
            cs = cases[:1]
            h = {c.name: host[c.name] for c in cs}
            rr = [MatrixRun(c, h, dev, q8=True) for c in cs]
            res = measure_layer(rr, dev, stream, args.steps, args.warmup, flush, e2e=False)
            res["workload"] = (f"Q8_0 route: W0 {cs[0].N}x{cs[0].K} int8 + fp16 scale per 32, X {cs[0].M} tokens bf16, "
                               f"LoRA r={cs[0].r}, fwd + dX + dA/dB")
            return res
        others["q8_0_70b_attention_m4096_r64"] = _side_leg(q8_leg)
        torch.cuda.empty_cache()

    if rank == 0:
        roof = head["roofline"]
        dominant = max(("dx", "fwd"), key=lambda k: roof[k]["launch_ms"])
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config_dict(cases, ws),
                "roofline": dict(roof[dominant], dominant_of_step=True),
                "roofline_other": roof["fwd" if dominant == "dx" else "dx"],
                "phases_ms": head["phases_ms"], "per_matrix": head["per_matrix"],
                "e2e": head["e2e"], "gpu_launches": LAUNCHES_PER_MATRIX * len(cases) * args.steps,
                "clocks": head["clocks"]}
        if sustained is not None:
            line["sustained"] = sustained
        if others:
            line["configs"] = others
        if not args.no_decode:
            k = max(5, args.steps // 2)
            line["quantize"] = _side_leg(lambda: quantize_pass(dev, k, args.warmup))
            line["dequant"] = _side_leg(lambda: dequant_pass(dev, k, args.warmup))
            line["decode"] = _side_leg(lambda: decode_sweep(dev, k, args.warmup, args.decode_layers))
            # the configuration's "~6.5e9 weights" counts a gate projection per layer as well
            line["decode_with_gate"] = _side_leg(lambda: decode_sweep(dev, k, args.warmup, args.decode_layers,
                                                                      with_gate=True, ms=(1,)))
            line["merge"] = _side_leg(lambda: merge_pass(dev, 5, args.warmup))
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = _side_leg(lambda: cpu_baseline(cases, host))
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


NCU_CASES = {
    # name: (list of (N, K), M, r, call run per matrix and step)
    "decode_m1": ([(4096, 4096)], 1, 8, "fwd"),
    "decode_m16": ([(4096, 4096)], 16, 8, "fwd"),
    # the 7B down projection at M = 1 (11 stages of 1024 k per unit: the steady state)
    "decode_m1_down": ([(4096, 11008)], 1, 0, "fwd"),
    "dx_70b_attn": ([(8192, 8192)], 4096, 0, "dx"),
    "fwd_70b_attn": ([(8192, 8192)], 4096, 0, "fwd"),
    # the forward with the adapter: the rank-r product U = X A^T, then the GEMM
    "fwd_r64_70b_attn": ([(8192, 8192)], 4096, 64, "fwd"),
    # the one-shot encode (fp32 -> NF4 + double quant) of the 8192 x 8192 matrix (268 MB in)
    "encode_70b_attn": ([(8192, 8192)], 0, 0, "enc"),
    # LoRA merge + requantize of the 8192 x 8192 matrix, r = 64 (merge kernel, then the encode)
    "merge_70b_attn": ([(8192, 8192)], 0, 64, "merge"),
    # the three matrices of the 70B layer, the GEMM kernel alone (r = 0) once each per step
    "dx_70b_layer": ([(8192, 8192), (28672, 8192), (8192, 28672)], 4096, 0, "dx"),
    "fwd_70b_layer": ([(8192, 8192), (28672, 8192), (8192, 28672)], 4096, 0, "fwd"),
}


def ncu_case(name, steps, warmup):
    """A small, fixed launch sequence for profiler captures: per step, one call of one kind
    (the forward, dX, the one-shot encode or the merge) on each listed matrix, nothing else
    after the setup."""
    import torch
    import bit_quantized_base_nf4_b200 as q
    from bit_quantized_base_nf4_b200 import synthetic as syn
    shapes, M, r, kind = NCU_CASES[name]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if kind == "merge":
        g = torch.Generator(device=dev)
        g.manual_seed(5200 + r)
        merges = []
        for N, K in shapes:
            W = torch.randn(N, K, generator=g, device=dev, dtype=torch.float32) * 0.015
            w = q.NF4Weight.empty(N, K, device=dev)
            q.qlora_quantize_nf4_dq(W, w)
            A = syn.normal_bf16((r, K), 1.0 / K, 5300 + r).to(dev)
            B = syn.normal_bf16((N, r), 0.01, 5400 + r).to(dev)
            merges.append((w, A, B, W, q.NF4Weight.empty(N, K, device=dev)))
        for _ in range(warmup + steps):
            for w, A, B, scratch, w_out in merges:
                q.qlora_lora_merge_requant(w, A, B, r, 16.0 / r, scratch, w_out)
        torch.cuda.synchronize(dev)
        q.qlora_sync_status()
        print(json.dumps({"ncu_case": name, "calls": (warmup + steps) * len(merges)}), flush=True)
        return
    if kind == "enc":
        g = torch.Generator(device=dev)
        g.manual_seed(5100)
        encs = []
        for N, K in shapes:
            W = torch.randn(N, K, generator=g, device=dev, dtype=torch.float32) * 0.015
            encs.append((W, q.NF4Weight.empty(N, K, device=dev)))
        for _ in range(warmup + steps):
            for W, w in encs:
                q.qlora_quantize_nf4_dq(W, w)
        torch.cuda.synchronize(dev)
        q.qlora_sync_status()
        print(json.dumps({"ncu_case": name, "calls": (warmup + steps) * len(encs)}), flush=True)
        return
    runs = []
    for i, (N, K) in enumerate(shapes):
        c = syn.LayerCase(f"{name}-{i}", M=M, N=N, K=K, r=r, alpha=2.0 * r, w_std=0.015, seed=7000 + 10 * i)
        runs.append(MatrixRun(c, host_tensors([c]), dev))
    st = torch.cuda.current_stream(dev)
    for _ in range(warmup + steps):
        for m in runs:
            (m.fwd if kind == "fwd" else m.dx)(st)
    torch.cuda.synchronize(dev)
    q.qlora_sync_status()
    print(json.dumps({"ncu_case": name, "calls": (warmup + steps) * len(runs)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the quantize, dequant, decode-sweep and merge GB/s measurements")
    ap.add_argument("--headline-only", action="store_true", help="skip the 7B layer configurations")
    ap.add_argument("--sustained-s", type=float, default=3.0,
                    help="seconds of back-to-back steps for the sustained figure (0 skips it)")
    ap.add_argument("--decode-only", action="store_true", help="run only the decode sweep (prints its JSON)")
    ap.add_argument("--decode-layers", type=int, default=DECODE_LAYERS)
    ap.add_argument("--merge-only", action="store_true", help="run only the merge + requantize pass (prints its JSON)")
    ap.add_argument("--ncu-case", choices=sorted(NCU_CASES), help="run one small fixed case for profiler captures")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from bit_quantized_base_nf4_b200 import synthetic as syn
    cases = syn.l70b_cases()
    if args.ncu_case:
        ncu_case(args.ncu_case, args.steps, args.warmup)
    elif args.impl == "reference":
        run_reference(args, cases)
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
        run_ours(args, cases)


if __name__ == "__main__":
    main()

"""Benchmark of the weight-only block-quantized matmul hot path on B200.

Default workload (one JSON line on rank 0): the Q4_0 decode GEMV of the
12288 x 4096 MLP up-projection (the micro-benchmark shape of the MLX issue
"quantized_matmul takes 14-41% longer than dequantize + bf16 matmul at prefill
sizes (> 512 tokens)", Repro) at M = 1, 8 and 32 tokens.  One step is one
quant_matmul call per token count, each on its own copy of the packed weights;
12 rotating copies (340 MB > 126 MB of L2) make every launch read its weights
from HBM.  value = packed weight + scale bytes read per step / step time.

Other workloads (--workload): affine4_prefill, affine8_sweep (TFLOP/s of the
fused kernel and of the unfused dequantize + bf16 GEMM pair), llama1b_stack
(tokens/s of the 112 projection matmuls of a 16-layer Llama-3.2-1B shape).

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no exchange step), timing is the max over ranks, value is the sum.
--impl reference times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# dram__bytes_read.sum + dram__bytes_write.sum of one launch, from one ncu capture of the
# current build of each kernel (`ncu --set full`, decode bench command); None for a kernel
# changed since its counters were taken.
NCU_TRAFFIC = {"gemv_kernel<Q4_0, M=1>": 28332800, "gemv_kernel<Q4_0, M=8>": 28389888,
               "gemv_kernel<Q4_0, M=32>": 28590592, "gemv_q8_kernel<M=1>": 28324608}
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- helpers (host only)
def dist_env():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"]))}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float across the process group (identity when world == 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    return units_per_rank * world / max_seconds


def rotation(n_copies: int, per_step: int, step: int, j: int) -> int:
    """Weight copy used by launch j of step `step` (every copy is read once per cycle)."""
    return (step * per_step + j) % n_copies


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 100):
        self.gpu_index, self.interval_ms = gpu_index, interval_ms
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.interval_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(self.interval_ms / 1000.0 * 1.5)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(1, 5) if r[2][i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- GPU workloads
def _fmt_args(fmt):
    return {"q4_0": (32, 4), "affine4": (64, 4), "affine8": (64, 8)}[fmt]


def make_weights(fmt, N, K, seed, dev):
    """Packed weights quantized on the GPU by the library from seeded synthetic fp32 W."""
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs
    g = inputs.generator(seed, "cpu")
    if fmt == "q4_0":
        w = inputs.weights_fp32(N, K, g).to(dev)
        wq, s = bq.q4_0_quantize(w)
        b = None
    else:
        gs, bits = _fmt_args(fmt)
        w = inputs.weights_bf16_valued(N, K, g).to(dev)
        wq, s, b = bq.affine_quantize(w, gs, bits)
    del w
    torch.cuda.synchronize()
    return wq, s, b


class GraphTimer:
    """Captures a callable into a CUDA graph; replays are timed with CUDA events on the current stream."""

    def __init__(self, fn):
        import torch
        self.stream = torch.cuda.Stream()
        self.stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.stream):
            fn()                      # first call outside capture (one-time host set-up)
        torch.cuda.current_stream().wait_stream(self.stream)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            fn()
        torch.cuda.synchronize()

    def replay(self):
        self.graph.replay()


def time_graphs(graphs, n_replays, world, device):
    """Replay graphs[i % len] n_replays times between a barrier + synchronize on both sides."""
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(n_replays):
        graphs[i % len(graphs)].replay()
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return start.elapsed_time(end) / 1000.0


def kernel_seconds(fn_list, reps):
    """Average device time of one call of each fn (back-to-back in one graph, CUDA events)."""
    import torch

    def body():
        for _ in range(reps):
            for f in fn_list:
                f()
    gt = GraphTimer(body)
    gt.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    gt.replay()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / 1000.0 / (reps * len(fn_list))


def run_decode(args, world, device, peaks):
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs, workloads

    wl = workloads.Q4_0_DECODE
    N, K, Ms = wl.N, wl.K, wl.Ms
    gs, bits = _fmt_args(wl.fmt)
    wq0, s0, _ = make_weights(wl.fmt, N, K, wl.seed, device)
    n_copies = 12
    copies = [(wq0, s0)] + [(wq0.clone(), s0.clone()) for _ in range(n_copies - 1)]
    g = inputs.generator(wl.seed + 1)
    xs = {M: inputs.activations_bf16(M, K, g).to(device) for M in Ms}
    ys = {M: torch.empty(M, N, dtype=torch.bfloat16, device=device) for M in Ms}
    wbytes = workloads.packed_weight_bytes(wl.fmt, N, K, gs)
    assert n_copies * wbytes > 2 * L2_BYTES

    def step_fn(phase):
        def f():
            for j, M in enumerate(Ms):
                wq, s = copies[rotation(n_copies, len(Ms), phase, j)]
                bq.quant_matmul(xs[M], wq, s, None, gs, bits, out=ys[M])
        return f

    n_phase = n_copies // math.gcd(n_copies, len(Ms))
    graphs = [GraphTimer(step_fn(p)) for p in range(n_phase)]
    for i in range(args.warmup):
        graphs[i % n_phase].replay()
    torch.cuda.synchronize()
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        secs = time_graphs(graphs, args.steps, world, device)
    secs_max = max_over_ranks(secs, world, device)
    units = args.steps * len(Ms) * wbytes                   # bytes of packed weights read by this rank
    value = aggregate(units, world, secs_max) / 1e9

    # per-kernel device time (each M is its own GEMV instantiation), same launch configuration
    per_m = {}
    for M in Ms:
        fns = [(lambda wq=wq, s=s, M=M: bq.quant_matmul(xs[M], wq, s, None, gs, bits, out=ys[M]))
               for (wq, s) in copies]
        t = kernel_seconds(fns, 4)
        per_m[str(M)] = {"us": round(t * 1e6, 3), "gbs": round(wbytes / t / 1e9, 1),
                         "frac_hbm": round(wbytes / t / 1e9 / peaks["hbm_gbs"], 4),
                         "tflops": round(2.0 * M * N * K / t / 1e12, 3)}
    # the quantized-activation path (opt-in, approximate): activation quantization
    # plus the Q4_0 x int8 GEMV, same weights, rotation and graph timing
    q8 = {}
    for M in Ms[:1]:                                  # a one-token path
        fns = [(lambda wq=wq, s=s, M=M: bq.quant_matmul_q8(*bq.q8_1_quantize(xs[M]), wq, s, out=ys[M]))
               for (wq, s) in copies]
        t_all = kernel_seconds(fns, 4)
        xq, dxq, qsq = bq.q8_1_quantize(xs[M])
        fns_g = [(lambda wq=wq, s=s, M=M: bq.quant_matmul_q8(xq, dxq, qsq, wq, s, out=ys[M])) for (wq, s) in copies]
        t_g = kernel_seconds(fns_g, 4)
        q8[str(M)] = {"us": round(t_all * 1e6, 3), "gbs": round(wbytes / t_all / 1e9, 1),
                      "gemv_us": round(t_g * 1e6, 3), "gemv_gbs": round(wbytes / t_g / 1e9, 1),
                      "gemv_frac_hbm": round(wbytes / t_g / 1e9 / peaks["hbm_gbs"], 4),
                      "gemv_traffic": NCU_TRAFFIC.get(f"gemv_q8_kernel<M={M}>")}
    dom = max(Ms, key=lambda M: per_m[str(M)]["us"])
    roof = {"bound": "hbm", "kernel": f"gemv_kernel<Q4_0, M={dom}>",
            "achieved": per_m[str(dom)]["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(per_m[str(dom)]["gbs"] / peaks["hbm_gbs"], 4),
            "traffic": NCU_TRAFFIC.get(f"gemv_kernel<Q4_0, M={dom}>"), "algorithmic_bytes_per_launch": wbytes}

    # end to end through the public API with host buffers: inputs H2D from pinned memory, y D2H
    e2e = None
    if not args.no_e2e:
        h_wq = wq0.cpu().pin_memory()
        h_s = s0.cpu().pin_memory()
        h_x = {M: xs[M].cpu().pin_memory() for M in Ms}
        h_y = {M: torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for M in Ms}
        d_wq, d_s = torch.empty_like(wq0), torch.empty_like(s0)
        d_x = {M: torch.empty_like(xs[M]) for M in Ms}
        e2e_steps = max(3, min(args.steps, 20))

        def e2e_step():
            # the step's inputs: the weight matrix (once) and each M's activations
            d_wq.copy_(h_wq, non_blocking=True)
            d_s.copy_(h_s, non_blocking=True)
            for M in Ms:
                d_x[M].copy_(h_x[M], non_blocking=True)
                bq.quant_matmul(d_x[M], d_wq, d_s, None, gs, bits, out=ys[M])
                h_y[M].copy_(ys[M], non_blocking=True)
        e2e_step()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(e2e_steps):
            e2e_step()
        t1.record()
        torch.cuda.synchronize()
        es = max_over_ranks(t0.elapsed_time(t1) / 1000.0, world, device)
        h2d = h_wq.numel() * h_wq.element_size() + h_s.numel() * 2 + sum(h_x[M].numel() * 2 for M in Ms)
        d2h = sum(M * N * 2 for M in Ms)
        e2e = {"value": round(aggregate(e2e_steps * len(Ms) * wbytes, world, es) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": e2e_steps}

    launches = args.steps * len(Ms)
    return {
        "value": round(value, 2), "unit": "GB/s", "ms_per_step": secs_max / args.steps * 1e3,
        "higher_is_better": True, "dtype": "q4_0 weights, bf16 activations, fp32 accumulate",
        "config": {"workload": wl.name, "fmt": "q4_0", "N": N, "K": K, "M": list(Ms),
                   "l2": f"{n_copies} rotating weight copies ({n_copies * wbytes / 1e6:.0f} MB > 126 MB L2)",
                   "bytes_per_step": len(Ms) * wbytes, "path": "quant_matmul auto -> gemv"},
        "per_m": per_m, "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clk.summary(),
        "secondary": {"q8_activation_path": dict(q8, note="opt-in approximate path: q8_1_quantize + "
                                                          "quant_matmul_q8; not the headline value")},
    }


def run_prefill(args, world, device, peaks, fmt, Ms):
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs, workloads

    N, K = 12288, 4096
    gs, bits = _fmt_args(fmt)
    wq, s, b = make_weights(fmt, N, K, 0, device)
    g = inputs.generator(1)
    ws = torch.empty(N * K, dtype=torch.bfloat16, device=device)
    res = {}
    total_flops, total_s = 0.0, 0.0
    for M in Ms:
        x = inputs.activations_bf16(M, K, g).to(device)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        flops = 2.0 * M * N * K
        reps = max(10, min(50, int(2e13 / flops)))
        fused_path = "tc_fused" if M > 32 else "gemv"
        t_fused = kernel_seconds([lambda: bq.quant_matmul_ex(x, wq, s, b, gs, bits, True, fused_path, out=y)], reps)
        t_auto = kernel_seconds([lambda: bq.quant_matmul_ex(x, wq, s, b, gs, bits, True, "auto", workspace=ws,
                                                           out=y)], reps)
        t_pair = kernel_seconds([lambda: bq.quant_matmul_ex(x, wq, s, b, gs, bits, True, "dequant_gemm",
                                                           workspace=ws, out=y)], reps)
        wb = ws.view(N, K)
        if fmt == "q4_0":
            bq.q4_0_dequantize(wq, s, out=wb)
        else:
            bq.affine_dequantize(wq, s, b, gs, bits, out=wb)
        t_gemm = kernel_seconds([lambda: bq.bf16_matmul(x, wb, out=y)], reps)
        t_cublas = kernel_seconds([lambda: torch.matmul(x, wb.t(), out=y)], reps)
        total_flops += flops
        total_s += t_fused
        res[str(M)] = {"fused_tflops": round(flops / t_fused / 1e12, 1),
                       "fused_frac": round(flops / t_fused / 1e12 / peaks["bf16_tflops"], 4),
                       "pair_tflops": round(flops / t_pair / 1e12, 1),
                       "bf16_gemm_tflops": round(flops / t_gemm / 1e12, 1),
                       "cublas_bf16_tflops": round(flops / t_cublas / 1e12, 1),
                       "fused_us": round(t_fused * 1e6, 2), "pair_us": round(t_pair * 1e6, 2),
                       "auto_path": bq.quant_matmul_select_path(M, N, K, gs, bits),
                       "auto_tflops": round(flops / t_auto / 1e12, 1)}
        del x, y
    return res, total_flops / total_s / 1e12


def run_widths(args, world, device, peaks):
    """Affine 2/3/6-bit weights and transpose=False (W stored [K][N], grouped along N), which run
    as the unfused pair: the dequantize (bytes moved, GB/s) and quant_matmul's auto path per M."""
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs

    N, K, G = 12288, 4096, 64
    ws = torch.empty(N * K, dtype=torch.bfloat16, device=device)
    res = {}
    for name, bits, transpose in (("affine2", 2, True), ("affine3", 3, True), ("affine6", 6, True),
                                  ("affine4_transpose0", 4, False), ("affine3_transpose0", 3, False)):
        g = inputs.generator(0)
        w = inputs.weights_bf16_valued(N, K, g) if transpose else inputs.weights_bf16_valued(K, N, g)
        wq, s, b = bq.affine_quantize(w.to(device), G, bits)
        del w
        packed = wq.numel() * 4 + 2 * s.numel() * 2
        entry = {"bits": bits, "transpose": transpose, "packed_bytes": packed}
        if transpose:
            t_dq = kernel_seconds([lambda: bq.affine_dequantize(wq, s, b, G, bits, out=ws.view(N, K))], 20)
            entry["dequant_us"] = round(t_dq * 1e6, 2)
            entry["dequant_gbs"] = round((packed + N * K * 2) / t_dq / 1e9, 1)
        xg = inputs.generator(1)
        for M in (1, 512, 2048):
            x = inputs.activations_bf16(M, K, xg).to(device)
            y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            flops = 2.0 * M * N * K
            t = kernel_seconds([lambda: bq.quant_matmul_ex(x, wq, s, b, G, bits, transpose, "auto", workspace=ws,
                                                           out=y)], max(10, min(50, int(2e13 / flops))))
            entry[str(M)] = {"us": round(t * 1e6, 2), "tflops": round(flops / t / 1e12, 1),
                             "frac_tensor": round(flops / t / 1e12 / peaks["bf16_tflops"], 4)}
            del x, y
        res[name] = entry
    return res


def run_stack(args, world, device, peaks):
    """Llama-3.2-1B-shaped projection stack, Q4_0: the 112 matmuls of 16 layers (q, k, v, o,
    gate, up, down), each layer with its own weights (547 MB packed > L2), at M = 512 and
    M = 1.  q/k/v and gate/up, which share an activation, go through quant_matmul_multi
    (one launch each at decode sizes).  One CUDA graph holds the whole stack;
    tokens/s = M / stack time."""
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs, workloads
    wl = workloads.LLAMA_1B_STACK
    g = inputs.generator(wl.seed, str(device.type) if device.type == "cuda" else "cpu")
    mats = []
    for _layer in range(wl.layers):
        for (N, K) in wl.shapes:
            w = inputs.weights_fp32(N, K, g, device=device)
            wq, d = bq.q4_0_quantize(w)
            mats.append((N, K, wq, d))
            del w
    torch.cuda.synchronize()
    packed = sum(workloads.packed_weight_bytes("q4_0", N, K, 32) for N, K, _, _ in mats)
    params = sum(N * K for N, K, _, _ in mats)
    gx = inputs.generator(wl.seed + 1)
    per_m, launches = {}, 0
    for M in wl.Ms:
        xs = {K: inputs.activations_bf16(M, K, gx).to(device) for K in sorted({K for _, K, _, _ in mats})}
        ys = [torch.empty(M, N, dtype=torch.bfloat16, device=device) for N, _, _, _ in mats]

        # per layer: q, k, v share one activation (one quant_matmul_multi call), then
        # o; gate and up share one (one call), then down
        per_layer = len(wl.shapes)
        calls = []
        for l0 in range(0, len(mats), per_layer):
            lm, ly = mats[l0:l0 + per_layer], ys[l0:l0 + per_layer]
            calls.append(("multi", lm[0:3], ly[0:3]))
            calls.append(("one", lm[3:4], ly[3:4]))
            calls.append(("multi", lm[4:6], ly[4:6]))
            calls.append(("one", lm[6:7], ly[6:7]))

        def stack():
            for kind, ms, yl in calls:
                K = ms[0][1]
                if kind == "multi":
                    bq.quant_matmul_multi(xs[K], [(wq, d, None) for _, _, wq, d in ms], 32, 4, outs=yl)
                else:
                    bq.quant_matmul(xs[K], ms[0][2], ms[0][3], None, 32, 4, out=yl[0])
        gt = GraphTimer(stack)
        for _ in range(max(3, args.warmup // 50)):
            gt.replay()
        reps = max(3, min(200, args.steps // 100))
        sec = max_over_ranks(time_graphs([gt], reps, world, device) / reps, world, device)
        paths = sorted({bq.quant_matmul_select_path(M, N, K, 32, 4) for N, K, _, _ in mats})
        launches += reps * (len(calls) if M <= 32 else len(mats))
        per_m[str(M)] = {"us_per_stack": round(sec * 1e6, 2), "tokens_per_s": round(aggregate(M, world, sec), 1),
                         "tflops": round(2.0 * M * params / sec / 1e12, 2),
                         "frac_tensor": round(2.0 * M * params / sec / 1e12 / peaks["bf16_tflops"], 4),
                         "gbs": round(packed / sec / 1e9, 1),
                         "frac_hbm": round(packed / sec / 1e9 / peaks["hbm_gbs"], 4),
                         "paths": [{v: k for k, v in bq.PATHS.items()}.get(p_, p_) for p_ in paths]}
        del gt, xs, ys
    return per_m, packed, params, launches


# ----------------------------------------------------------------------------- CPU oracle (baseline / reference arm)
def oracle_decode_sample(budget_s: float):
    """Time the CPU oracle on the decode workload: per step, dequantize W and take the
    float64 matmul for M = 1, 8, 32.  Runs whole steps until ~budget_s has passed."""
    import numpy as np
    import oracle
    from bit_quantized_gemm_quant_b200 import inputs, workloads
    wl = workloads.Q4_0_DECODE
    g = inputs.generator(wl.seed)
    w = inputs.weights_fp32(wl.N, wl.K, g).numpy()
    wq, d = oracle.q4_0_quantize(w)
    xs = {M: inputs.activations_bf16(M, wl.K, g).view(dtype=__import__("torch").int16).numpy().view(np.uint16)
          for M in wl.Ms}
    wbytes = workloads.packed_weight_bytes("q4_0", wl.N, wl.K, 32)
    steps, threads = 0, 1
    t0 = time.perf_counter()
    while True:
        for M in wl.Ms:
            wb = oracle.q4_0_dequantize(wq, d)
            _, _, threads = oracle.matmul_ref(xs[M], wb, nthreads=os.cpu_count())
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": round(steps * len(wl.Ms) * wbytes / el / 1e9, 5), "unit": "GB/s", "cores": int(threads),
            "kind": "oracle", "sample": f"{steps} full decode step(s) (dequantize + float64 matmul at M=1,8,32) "
                                        f"in {el:.1f} s"}, el / steps


# ----------------------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["q4_0_decode", "affine4_prefill", "affine8_sweep", "q4_0_prefill",
                                           "llama1b_stack", "affine_widths"],
                    default="q4_0_decode")
    ap.add_argument("--ms", type=str, default=None, help="comma-separated M list for a prefill workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the secondary prefill measurement")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    rank, local_rank, world = dist_env()
    peaks, peak_src = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return 0
        cb, sec_per_step = oracle_decode_sample(args.cpu_budget)
        line = {"metric": "prefill TFLOP/s (% bf16 TC peak); M=1 GEMV GB/s (% HBM peak)", "impl": "reference",
                "value": cb["value"], "unit": cb["unit"], "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": sec_per_step * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": "q4_0_decode_n12288_k4096", "M": [1, 8, 32]}, "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": cb["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                "gpu_launches": 0}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import bit_quantized_gemm_quant_b200 as bq
    bq.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    if args.workload == "q4_0_decode":
        r = run_decode(args, world, device, peaks)
        if not args.no_prefill:
            pre, _ = run_prefill(args, world, device, peaks, "affine4", (2048,))
            r.setdefault("secondary", {})["prefill_affine4_n12288_k4096_m2048"] = pre["2048"]
    elif args.workload == "llama1b_stack":
        with ClockSampler(local_rank) as clk:
            per_m, packed, params, launches = run_stack(args, world, device, peaks)
        r = {"value": per_m["512"]["tokens_per_s"], "unit": "tokens/s", "ms_per_step": per_m["512"]["us_per_stack"] / 1e3,
             "dtype": "q4_0 weights, bf16 activations, fp32 accumulate",
             "config": {"workload": "llama3.2_1b_q4_0_projection_stack_16_layers", "M": [512, 1],
                        "params": params, "packed_bytes": packed,
                        "l2": f"{packed / 1e6:.0f} MB of distinct packed weights per stack (> 126 MB L2)"},
             "per_m": per_m,
             "roofline": {"bound": "tensor", "kernel": "whole stack at M=512", "achieved": per_m["512"]["tflops"],
                          "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": per_m["512"]["frac_tensor"],
                          "traffic": None},
             "clocks": clk.summary(), "gpu_launches": launches, "e2e": None}
    elif args.workload == "affine_widths":
        with ClockSampler(local_rank) as clk:
            res = run_widths(args, world, device, peaks)
        mean = sum(v["2048"]["tflops"] for v in res.values()) / len(res)
        r = {"value": round(mean, 1), "unit": "TFLOP/s", "ms_per_step": None,
             "dtype": "affine 2/3/4/6-bit weights, bf16 activations, fp32 accumulate",
             "config": {"workload": "affine_widths_and_transpose0_g64_n12288_k4096", "M": [1, 512, 2048],
                        "value": "mean TFLOP/s at M=2048 over the five weight layouts"},
             "per_format": res,
             "roofline": {"bound": "tensor", "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": round(mean / peaks["bf16_tflops"], 4), "achieved": round(mean, 1), "traffic": None},
             "clocks": clk.summary(), "gpu_launches": None, "e2e": None}
    else:
        fmt, Ms = {"affine4_prefill": ("affine4", (512, 2048, 8192)),
                   "affine8_sweep": ("affine8", (1, 32, 512, 2048, 8192)),
                   "q4_0_prefill": ("q4_0", (512, 2048, 8192))}[args.workload]
        if args.ms:
            Ms = tuple(int(v) for v in args.ms.split(","))
        with ClockSampler(local_rank) as clk:
            res, tflops = run_prefill(args, world, device, peaks, fmt, Ms)
        r = {"value": round(tflops, 1), "unit": "TFLOP/s", "ms_per_step": None, "higher_is_better": True,
             "dtype": f"{fmt} weights, bf16 activations, fp32 accumulate",
             "config": {"workload": f"{fmt}_g{_fmt_args(fmt)[0]}_n12288_k4096", "M": list(Ms)}, "per_m": res,
             "crossover_m": next((int(m) for m, v in res.items() if v["pair_us"] < v["fused_us"]), None),
             "roofline": {"bound": "tensor", "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": round(tflops / peaks["bf16_tflops"], 4), "achieved": round(tflops, 1),
                          "traffic": None},
             "clocks": clk.summary(), "gpu_launches": None, "e2e": None}
    r["roofline"]["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"

    line = {"metric": "prefill TFLOP/s (% bf16 TC peak); M=1 GEMV GB/s (% HBM peak)", "value": r["value"],
            "unit": r["unit"], "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": r["dtype"], "data": "synthetic (seeded N(0, 0.02) weights, N(0, 1) bf16 activations)",
            "config": dict(r["config"], parallelism=f"replicas x{world}")}
    for k in ("per_m", "per_format", "crossover_m", "roofline", "e2e", "gpu_launches", "clocks", "secondary"):
        if k in r:
            line[k] = r[k]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb, _ = oracle_decode_sample(args.cpu_budget)
        line["cpu_baseline"] = cb
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

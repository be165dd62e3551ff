"""Benchmark of the weight-only block-quantized matmul hot path on B200.

Headline (one JSON line on rank 0): the Q4_0 decode GEMV, one token, of the
12288 x 4096 MLP up-projection -- the micro-benchmark shape of the MLX issue
"quantized_matmul takes 14-41% longer than dequantize + bf16 matmul at prefill
sizes (> 512 tokens)" (Repro).  One step is one quant_matmul call; 12 rotating
copies of the packed weights (340 MB > 126 MB of L2) make every launch read its
weights from HBM.  value = packed weight + scale bytes read / time, and
roofline.frac = that over the measured copy bandwidth.

The default run also measures, under "secondary", every other workload of the
scope: decode at 8, 16 and 32 tokens; prefill of Q4_0, affine 4-bit and affine
8-bit at 512 / 2048 / 8192 tokens (fused kernel, unfused pair, our bf16 GEMM,
cuBLAS for context, and the dispatcher's choice), the affine 8-bit sweep with
its fused/unfused crossover, the 16 x 256 x 512 Q4_0 check problem, the
Llama-3.2-1B-shaped projection stack at 512 tokens and 1 token, and the CPU
oracle on prefill sizes (full at 512 tokens, a 64-token sample above).

Multi-GPU (torchrun): the weight rows of one tall matrix are sharded across
ranks, 12288 rows per rank, x replicated (weak scaling; no exchange is needed
for the matmul itself, --gather adds an NCCL all-gather of y, timed apart).
--impl reference times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
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

METRIC = "prefill TFLOP/s (% bf16 TC peak); M=1 GEMV GB/s (% HBM peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
CSRC = os.path.join(ROOT, "bit_quantized_gemm_quant_b200", "csrc")

# dram__bytes_read.sum + dram__bytes_write.sum of one launch from one ncu capture,
# with the hash of the kernel's source file at that capture.  A kernel whose
# source changed since reports traffic null.
NCU_TRAFFIC = {
    "gemv_kernel<Q4_0> M=1": {"bytes": 28332288, "source": "gemv.cuh", "sha16": "94efba42044385eb",
                              "capture": "2026-12-02 ncu --set full, profiles/gemv_kernel_q4_0_decode_m1_n12288_k4096.md"},
    "gemv_tma_kernel<Q4_0> M=1": {"bytes": 28392704, "source": "gemv_stream.cuh", "sha16": "1b64b04575034f32",
                                  "capture": "2026-12-02 ncu --set full, profiles/gemv_tma_kernel_q4_0_decode_m1_n12288_k4096.md"},
}


def source_sha16(name: str) -> str:
    with open(os.path.join(CSRC, name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def stored_traffic(kernel: str):
    """(bytes per launch or None, provenance) of the stored capture of `kernel`."""
    e = NCU_TRAFFIC.get(kernel)
    if not e or e["bytes"] is None:
        return None, "no capture stored for this kernel build"
    cur = source_sha16(e["source"])
    if cur != e["sha16"]:
        return None, f"stale: {e['source']} is {cur}, the capture was of {e['sha16']}"
    return e["bytes"], f"ncu capture {e['capture']} of {e['source']} {e['sha16']}"


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


def decode_kernel(bq, M, N, K, gs, bits, path=None):
    """Which kernel(s) quant_matmul runs for this shape (the library's own answer,
    quant_matmul_gemv_kernel): the dispatcher's path, and on a decode path the kernel
    and its launches per call."""
    if path is None:
        path = {v: k for k, v in bq.PATHS.items()}[bq.quant_matmul_select_path(M, N, K, gs, bits)]
    k = bq.quant_matmul_gemv_kernel(M, N, K, gs, bits, path) if path in ("gemv", "gemv_stream") else -1
    if k < 0:
        return {"path": path, "kernel": path, "launches_per_call": None}
    return {"path": path, "kernel": bq.GEMV_KERNELS[k], "launches_per_call": 2 if k == 2 else 1}


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




# ----------------------------------------------------------------------------- row shards (multi-GPU)
def shard_rows(rows_per_rank: int, rank: int) -> tuple:
    """Rows [first, last) of the tall matrix that `rank` owns: each rank holds
    rows_per_rank consecutive weight rows (with their scales), x is replicated."""
    return rank * rows_per_rank, (rank + 1) * rows_per_rank


def shard_seed(seed: int, rank: int) -> int:
    """Seed of the generator of rank `rank`'s rows (rank 0 keeps the workload's seed)."""
    return seed + 7919 * rank


def assemble_shards(shards):
    """y [M][N_total] from the per-rank y [M][rows_per_rank] in rank order (torch tensors)."""
    import torch
    return torch.cat(list(shards), dim=1)


def decode_config(world: int) -> dict:
    """The headline workload, identical in both arms."""
    from bit_quantized_gemm_quant_b200 import workloads
    wl = workloads.Q4_0_DECODE
    return {"workload": "q4_0_decode_m1_n12288_k4096", "fmt": "q4_0", "N": wl.N * world, "K": wl.K, "M": 1,
            "rows_per_rank": wl.N, "parallelism": f"weight-row shards x{world}"}


# ----------------------------------------------------------------------------- GPU workloads
def run_decode(args, world, rank, device, peaks):
    """Headline: one-token Q4_0 GEMV over this rank's 12288 x 4096 shard, 12 rotating copies."""
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs, workloads

    wl = workloads.Q4_0_DECODE
    N, K = wl.N, wl.K
    gs, bits = _fmt_args(wl.fmt)
    wq0, s0, _ = make_weights(wl.fmt, N, K, shard_seed(wl.seed, rank), device)
    n_copies = 12
    copies = [(wq0, s0)] + [(wq0.clone(), s0.clone()) for _ in range(n_copies - 1)]
    g = inputs.generator(wl.seed + 1)                      # x is replicated: the same on every rank
    xs = {M: inputs.activations_bf16(M, K, g).to(device) for M in (1, 2, 8, 16, 32)}
    ys = {M: torch.empty(M, N, dtype=torch.bfloat16, device=device) for M in xs}
    wbytes = workloads.packed_weight_bytes(wl.fmt, N, K, gs)
    assert n_copies * wbytes > 2 * L2_BYTES

    def steps_fn(n):
        # n consecutive steps, each on the next copy: every copy is read once per 12 steps
        def f():
            for j in range(n):
                wq, s = copies[j % n_copies]
                bq.quant_matmul(xs[1], wq, s, None, gs, bits, out=ys[1])
        return f

    # the timed steps run as graphs of 12 launches (the launches of one graph may
    # overlap their set-up with the previous kernel) plus one graph of the rest
    full, rest = divmod(args.steps, n_copies)
    g_full = GraphTimer(steps_fn(n_copies))
    g_rest = GraphTimer(steps_fn(rest)) if rest else None
    for _ in range(max(1, -(-args.warmup // n_copies))):
        g_full.replay()
    torch.cuda.synchronize()
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        secs = time_graphs([g_full] * full + ([g_rest] if g_rest else []), full + (1 if g_rest else 0), world,
                           device)
    secs_max = max_over_ranks(secs, world, device)
    value = aggregate(args.steps * wbytes, world, secs_max) / 1e9

    # per-launch device time of each token count, same launch configuration
    per_m = {}
    for M in xs:
        fns = [(lambda wq=wq, s=s, M=M: bq.quant_matmul(xs[M], wq, s, None, gs, bits, out=ys[M]))
               for (wq, s) in copies]
        t = kernel_seconds(fns, 4)
        per_m[str(M)] = {"us": round(t * 1e6, 3), "gbs": round(wbytes / t / 1e9, 1),
                         "frac_hbm": round(wbytes / t / 1e9 / peaks["hbm_gbs"], 4),
                         "tflops": round(2.0 * M * N * K / t / 1e12, 3), **decode_kernel(bq, M, N, K, gs, bits)}
    # the streamed integer-MMA kernel forced at one and two tokens (BQ_PATH_GEMV takes it
    # at one token, and at two for the affine formats)
    forced = {}
    for M in (1, 2):
        fns = [(lambda wq=wq, s=s, M=M: bq.quant_matmul_ex(xs[M], wq, s, None, gs, bits, True, "gemv_stream",
                                                             out=ys[M])) for (wq, s) in copies]
        t = kernel_seconds(fns, 4)
        forced[str(M)] = {"us": round(t * 1e6, 3), "gbs": round(wbytes / t / 1e9, 1),
                          "frac_hbm": round(wbytes / t / 1e9 / peaks["hbm_gbs"], 4),
                          **decode_kernel(bq, M, N, K, gs, bits, "gemv_stream")}
    # affine 4-bit weights stored [K][N] (transpose = 0, groups of 64 along N) at the
    # same N and K: the dispatcher's decode GEMV over [K][N] (1 to 4 tokens) against
    # the unfused pair (forced), same rotation over copies and graph timing
    transpose0 = None
    if not args.no_secondary:
        gk = inputs.generator(wl.seed + 2)
        w_kn = inputs.weights_bf16_valued(K, N, gk).to(device).float()
        kq, ks_, kb_ = bq.affine_quantize(w_kn, 64, 4)
        del w_kn
        kbytes = kq.numel() * 4 + ks_.numel() * 2 + kb_.numel() * 2
        kcopies = [(kq, ks_, kb_)] + [(kq.clone(), ks_.clone(), kb_.clone())
                                      for _ in range(-(-2 * L2_BYTES // kbytes))]
        transpose0 = {"weights": f"affine 4-bit [K={K}][N={N}], group 64 along N", "copies": len(kcopies)}
        for M in (1, 2, 4):
            xk = inputs.activations_bf16(M, K, gk).to(device)
            yk = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            tg = kernel_seconds([(lambda c=c: bq.quant_matmul(xk, c[0], c[1], c[2], 64, 4, False, out=yk))
                                 for c in kcopies], 4)
            tp = kernel_seconds([(lambda c=c: bq.quant_matmul_ex(xk, c[0], c[1], c[2], 64, 4, False, "dequant_gemm",
                                                                 out=yk)) for c in kcopies[:4]], 2)
            transpose0[str(M)] = {"gemv_us": round(tg * 1e6, 3), "gemv_gbs": round(kbytes / tg / 1e9, 1),
                                  "gemv_frac_hbm": round(kbytes / tg / 1e9 / peaks["hbm_gbs"], 4),
                                  "kernel": "gemv_t_kernel", "pair_us": round(tp * 1e6, 3)}
        del kcopies

    # the quantized-activation path (opt-in, approximate): activation quantization
    # plus the Q4_0 x int8 GEMV, same weights, rotation and graph timing
    fns = [(lambda wq=wq, s=s: bq.quant_matmul_q8(*bq.q8_1_quantize(xs[1]), wq, s, out=ys[1])) for (wq, s) in copies]
    t_all = kernel_seconds(fns, 4)
    xq, dxq, qsq = bq.q8_1_quantize(xs[1])
    t_g = kernel_seconds([(lambda wq=wq, s=s: bq.quant_matmul_q8(xq, dxq, qsq, wq, s, out=ys[1]))
                          for (wq, s) in copies], 4)
    q8 = {"us": round(t_all * 1e6, 3), "gbs": round(wbytes / t_all / 1e9, 1), "gemv_us": round(t_g * 1e6, 3),
          "gemv_gbs": round(wbytes / t_g / 1e9, 1), "gemv_frac_hbm": round(wbytes / t_g / 1e9 / peaks["hbm_gbs"], 4),
          "note": "opt-in approximate path: q8_1_quantize + quant_matmul_q8; not the headline value"}

    t1 = per_m["1"]["us"] * 1e-6
    kname = per_m["1"]["kernel"]
    traffic, traffic_src = stored_traffic(f"{kname.split(' ')[-1]}<Q4_0> M=1")
    roof = {"bound": "hbm", "kernel": f"{kname} <Q4_0> (M=1)", "achieved": per_m["1"]["gbs"],
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": per_m["1"]["frac_hbm"], "traffic": traffic,
            "traffic_source": traffic_src, "algorithmic_bytes_per_launch": wbytes,
            "launch_us": round(t1 * 1e6, 3)}

    # end to end through the public API with host buffers: the step's inputs (this
    # rank's weight shard and x) copied in from pinned memory, y read back
    e2e = None
    if not args.no_e2e:
        h_wq, h_s, h_x = wq0.cpu().pin_memory(), s0.cpu().pin_memory(), xs[1].cpu().pin_memory()
        h_y = torch.empty(1, N, dtype=torch.bfloat16).pin_memory()
        d_wq, d_s, d_x = torch.empty_like(wq0), torch.empty_like(s0), torch.empty_like(xs[1])
        e2e_steps = max(3, min(args.steps, 20))

        def e2e_step():
            d_wq.copy_(h_wq, non_blocking=True)
            d_s.copy_(h_s, non_blocking=True)
            d_x.copy_(h_x, non_blocking=True)
            bq.quant_matmul(d_x, d_wq, d_s, None, gs, bits, out=ys[1])
            h_y.copy_(ys[1], non_blocking=True)
        e2e_step()
        torch.cuda.synchronize()
        t0, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(e2e_steps):
            e2e_step()
        t1e.record()
        torch.cuda.synchronize()
        es = max_over_ranks(t0.elapsed_time(t1e) / 1000.0, world, device)
        h2d = h_wq.numel() * h_wq.element_size() + h_s.numel() * 2 + h_x.numel() * 2
        e2e = {"value": round(aggregate(e2e_steps * wbytes, world, es) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(h_y.numel() * 2), "steps": e2e_steps}

    # optional: reassemble y of the whole tall matrix on every rank (NCCL all-gather), timed apart
    gather = None
    if args.gather and world > 1:
        import torch.distributed as dist
        y1 = ys[1].contiguous()
        outs = [torch.empty_like(y1) for _ in range(world)]
        dist.all_gather(outs, y1)
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 20
        dist.barrier()
        ev0.record()
        for _ in range(reps):
            dist.all_gather(outs, y1)
        ev1.record()
        torch.cuda.synchronize()
        gsec = max_over_ranks(ev0.elapsed_time(ev1) / 1000.0 / reps, world, device)
        full = assemble_shards(outs)
        gather = {"us": round(gsec * 1e6, 3), "y_shape": list(full.shape), "collective": "NCCL all_gather of y"}

    return {
        "value": round(value, 2), "unit": "GB/s", "ms_per_step": secs_max / args.steps * 1e3,
        "frac_hbm": round(value / world / peaks["hbm_gbs"], 4),
        "higher_is_better": True, "dtype": "q4_0 weights, bf16 activations, fp32 accumulate",
        "config": decode_config(world),
        "notes": {"l2": f"{n_copies} rotating weight copies per rank ({n_copies * wbytes / 1e6:.0f} MB > 126 MB L2)",
                  "bytes_per_step": wbytes * world, "path": "quant_matmul auto -> " + per_m["1"]["path"],
                  "timing": "CUDA events around graph replays of back-to-back launches, max over ranks"},
        "per_m": per_m, "roofline": roof, "e2e": e2e,
        "gpu_launches": args.steps * per_m["1"]["launches_per_call"], "clocks": clk.summary(),
        "secondary": {"q8_activation_path_m1": q8, "streamed_int_kernel_forced": forced,
                      "transpose0_affine4_decode": transpose0}, "gather": gather,
    }


def run_prefill(args, world, device, peaks, fmt, Ms):
    """TFLOP/s per token count of the fused kernel (GEMV at decode sizes), the unfused
    pair, our bf16 GEMM alone, cuBLAS bf16 (context) and the dispatcher's own choice,
    on the 12288 x 4096 projection; the fused/pair crossover is the first measured M
    from which the pair is faster."""
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs

    N, K = 12288, 4096
    gs, bits = _fmt_args(fmt)
    wq, s, b = make_weights(fmt, N, K, 0, device)
    g = inputs.generator(1)
    ws = torch.empty(N * K, dtype=torch.bfloat16, device=device)
    wb = ws.view(N, K)
    res = {}
    names = {v: k for k, v in bq.PATHS.items()}
    for M in Ms:
        x = inputs.activations_bf16(M, K, g).to(device)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        flops = 2.0 * M * N * K
        reps = max(10, min(50, int(2e13 / flops)))
        fused_path = "tc_fused" if M > 32 else "gemv"
        t_fused = kernel_seconds([lambda: bq.quant_matmul_ex(x, wq, s, b, gs, bits, True, fused_path, out=y)], reps)
        if M <= 32:
            # decode sizes: rotating weight copies (> 2x L2) so that every launch reads HBM
            from bit_quantized_gemm_quant_b200 import workloads
            nc = -(-3 * L2_BYTES // workloads.packed_weight_bytes(fmt, N, K, gs))
            cps = [(wq.clone(), s.clone(), None if b is None else b.clone()) for _ in range(nc)]
            t_auto = kernel_seconds([(lambda c=c: bq.quant_matmul(x, c[0], c[1], c[2], gs, bits, out=y))
                                     for c in cps], 4)
            del cps
        else:
            t_auto = kernel_seconds([lambda: bq.quant_matmul(x, wq, s, b, gs, bits, out=y)], reps)
        t_pair = kernel_seconds([lambda: bq.quant_matmul_ex(x, wq, s, b, gs, bits, True, "dequant_gemm",
                                                           workspace=ws, out=y)], reps)
        if fmt == "q4_0":
            bq.q4_0_dequantize(wq, s, out=wb)
        else:
            bq.affine_dequantize(wq, s, b, gs, bits, out=wb)
        t_gemm = kernel_seconds([lambda: bq.bf16_matmul(x, wb, out=y)], reps)
        t_cublas = kernel_seconds([lambda: torch.matmul(x, wb.t(), out=y)], reps)
        auto = names[bq.quant_matmul_select_path(M, N, K, gs, bits)]
        tf = flops / t_auto / 1e12
        res[str(M)] = {"fused_us": round(t_fused * 1e6, 2), "pair_us": round(t_pair * 1e6, 2),
                       "auto_us": round(t_auto * 1e6, 2), "auto_path": auto,
                       "fused_tflops": round(flops / t_fused / 1e12, 1), "pair_tflops": round(flops / t_pair / 1e12, 1),
                       "auto_tflops": round(tf, 1), "bf16_gemm_tflops": round(flops / t_gemm / 1e12, 1),
                       "cublas_bf16_tflops": round(flops / t_cublas / 1e12, 1),
                       "roofline": {"bound": "tensor" if M > 32 else "hbm", "kernel": f"quant_matmul auto -> {auto}",
                                    "achieved": round(tf, 1) if M > 32 else None,
                                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                    "frac": round(tf / peaks["bf16_tflops"], 4)}}
        if M <= 32:
            from bit_quantized_gemm_quant_b200 import workloads
            wbytes = workloads.packed_weight_bytes(fmt, N, K, gs)
            res[str(M)]["roofline"] = {"bound": "hbm", "kernel": f"quant_matmul auto -> {auto}",
                                       "achieved": round(wbytes / t_auto / 1e9, 1), "peak": peaks["hbm_gbs"],
                                       "unit": "GB/s", "frac": round(wbytes / t_auto / 1e9 / peaks["hbm_gbs"], 4),
                                       "note": "auto path over rotating weight copies (HBM reads)"}
        del x, y
    cross = next((int(m) for m, v in sorted(res.items(), key=lambda kv: int(kv[0]))
                  if int(m) > 32 and v["pair_us"] < v["fused_us"]), None)
    return res, cross


def run_small(args, device, peaks):
    """The 16 x 256 x 512 Q4_0 check problem (launch-bound): auto path time."""
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    from bit_quantized_gemm_quant_b200 import inputs, workloads
    wl = workloads.Q4_0_SMALL
    wq, s, _ = make_weights("q4_0", wl.N, wl.K, wl.seed, device)
    x = inputs.activations_bf16(16, wl.K, inputs.generator(wl.seed + 1)).to(device)
    y = torch.empty(16, wl.N, dtype=torch.bfloat16, device=device)
    t = kernel_seconds([lambda: bq.quant_matmul(x, wq, s, None, 32, 4, out=y)], 50)
    return {"us": round(t * 1e6, 3), "tflops": round(2.0 * 16 * wl.N * wl.K / t / 1e12, 4),
            "path": {v: k for k, v in bq.PATHS.items()}[bq.quant_matmul_select_path(16, wl.N, wl.K, 32, 4)]}


def run_widths(args, world, device, peaks):
    """Affine 2/3/6-bit weights and transpose=False (W stored [K][N], grouped along N): the
    dequantize (bytes moved, GB/s) and quant_matmul's auto path per M (the decode GEMV at one
    token -- over [K][N] for affine4_transpose0 -- the unfused pair at 512 and 2048 tokens)."""
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
def _decode_problem():
    import numpy as np
    import torch
    import oracle
    from bit_quantized_gemm_quant_b200 import inputs, workloads
    wl = workloads.Q4_0_DECODE
    g = inputs.generator(wl.seed)
    w = inputs.weights_fp32(wl.N, wl.K, g).numpy()
    wq, d = oracle.q4_0_quantize(w)
    x = inputs.activations_bf16(1, wl.K, inputs.generator(wl.seed + 1)).view(torch.int16).numpy().view(np.uint16)
    return wl, wq, d, x


def oracle_decode_step(wq, d, x, rows: int) -> int:
    """One oracle decode step over the first `rows` weight rows: dequantize them and
    take the float64 product with the one token.  Returns the host threads used."""
    import os as _os
    import oracle
    wb = oracle.q4_0_dequantize(wq[:rows], d[:rows])
    _, _, threads = oracle.matmul_ref(x, wb, nthreads=_os.cpu_count())
    return threads


def oracle_decode_timing(steps: int, warmup: int, budget_s: float):
    """The oracle on the headline workload, exactly warmup + steps steps; each step a
    row sample of the 12288 x 4096 matrix sized so that the run takes about
    budget_s (all rows when that fits).  GB/s of the sampled rows' packed bytes."""
    from bit_quantized_gemm_quant_b200 import workloads
    wl, wq, d, x = _decode_problem()
    t0 = time.perf_counter()
    oracle_decode_step(wq, d, x, 512)
    per_row = (time.perf_counter() - t0) / 512
    rows = int(budget_s / max(1, steps + warmup) / per_row)
    rows = max(16, min(wl.N, rows // 16 * 16))
    for _ in range(warmup):
        oracle_decode_step(wq, d, x, rows)
    t0 = time.perf_counter()
    threads = 1
    for _ in range(steps):
        threads = oracle_decode_step(wq, d, x, rows)
    el = time.perf_counter() - t0
    wbytes = workloads.packed_weight_bytes("q4_0", rows, wl.K, 32)
    return {"value": round(steps * wbytes / el / 1e9, 5), "unit": "GB/s", "cores": int(threads), "kind": "oracle",
            "sample": f"{steps} step(s) of a one-token decode over {rows} of the {wl.N} weight rows "
                      f"(dequantize + float64 product), {el:.1f} s"}, el / steps


def oracle_prefill_timing(budget_s: float):
    """The oracle on prefill sizes of the affine 4-bit projection: 512 tokens in full,
    2048 and 8192 tokens on a 64-token sample (rate extrapolated to the full size)."""
    import numpy as np
    import torch
    import oracle
    from bit_quantized_gemm_quant_b200 import inputs
    N, K = 12288, 4096
    g = inputs.generator(0)
    w = inputs.weights_bf16_valued(N, K, g).numpy()
    wq, s, b = oracle.affine_quantize(w, 64, 4)
    t0 = time.perf_counter()
    wb = oracle.affine_dequantize(wq, s, b, 64, 4)
    t_deq = time.perf_counter() - t0
    out = {"dequantize_s": round(t_deq, 3)}
    xg = inputs.generator(1)
    for M, sample in ((512, 512), (2048, 64), (8192, 64)):
        if time.perf_counter() - t0 > budget_s:
            break
        x = inputs.activations_bf16(sample, K, xg).view(torch.int16).numpy().view(np.uint16)
        t1 = time.perf_counter()
        _, _, threads = oracle.matmul_ref(x, wb, nthreads=os.cpu_count())
        el = time.perf_counter() - t1
        rate = 2.0 * sample * N * K / el
        out[str(M)] = {"gflops": round(rate / 1e9, 3), "cores": int(threads), "tokens_timed": sample,
                       "full_s": round(2.0 * M * N * K / rate + t_deq, 2),
                       "extrapolated": sample < M}
    return out


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
    ap.add_argument("--no-secondary", action="store_true", help="only the headline decode measurement")
    ap.add_argument("--gather", action="store_true", help="N > 1: all-gather y of the sharded matrix (timed apart)")
    ap.add_argument("--cpu-budget", type=float, default=25.0)
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    rank, local_rank, world = dist_env()
    peaks, peak_src = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return 0
        cb, sec_per_step = oracle_decode_timing(args.steps, args.warmup, args.cpu_budget)
        line = {"metric": METRIC, "impl": "reference", "value": cb["value"], "unit": cb["unit"],
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_step * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded N(0, 0.02) weights, N(0, 1) bf16 activations)",
                "config": decode_config(args.gpus), "cpu_baseline": cb,
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
        r = run_decode(args, world, rank, device, peaks)
        if not args.no_secondary and world == 1:
            sec = r["secondary"]
            for fmt, Ms in (("q4_0", (512, 2048, 8192)), ("affine4", (512, 2048, 8192)),
                            ("affine8", (1, 32, 64, 128, 256, 512, 2048, 8192))):
                res, cross = run_prefill(args, world, device, peaks, fmt, Ms)
                sec[f"{fmt}_n12288_k4096"] = {"per_m": res, "crossover_m": cross}
            sec["q4_0_m16_n256_k512"] = run_small(args, device, peaks)
            per_m, packed, params, _ = run_stack(args, world, device, peaks)
            sec["llama3.2_1b_q4_0_projection_stack"] = {"per_m": per_m, "packed_bytes": packed, "params": params}
    elif args.workload == "llama1b_stack":
        with ClockSampler(local_rank) as clk:
            per_m, packed, params, launches = run_stack(args, world, device, peaks)
        r = {"value": per_m["512"]["tokens_per_s"], "unit": "tokens/s", "ms_per_step": per_m["512"]["us_per_stack"] / 1e3,
             "dtype": "q4_0 weights, bf16 activations, fp32 accumulate",
             "config": {"workload": "llama3.2_1b_q4_0_projection_stack_16_layers", "M": [512, 1],
                        "params": params, "packed_bytes": packed},
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
                   "affine8_sweep": ("affine8", (1, 32, 64, 128, 256, 512, 2048, 8192)),
                   "q4_0_prefill": ("q4_0", (512, 2048, 8192))}[args.workload]
        if args.ms:
            Ms = tuple(int(v) for v in args.ms.split(","))
        with ClockSampler(local_rank) as clk:
            res, cross = run_prefill(args, world, device, peaks, fmt, Ms)
        big = [m for m in Ms if m > 32]
        tflops = (sum(2.0 * m * 12288 * 4096 for m in big) /
                  sum(res[str(m)]["auto_us"] * 1e-6 for m in big) / 1e12) if big else 0.0
        r = {"value": round(tflops, 1), "unit": "TFLOP/s", "ms_per_step": None, "higher_is_better": True,
             "dtype": f"{fmt} weights, bf16 activations, fp32 accumulate",
             "config": {"workload": f"{fmt}_g{_fmt_args(fmt)[0]}_n12288_k4096", "M": list(Ms)}, "per_m": res,
             "crossover_m": cross,
             "roofline": {"bound": "tensor", "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": round(tflops / peaks["bf16_tflops"], 4), "achieved": round(tflops, 1),
                          "traffic": None},
             "clocks": clk.summary(), "gpu_launches": None, "e2e": None}
    r["roofline"]["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"

    line = {"metric": METRIC, "value": r["value"], "unit": r["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": r["dtype"],
            "data": "synthetic (seeded N(0, 0.02) weights, N(0, 1) bf16 activations)", "config": r["config"]}
    for k in ("frac_hbm", "notes", "per_m", "per_format", "crossover_m", "roofline", "e2e", "gpu_launches", "clocks",
              "gather", "secondary"):
        if k in r and r[k] is not None:
            line[k] = r[k]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb, _ = oracle_decode_timing(max(1, int(args.cpu_budget / 2)), 1, args.cpu_budget / 2)
        line["cpu_baseline"] = cb
        if args.workload == "q4_0_decode" and not args.no_secondary:
            line.setdefault("secondary", {})["oracle_cpu_affine4_prefill"] = oracle_prefill_timing(args.cpu_budget)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

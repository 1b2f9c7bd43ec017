#!/usr/bin/env python
"""Benchmark of the B200 QLoRA NF4 hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of the 7B-class
decoder MLP workload (gate/up W 18944x3584, down W 3584x18944, 8192 tokens,
r=64, alpha=16), for each of the three projections:

    qlora_quantize_4bit + nf4_double_quantize_hist
                                         (quantise the frozen bf16 weight; the
                                          DQ mean's histogram is built while
                                          quantising)
    nf4_dequantize                       (bf16 export of the base weight)
    qlora_linear_fwd                     (fused NF4-dequant GEMM + adapter)
    qlora_linear_bwd                     (dX, dA, dB; T saved by the forward)
    qlora_linear_fwd at 16 tokens        (decode-sized call)

Inputs are seeded synthetic Gaussians (qlora_linear_layers_b200.synth) and
larger than L2 per step (no flush needed).  `value` is the layer's tensor
FLOPs (forward, backward and decode of all projections, all ranks) divided
by the device time of the step, inputs resident in HBM.  `e2e` is the same
metric with every step's inputs copied from pinned host memory and the
adapter gradients read back.  Under torchrun every rank runs the same
workload on its own tokens and the adapter gradients are all-reduced
(data-parallel; weak scaling).

--impl reference times the CPU oracle (oracle/, NumPy fp64) on a bounded
sample of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA NF4 linear TFLOP/s & quant/dequant GB/s, % of B200 roofline"
# DRAM bytes (read + write) per launch of the fused forward GEMM
# (k_qlora_gemm_dual) on this workload, averaged over the step's three
# launches, from one ncu capture of each shape (dram__bytes_read.sum +
# dram__bytes_write.sum of `bench.py --case fwd --tokens 8192 --proj 0|2`):
# gate and up 369.9 MB, down 537.4 MB.  Set back to None when the
# kernel changes: the figure belongs to the kernel it was measured on.  The
# algorithmic bytes are about 405 MB per launch.
FWD_GEMM_DRAM_BYTES_PER_LAUNCH = (369.9e6 * 2 + 537.4e6) / 3
WORKLOAD = "mlp_7b"
DECODE_M = 16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the per-workload kernel timings after the step")
    ap.add_argument("--case", choices=["fwd", "bwd", "quantize", "dequantize", "dq", "decode", "merge"],
                    help="profiling aid: run one operation on one projection and exit")
    ap.add_argument("--proj", type=int, default=0, help="--case: projection 0 gate, 1 up, 2 down")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="--case: workload whose weight shape and rank to use (mlp_7b, decode_70b, "
                         "attn_proj_4096, bwd_4096)")
    ap.add_argument("--tokens", type=int, default=2048, help="--case: token count")
    ap.add_argument("--repeat", type=int, default=3, help="--case: timed calls after one warm-up call")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------
# Work accounting (algorithmic FLOPs and bytes)
# ---------------------------------------------------------------------------

def layer_flops(M, N, K, r):
    fwd = 2 * M * N * K + 2 * M * K * r + 2 * M * N * r
    # dX = dY W' + s U A, U = dY B, dA = s U^T X, dB = s dY^T T (T saved)
    bwd = 2 * M * N * K + 2 * M * N * r + 2 * M * K * r + 2 * M * K * r + 2 * M * N * r
    return fwd, bwd


def quant_bytes(n):          # read bf16, write codes + fp32 absmax
    return n * 2 + n // 2 + 4 * (n // 64)


def dq_bytes(n):             # finalise pass: read absmax, write int8 + group scales
    na = n // 64                 # (the quantise pass built the mean's histogram)
    return 4 * na + na + 4 * ((na + 255) // 256)


def dq_standalone_bytes(n):  # from an absmax array: read it twice (histogram, codes)
    na = n // 64
    return 8 * na + na + 4 * ((na + 255) // 256)


def dequant_bytes(n):        # read codes + int8 scales + group scales, write bf16
    na = n // 64
    return n // 2 + na + 4 * ((na + 255) // 256) + 2 * n


def merge_bytes(N, K, r):     # codes + int8 scales + group scales + A + B read, bf16 written
    n = N * K
    na = n // 64
    return n // 2 + na + 4 * ((na + 255) // 256) + 2 * r * (N + K) + 2 * n


def decode_bytes(M, N, K, r):
    n = N * K
    na = n // 64
    return n // 2 + na + 4 * ((na + 255) // 256) + 2 * M * K + 2 * r * K + 2 * N * r + 2 * M * N


# ---------------------------------------------------------------------------
# Clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_indices):
        self.idx = ",".join(str(i) for i in gpu_indices)
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", self.idx, "-lms", "100"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx.append(float(f[2]))
                    power.append(float(f[3]))
                except ValueError:
                    continue
                for nm, v in zip(names, f[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s, p in zip(sm, power) if p > 0.5 * max(power)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power)}


# ---------------------------------------------------------------------------
# Our implementation
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from qlora_linear_layers_b200.build import build
    build()
    import qlora_linear_layers_b200 as q
    from qlora_linear_layers_b200 import _lib, dp, synth

    lib = _lib.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[WORKLOAD]
    M, r, alpha = wl.M, wl.r, wl.alpha

    # ---- inputs: seeded on the host (pinned, for the end-to-end leg), then resident in HBM
    host, devt = [], []
    for p, (N, K) in enumerate(wl.weights):
        # replicated frozen weight and adapters; each rank its own tokens
        W = synth.weight(N, K, dp.replica_seed(wl.seed(synth.TID_W, p), rank), "bf16")
        X = synth.activations(M, K, dp.token_seed(wl.seed(synth.TID_X, p), rank))
        A = synth.activations(r, K, dp.replica_seed(wl.seed(synth.TID_A, p), rank), sigma=0.02)
        B = synth.activations(N, r, dp.replica_seed(wl.seed(synth.TID_B, p), rank), sigma=0.02)
        dY = synth.activations(M, N, dp.token_seed(wl.seed(synth.TID_DY, p), rank))
        h = {k: v.pin_memory() for k, v in dict(W=W, X=X, A=A, B=B, dY=dY).items()}
        host.append(h)
        d = {k: v.to(dev) for k, v in h.items()}
        n = N * K
        na = n // 64
        d["wq"] = q.NF4Tensor(
            packed=torch.empty(n // 2, dtype=torch.uint8, device=dev), rows=N, cols=K,
            absmax=torch.empty(na, dtype=torch.float32, device=dev),
            qabsmax=torch.empty(na, dtype=torch.int8, device=dev),
            dq_scale=torch.empty((na + 255) // 256, dtype=torch.float32, device=dev),
            dq_mean=torch.empty(4, dtype=torch.float32, device=dev)[:1], double_quant=True)
        d["Wdeq"] = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        d["Y"] = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        d["T"] = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
        d["dX"] = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        d["dA"] = torch.empty(r, K, dtype=torch.bfloat16, device=dev)
        d["dB"] = torch.empty(N, r, dtype=torch.bfloat16, device=dev)
        d["Ydec"] = torch.empty(DECODE_M, N, dtype=torch.bfloat16, device=dev)
        h["dA_out"] = torch.empty(r, K, dtype=torch.bfloat16).pin_memory()
        h["dB_out"] = torch.empty(N, r, dtype=torch.bfloat16).pin_memory()
        devt.append(d)
    ws_bytes = 0
    for (N, K) in wl.weights:
        ws_bytes = max(ws_bytes, q.workspace_bytes(_lib.QLORA_OP_FWD, M, N, K, r),
                       q.workspace_bytes(_lib.QLORA_OP_BWD, M, N, K, r),
                       q.workspace_bytes(_lib.QLORA_OP_FWD, DECODE_M, N, K, r),
                       q.workspace_bytes(_lib.QLORA_OP_DOUBLE_QUANT, 0, N * K // 64, 0, 0))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    torch.cuda.synchronize()

    comps = ("quantize", "double_quant", "dequantize", "fwd", "bwd", "decode")
    stream = torch.cuda.current_stream()

    def step_proj(p, d, record, gemm_ev):
        wq = d["wq"]
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)] if record is not None else None
        if ev: ev[0].record(stream)
        # quantise, building the DQ mean's histogram on the way; then the DQ pass
        q.qlora_quantize_4bit(d["W"], wq.packed, wq.absmax, 0, hist)
        if ev: ev[1].record(stream)
        q.nf4_double_quantize_hist(wq.absmax, hist, wq.absmax.numel(), wq.qabsmax, wq.dq_scale,
                                   wq.dq_mean)
        if ev: ev[2].record(stream)
        q.nf4_dequantize(wq, d["Wdeq"])
        if ev: ev[3].record(stream)
        if gemm_ev is not None:
            g0, g1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
            # torch creates the CUDA event on first record; the library's
            # record at the GEMM launch supersedes this one
            g0.record(stream)
            g1.record(stream)
            lib.qlora_profile_gemm_events(g0.cuda_event, g1.cuda_event)
            gemm_ev.append((p, g0, g1))
        q.qlora_linear_fwd(wq, d["X"], d["A"], d["B"], alpha, d["Y"], d["T"], ws)
        if ev: ev[4].record(stream)
        q.qlora_linear_bwd(wq, d["X"], d["dY"], d["A"], d["B"], alpha, d["dX"], d["dA"], d["dB"],
                           T=d["T"], ws=ws)
        if ev: ev[5].record(stream)
        q.qlora_linear_fwd(wq, d["X"][:DECODE_M], d["A"], d["B"], alpha, d["Ydec"], None, ws)
        if ev: ev[6].record(stream)
        if world > 1:
            dp.allreduce_adapter_grads(d["dA"], d["dB"])
        if record is not None:
            record.append((p, ev))

    def step(record, gemm_ev):
        for p, d in enumerate(devt):
            step_proj(p, d, record, gemm_ev)

    def timed(nsteps, body):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(nsteps):
            body()
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = t0.elapsed_time(t1)
        if world > 1:
            t = torch.tensor([ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        return ms

    for _ in range(args.warmup):
        step(None, None)
    torch.cuda.synchronize()
    st = q.qlora_check_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    rec, gemm_ev = [], []
    sampler = ClockSampler(range(world)) if rank == 0 else None
    if sampler:
        sampler.start()
    l0 = lib.qlora_kernel_launches()
    total_ms = timed(args.steps, lambda: step(rec, gemm_ev))
    launches = lib.qlora_kernel_launches() - l0
    st = q.qlora_check_status()
    if st != 0:
        raise RuntimeError(f"device status {st} in the timed region")

    # ---- accounting
    step_flops = 0
    fwd_fl, bwd_fl, dec_fl = [], [], []
    for (N, K) in wl.weights:
        f, b = layer_flops(M, N, K, r)
        dfl, _ = layer_flops(DECODE_M, N, K, r)
        fwd_fl.append(f); bwd_fl.append(b); dec_fl.append(dfl)
        step_flops += f + b + dfl
    ms_step = total_ms / args.steps
    value = step_flops * world / (ms_step * 1e-3) / 1e12

    comp_ms = {c: 0.0 for c in comps}
    per_proj = [{c: 0.0 for c in comps} for _ in wl.weights]
    for p, ev in rec:
        for i, c in enumerate(comps):
            t = ev[i].elapsed_time(ev[i + 1])
            comp_ms[c] += t / args.steps
            per_proj[p][c] += t / args.steps
    gemm_ms = [0.0 for _ in wl.weights]
    for p, g0, g1 in gemm_ev:
        gemm_ms[p] += g0.elapsed_time(g1) / args.steps

    pk = peaks()
    hbm = pk["hbm_gbs"]
    tc_sus = pk["bf16_tflops_sustained"]
    tc_burst = pk["bf16_tflops"]
    nsum = sum(N * K for (N, K) in wl.weights)
    gbs = lambda nbytes, ms: nbytes / (ms * 1e-3) / 1e9
    components = {
        "quantize": {"ms": comp_ms["quantize"], "GB/s": gbs(sum(quant_bytes(N * K) for N, K in wl.weights), comp_ms["quantize"])},
        "double_quant": {"ms": comp_ms["double_quant"], "GB/s": gbs(sum(dq_bytes(N * K) for N, K in wl.weights), comp_ms["double_quant"])},
        "dequantize": {"ms": comp_ms["dequantize"], "GB/s": gbs(sum(dequant_bytes(N * K) for N, K in wl.weights), comp_ms["dequantize"])},
        "fwd": {"ms": comp_ms["fwd"], "TFLOP/s": sum(fwd_fl) / (comp_ms["fwd"] * 1e-3) / 1e12},
        "bwd": {"ms": comp_ms["bwd"], "TFLOP/s": sum(bwd_fl) / (comp_ms["bwd"] * 1e-3) / 1e12},
        "decode": {"ms": comp_ms["decode"], "GB/s": gbs(sum(decode_bytes(DECODE_M, N, K, r) for N, K in wl.weights), comp_ms["decode"])},
    }
    for c, v in components.items():
        if "GB/s" in v:
            v["frac_hbm"] = v["GB/s"] / hbm
        else:
            v["frac_tensor"] = v["TFLOP/s"] / tc_burst
    components["per_projection_ms"] = per_proj

    # dominant kernel: the fused NF4-dequant forward GEMM (one launch per
    # projection).  The timed region lasts well under a second, so the burst
    # peak is the denominator; the sustained peak is reported beside it.
    gemm_flops = [2 * M * N * K + 2 * M * N * r for (N, K) in wl.weights]
    achieved = sum(gemm_flops) / (sum(gemm_ms) * 1e-3) / 1e12
    roofline = {"kernel": "k_qlora_gemm_dual (fused NF4-dequant forward GEMM, two token tiles per weight stage, adapter as extra K steps, paired SMs)",
                "bound": "tensor", "achieved": achieved, "peak": tc_burst, "unit": "TFLOP/s",
                "frac": achieved / tc_burst, "traffic": FWD_GEMM_DRAM_BYTES_PER_LAUNCH,
                "peak_kind": f"bf16 dense, burst ({pk['source']}); the timed region lasts "
                             f"{total_ms / 1e3:.2f} s",
                "frac_of_sustained_peak": achieved / tc_sus,
                "per_launch_ms": gemm_ms,
                "per_launch_frac": [f / (t * 1e-3) / 1e12 / tc_burst for f, t in zip(gemm_flops, gemm_ms)],
                "algorithmic_flops_per_launch": gemm_flops,
                "algorithmic_bytes_per_launch": [N * K // 2 + (N * K // 64) + 4 * ((N * K // 64 + 255) // 256)
                                                 + 2 * M * K + 2 * M * r + 2 * N * r + 2 * M * N
                                                 for (N, K) in wl.weights],
                # the same launches counted on the base product 2MNK alone
                "achieved_base_only": sum(2 * M * N * K for (N, K) in wl.weights) / (sum(gemm_ms) * 1e-3) / 1e12}

    # ---- end-to-end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        h2d = sum(h[k].numel() * h[k].element_size() for h in host for k in ("W", "X", "A", "B", "dY"))
        d2h = sum(h[k].numel() * h[k].element_size() for h in host for k in ("dA_out", "dB_out"))

        # Each step copies every projection's inputs from pinned host memory on
        # a copy stream; a projection's compute waits for its own copies only,
        # and the next step's copies into a projection's buffers wait for the
        # compute that read them.  dA and dB are read back every step.
        copy_stream = torch.cuda.Stream(device=dev)
        ready = [torch.cuda.Event() for _ in devt]
        done = [torch.cuda.Event() for _ in devt]
        for e in done:
            e.record(stream)

        def e2e_step():
            for p, (h, d) in enumerate(zip(host, devt)):
                copy_stream.wait_event(done[p])
                with torch.cuda.stream(copy_stream):
                    for k in ("W", "X", "A", "B", "dY"):
                        d[k].copy_(h[k], non_blocking=True)
                ready[p].record(copy_stream)
            for p, (h, d) in enumerate(zip(host, devt)):
                stream.wait_event(ready[p])
                step_proj(p, d, None, None)
                done[p].record(stream)
                h["dA_out"].copy_(d["dA"], non_blocking=True)
                h["dB_out"].copy_(d["dB"], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        for e in done:
            e.record(stream)
        e_ms = timed(args.steps, e2e_step)
        e2e = {"value": step_flops * world / (e_ms / args.steps * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms / args.steps}
        if q.qlora_check_status() != 0:
            raise RuntimeError("device status set in the end-to-end leg")

    clocks = sampler.stop() if sampler else None
    extras = None
    if world == 1 and not args.no_extras:
        del devt, host, ws
        torch.cuda.empty_cache()
        extras = workload_timings(q, lib, dev, pk)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(budget_s=20.0)

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded Gaussian, no real weights)",
            "config": {"workload": "mlp_7b: 7B-class decoder MLP, gate/up W 18944x3584 and down "
                                   "W 3584x18944 NF4 (block 64, DQ 256), 8192 tokens per GPU, "
                                   "r=64, alpha=16; decode calls at 16 tokens",
                       "tokens_per_gpu": M, "r": r, "alpha": alpha,
                       "step": "quantize+DQ, dequantize, fwd, bwd, decode(16) per projection",
                       "l2": "inputs larger than L2 every step (>1 GB per step); no flush",
                       "parallelism": f"dp{world}"},
            "e2e": e2e, "gpu_launches": int(launches),
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clocks,
            "components": components,
            "workloads": extras,
        }
        print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# Kernel timings on the other workloads (single GPU, after the step)
# ---------------------------------------------------------------------------

def _time_op(fn, reps, flush):
    """Median device time (ms) of `fn` over `reps` calls, each preceded by an
    L2 flush outside the timed events."""
    import torch
    stream = torch.cuda.current_stream()
    fn()                                          # warm-up
    times = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def workload_timings(q, lib, dev, pk):
    """Quantise / DQ / dequantise and decode GEMV on the 70B-class projection
    (28672 x 8192, with and without 1 % outliers, M in {1, 4, 16}); the
    forward GEMM on the 4096^2 attention projection (4096 tokens, r = 16);
    the backward on 4096^2 (8192 tokens, r = 64).  Each figure is the median
    of CUDA-event times of single calls, with L2 flushed (a 256 MB write)
    before every call."""
    import torch
    from qlora_linear_layers_b200 import _lib, synth
    hbm, tc = pk["hbm_gbs"], pk["bf16_tflops"]
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush = lambda: scratch.zero_()
    gbs = lambda nbytes, ms: nbytes / (ms * 1e-3) / 1e9
    out = {"timing": "median of single calls, L2 flushed before each (256 MB write outside the events)",
           "peaks": {"hbm_gbs": hbm, "bf16_tflops": tc, "source": pk["source"]}}

    # ---- 70B-class projection: bulk quantisation and decode
    wl = synth.WORKLOADS["decode_70b"]
    N, K = wl.weights[0]
    n, na = N * K, N * K // 64
    r, alpha = wl.r, wl.alpha
    A = synth.activations(r, K, wl.seed(synth.TID_A), sigma=0.02).to(dev)
    B = synth.activations(N, r, wl.seed(synth.TID_B), sigma=0.02).to(dev)
    wsz = max(q.workspace_bytes(_lib.QLORA_OP_FWD, m, N, K, r) for m in wl.decode_M)
    wsz = max(wsz, q.workspace_bytes(_lib.QLORA_OP_DOUBLE_QUANT, 0, na, 0, 0))
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
    dec = {}
    for outliers in (False, True):
        W = synth.weight(N, K, wl.seed(synth.TID_W), "bf16", outliers=outliers).to(dev)
        wq = q.NF4Tensor(
            packed=torch.empty(n // 2, dtype=torch.uint8, device=dev), rows=N, cols=K,
            absmax=torch.empty(na, dtype=torch.float32, device=dev),
            qabsmax=torch.empty(na, dtype=torch.int8, device=dev),
            dq_scale=torch.empty((na + 255) // 256, dtype=torch.float32, device=dev),
            dq_mean=torch.empty(4, dtype=torch.float32, device=dev)[:1], double_quant=True)
        Wd = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        hist = torch.empty(256, dtype=torch.int64, device=dev)
        t_q = _time_op(lambda: q.qlora_quantize_4bit(W, wq.packed, wq.absmax, 0, hist), 10, flush)
        t_dq = _time_op(lambda: q.nf4_double_quantize_hist(wq.absmax, hist, na, wq.qabsmax,
                                                           wq.dq_scale, wq.dq_mean), 10, flush)
        t_dqs = _time_op(lambda: q.nf4_double_quantize(wq.absmax, wq.qabsmax, wq.dq_scale,
                                                       wq.dq_mean, ws), 10, flush)
        t_dd = _time_op(lambda: q.nf4_dequantize(wq, Wd), 10, flush)
        key = "outliers_1pct" if outliers else "gaussian"
        rec = {
            "quantize": {"us": t_q * 1e3, "GB/s": gbs(quant_bytes(n), t_q),
                         "frac_hbm": gbs(quant_bytes(n), t_q) / hbm, "bytes": quant_bytes(n)},
            "double_quant": {"us": t_dq * 1e3, "GB/s": gbs(dq_bytes(n), t_dq),
                             "frac_hbm": gbs(dq_bytes(n), t_dq) / hbm, "bytes": dq_bytes(n),
                             "pass": "finalise from the histogram built while quantising"},
            "double_quant_standalone": {"us": t_dqs * 1e3, "GB/s": gbs(dq_standalone_bytes(n), t_dqs),
                                        "frac_hbm": gbs(dq_standalone_bytes(n), t_dqs) / hbm,
                                        "bytes": dq_standalone_bytes(n)},
            "quantize_plus_dq": {"us": (t_q + t_dq) * 1e3,
                                 "GB/s": gbs(quant_bytes(n) + dq_bytes(n), t_q + t_dq),
                                 "frac_hbm": gbs(quant_bytes(n) + dq_bytes(n), t_q + t_dq) / hbm},
            "dequantize": {"us": t_dd * 1e3, "GB/s": gbs(dequant_bytes(n), t_dd),
                           "frac_hbm": gbs(dequant_bytes(n), t_dd) / hbm, "bytes": dequant_bytes(n)},
        }
        if not outliers:
            # the merge for export: codes + scales + A + B read, bf16 written
            t_m = _time_op(lambda: q.qlora_merge(wq, A, B, alpha, Wd), 10, flush)
            nb = merge_bytes(N, K, r)
            rec["merge"] = {"us": t_m * 1e3, "GB/s": gbs(nb, t_m), "frac_hbm": gbs(nb, t_m) / hbm,
                            "bytes": nb}
        del W, Wd
        for m in (wl.decode_M if not outliers else (16,)):
            X = synth.activations(m, K, wl.seed(synth.TID_X) + m).to(dev)
            Y = torch.empty(m, N, dtype=torch.bfloat16, device=dev)
            t = _time_op(lambda: q.qlora_linear_fwd(wq, X, A, B, alpha, Y, None, ws), 20, flush)
            nb = decode_bytes(m, N, K, r)
            rec[f"decode_M{m}"] = {"us": t * 1e3, "GB/s": gbs(nb, t), "frac_hbm": gbs(nb, t) / hbm,
                                   "bytes": nb}
        dec[key] = rec
        del wq
        torch.cuda.empty_cache()
    out["decode_70b"] = {"workload": wl.name, **dec}
    del ws, A, B
    torch.cuda.empty_cache()

    # ---- the merge on the 7B-class gate projection (r = 64)
    wl = synth.WORKLOADS["mlp_7b"]
    (N, K), r, alpha = wl.weights[0], wl.r, wl.alpha
    W = synth.weight(N, K, wl.seed(synth.TID_W), "bf16").to(dev)
    A = synth.activations(r, K, wl.seed(synth.TID_A), sigma=0.02).to(dev)
    B = synth.activations(N, r, wl.seed(synth.TID_B), sigma=0.02).to(dev)
    wq = q.quantize(W)
    Wd = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    t_m = _time_op(lambda: q.qlora_merge(wq, A, B, alpha, Wd), 10, flush)
    nb = merge_bytes(N, K, r)
    out["mlp_7b_gate_merge"] = {"us": t_m * 1e3, "GB/s": gbs(nb, t_m), "frac_hbm": gbs(nb, t_m) / hbm,
                                "bytes": nb, "shape": [N, K, r]}
    del W, A, B, wq, Wd
    torch.cuda.empty_cache()

    # ---- the 4096^2 attention projection forward and the 4096^2 backward
    for name in ("attn_proj_4096", "bwd_4096"):
        wl = synth.WORKLOADS[name]
        (N, K), M, r, alpha = wl.weights[0], wl.M, wl.r, wl.alpha
        W, X, A, B = (t.to(dev) for t in synth.layer_inputs(wl, 0))
        wq = q.quantize(W)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        T = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(q.workspace_bytes(_lib.QLORA_OP_FWD, M, N, K, r),
                             q.workspace_bytes(_lib.QLORA_OP_BWD, M, N, K, r)),
                         dtype=torch.uint8, device=dev)
        f_fl, b_fl = layer_flops(M, N, K, r)
        if name == "attn_proj_4096":
            t = _time_op(lambda: q.qlora_linear_fwd(wq, X, A, B, alpha, Y, T, ws), 10, flush)
            # the GEMM launch alone, from the library's events around it
            g = []
            for _ in range(5):
                flush()
                g0, g1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
                g0.record(); g1.record()
                lib.qlora_profile_gemm_events(g0.cuda_event, g1.cuda_event)
                q.qlora_linear_fwd(wq, X, A, B, alpha, Y, T, ws)
                g1.synchronize()
                g.append(g0.elapsed_time(g1))
            tg = statistics.median(g)
            gf = 2 * M * N * K + 2 * M * N * r
            out[name] = {"workload": wl.name,
                         "fwd": {"us": t * 1e3, "TFLOP/s": f_fl / (t * 1e-3) / 1e12,
                                 "frac_tensor": f_fl / (t * 1e-3) / 1e12 / tc},
                         "fwd_gemm_kernel": {"us": tg * 1e3, "TFLOP/s": gf / (tg * 1e-3) / 1e12,
                                             "frac_tensor": gf / (tg * 1e-3) / 1e12 / tc}}
        else:
            dY = synth.upstream_grad(wl, 0).to(dev)
            dX, dA, dB = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B)
            q.qlora_linear_fwd(wq, X, A, B, alpha, Y, T, ws)
            t = _time_op(lambda: q.qlora_linear_bwd(wq, X, dY, A, B, alpha, dX, dA, dB, T=T, ws=ws),
                         10, flush)
            g = []
            for _ in range(5):
                flush()
                g0, g1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
                g0.record(); g1.record()
                lib.qlora_profile_gemm_events(g0.cuda_event, g1.cuda_event)
                q.qlora_linear_bwd(wq, X, dY, A, B, alpha, dX, dA, dB, T=T, ws=ws)
                g1.synchronize()
                g.append(g0.elapsed_time(g1))
            tg = statistics.median(g)
            gf = 2 * M * N * K + 2 * M * K * r
            out[name] = {"workload": wl.name,
                         "bwd": {"us": t * 1e3, "TFLOP/s": b_fl / (t * 1e-3) / 1e12,
                                 "frac_tensor": b_fl / (t * 1e-3) / 1e12 / tc},
                         "bwd_dx_gemm_kernel": {"us": tg * 1e3, "TFLOP/s": gf / (tg * 1e-3) / 1e12,
                                                "frac_tensor": gf / (tg * 1e-3) / 1e12 / tc}}
        del W, X, A, B, wq, Y, T, ws
        torch.cuda.empty_cache()
    st = q.qlora_check_status()
    if st != 0:
        raise RuntimeError(f"device status {st} in the workload timings")
    return out


# ---------------------------------------------------------------------------
# The oracle on the host cores (bounded sample of the same workload)
# ---------------------------------------------------------------------------

def _oracle_inputs(rows, tokens):
    """Seeded inputs of the sampled sub-layers (generation is not timed)."""
    from qlora_linear_layers_b200 import synth
    wl = synth.WORKLOADS[WORKLOAD]
    out = []
    for p, (N, K) in enumerate(wl.weights):
        n = min(rows, N)
        out.append(dict(
            W=synth.weight(n, K, wl.seed(synth.TID_W, p), "bf16").float().numpy(),
            X=synth.activations(tokens, K, wl.seed(synth.TID_X, p)).float().numpy(),
            A=synth.activations(wl.r, K, wl.seed(synth.TID_A, p), sigma=0.02).float().numpy(),
            B=synth.activations(n, wl.r, wl.seed(synth.TID_B, p), sigma=0.02).float().numpy(),
            dY=synth.activations(tokens, n, wl.seed(synth.TID_DY, p)).float().numpy()))
    return out


def _oracle_sample(inputs):
    """Quantise + DQ + dequantise each sampled weight (its first output rows),
    then forward, backward and a 16-token decode of that sub-layer; returns the
    tensor FLOPs done."""
    import oracle
    from qlora_linear_layers_b200 import synth
    wl = synth.WORKLOADS[WORKLOAD]
    flops = 0
    for d in inputs:
        W, X, A, B, dY = d["W"], d["X"], d["A"], d["B"], d["dY"]
        n, K = W.shape
        tokens = X.shape[0]
        codes, a = oracle.quantize(W)
        qa, s, mu = oracle.double_quantize(a)
        Wd = oracle.dequantize(oracle.pack(codes), oracle.dq_absmax(qa, s, mu), W.shape)
        oracle.linear_fwd(X, Wd, A, B, wl.alpha, wl.r)
        oracle.linear_bwd(X, dY, Wd, A, B, wl.alpha, wl.r)
        oracle.linear_fwd(X[:DECODE_M], Wd, A, B, wl.alpha, wl.r)
        f, b = layer_flops(tokens, n, K, wl.r)
        dd, _ = layer_flops(DECODE_M, n, K, wl.r)
        flops += f + b + dd
    return flops


def _calibrate(budget_s):
    """Sample size (rows = tokens) whose oracle pass takes about budget_s."""
    size = 64
    while True:
        inp = _oracle_inputs(size, size)
        t = time.perf_counter()
        _oracle_sample(inp)
        el = time.perf_counter() - t
        if el >= budget_s / 4 or size >= 4096:
            break
        size *= 2
    # cost grows between linearly and quadratically with size
    scale = max(1.0, (budget_s / max(el, 1e-3)) ** 0.6)
    return int(min(8192, size * scale))


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _host_info():
    """The host CPU model and NumPy's BLAS, recorded beside the CPU timing."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    blas = "unknown"
    try:
        dep = np.show_config(mode="dicts")["Build Dependencies"]["blas"]
        blas = f"{dep.get('name', '?')} {dep.get('version', '')}".strip()
    except Exception:
        pass
    return {"cpu_model": model, "blas": blas}


def cpu_baseline(budget_s: float):
    """Time the oracle on a sample sized to roughly `budget_s` seconds."""
    size = _calibrate(budget_s)
    inp = _oracle_inputs(size, size)
    t = time.perf_counter()
    flops = _oracle_sample(inp)
    el = time.perf_counter() - t
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": f"each projection cut to its first {size} output rows and {size} tokens: "
                      "NumPy quantise + DQ + dequantise, fp64 forward, backward, 16-token decode",
            "seconds": el, **_host_info()}


def run_reference(args, rank, world):
    if rank != 0:
        return
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    size = _calibrate(budget)
    inp = _oracle_inputs(size, size)
    for _ in range(args.warmup):
        _oracle_sample(inp)
    t = time.perf_counter()
    flops = 0
    for _ in range(args.steps):
        flops += _oracle_sample(inp)
    el = time.perf_counter() - t
    value = flops / el / 1e12
    sample = (f"each projection cut to its first {size} output rows and {size} tokens per step: "
              "NumPy quantise + DQ + dequantise, fp64 forward, backward, 16-token decode")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Gaussian)",
           "config": {"workload": "mlp_7b (sampled for the CPU oracle)", "parallelism": "none"},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                            "sample": sample, **_host_info()},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_case(args):
    """One operation on one projection of the workload, `--repeat` times, for
    ncu captures of a single kernel on a small case."""
    import torch
    from qlora_linear_layers_b200.build import build
    build()
    import qlora_linear_layers_b200 as q
    from qlora_linear_layers_b200 import _lib, synth
    wl = synth.WORKLOADS[args.workload]
    N, K = wl.weights[min(args.proj, len(wl.weights) - 1)]
    M = min(args.tokens, DECODE_M) if args.case == "decode" else args.tokens
    r, alpha = wl.r, wl.alpha
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(1234 + args.proj)
    W = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    X = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
    A = (torch.randn(r, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    B = (torch.randn(N, r, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    dY = torch.randn(M, N, device=dev, generator=g).to(torch.bfloat16)
    wq = q.quantize(W)
    Y, T = q.linear_fwd(wq, X, A, B, alpha)
    Wd = torch.empty_like(W)
    ws = torch.empty(max(q.workspace_bytes(_lib.QLORA_OP_FWD, M, N, K, r),
                         q.workspace_bytes(_lib.QLORA_OP_BWD, M, N, K, r), 2048),
                     dtype=torch.uint8, device=dev)
    dX, dA, dB = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B)
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    ops = {
        "fwd": lambda: q.qlora_linear_fwd(wq, X, A, B, alpha, Y, T, ws),
        "decode": lambda: q.qlora_linear_fwd(wq, X, A, B, alpha, Y, None, ws),
        "bwd": lambda: q.qlora_linear_bwd(wq, X, dY, A, B, alpha, dX, dA, dB, T=T, ws=ws),
        "quantize": lambda: q.qlora_quantize_4bit(W, wq.packed, wq.absmax, 0, hist),
        "dq": lambda: q.nf4_double_quantize_hist(wq.absmax, hist, wq.absmax.numel(), wq.qabsmax,
                                                 wq.dq_scale, wq.dq_mean),
        "dequantize": lambda: q.nf4_dequantize(wq, Wd),
        "merge": lambda: q.qlora_merge(wq, A, B, alpha, Wd),
    }
    torch.cuda.synchronize()
    ops[args.case]()                                  # warm-up call
    torch.cuda.synchronize()
    # back-to-back calls so the host runs ahead and the events time the GPU
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.repeat):
        ops[args.case]()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": args.case, "N": N, "K": K, "M": M, "calls": args.repeat,
                      "ms_per_call": e0.elapsed_time(e1) / args.repeat}), flush=True)
    st = q.qlora_check_status()
    if st != 0:
        raise RuntimeError(f"device status {st}")


def _spawned_rank(local_rank, args, world, port):
    os.environ.update({"RANK": str(local_rank), "LOCAL_RANK": str(local_rank),
                       "WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    _run(args)


def _run(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def main():
    args = parse()
    if args.case:
        run_case(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not launched by torchrun: start one process per GPU here, ranks
        # meeting over NCCL on 127.0.0.1
        import socket
        import torch.multiprocessing as mp
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        mp.spawn(_spawned_rank, args=(args, args.gpus, port), nprocs=args.gpus, join=True)
        return
    _run(args)


if __name__ == "__main__":
    main()

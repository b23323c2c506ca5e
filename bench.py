"""Benchmark: FP8 fine-grained-scaled GEMM on B200 (dense NT projection sweep).

Workload (the dense sweep the pages' headline numbers are quoted on): M in
{64, 128, 4096} x (N, K) in {(2112,7168), (24576,1536), (32768,512),
(7168,16384), (4096,7168), (7168,2048)}; A, B ~ N(0,1) float32 from seeded
streams. Weights B are quantised once at set-up (128x128 blocks, static FP8
weights). One step = for every shape: quantise A (1x128 strips) on the GPU and
run D = A @ B.T (BF16 out), i.e. the whole hot path per shape. L2 is flushed
(256 MiB write) before every shape, outside the per-shape timing.

Reported (one JSON line, rank 0):
  value        whole-job TFLOP/s = sum of GEMM FLOPs / device time of the step
               (events around each shape's quantise + GEMM pair; the per-kernel
               split comes from a separate pass with an event between them)
  e2e          same metric through the public API with the activations copied
               from pinned host memory and D copied back inside the timed loop
  roofline     dominant kernel (the GEMM on its largest shape): achieved TFLOP/s
               vs the measured-derived FP8 peak; plus an HBM block for the
               decode shapes (M <= 128)
  cpu_baseline the CPU oracle on a bounded row sample of the same workload
--impl reference times that oracle as the reference arm (no GPU work).
Multi-GPU (--gpus N under torchrun): N independent replicas (the path has no
exchange step); value = work of all ranks / max over ranks of the step time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
import synth.workloads as wl  # noqa: E402

METRIC = "FP8 block-scaled GEMM TFLOPS & % of B200 FP8 peak; decode-shape HBM GB/s"
WORKLOAD = "dense_fp8_gemm_nt_sweep"
NOMINAL_FP8_TFLOPS = 4500.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK["hbm_gbs"], "bf16_tflops": FALLBACK["bf16_tflops"],
            "bf16_tflops_sustained": FALLBACK["bf16_tflops"], "source": "fallback"}


def shape_flops(M, N, K):
    return 2.0 * M * N * K


def shape_bytes(M, N, K):
    """Algorithmic bytes of one GEMM: A and B codes read once, D (bf16) written
    once, plus the FP32 scales."""
    return M * K + N * K + 2 * M * N + 4 * ((M + 3) // 4 * 4) * (K // 128) + \
        4 * ((N + 127) // 128) * (K // 128)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi every 100 ms from before the warm-up; stop() keeps
    the samples taken inside [t_start, t_end] (host wall clock), or the two
    nearest ones if the timed region was shorter than the sampling period."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.proc = None
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            import threading
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.5)  # let the first samples arrive before the timed region
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line))

    def stop(self, t_start: float, t_end: float):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        inside = [r for r in rows if t_start <= r[0] <= t_end + 0.1]
        if not inside:
            inside = sorted(rows, key=lambda r: abs(r[0] - 0.5 * (t_start + t_end)))[:2]
        reasons = set()
        for r in inside:
            for n, v in zip(names, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "samples": len(inside),
                "timed_region_s": round(t_end - t_start, 3), "reasons": sorted(reasons)}


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_grouped_gemm_07_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_from_profile(key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    e = d.get("launches", {}).get(key)
    return None if e is None else float(e["dram_bytes"])


# ----------------------------------------------------------------- CPU oracle
def oracle_sample(shapes, rows_per_shape, inputs):
    """Times the oracle on `rows_per_shape` rows of every shape: quantise those
    A rows and compute those output rows. B is quantised beforehand (static
    weights, as on the GPU side). Returns (flops, seconds, cores)."""
    import oracle
    flops = 0.0
    t0 = time.perf_counter()
    for (M, N, K) in shapes:
        A, qb, sb = inputs[(M, N, K)]
        rows = min(rows_per_shape, M)
        qa, sa = oracle.quantize(np.ascontiguousarray(A[:rows]), oracle.ROW_1x128)
        oracle.gemm_nt(qa, sa, qb, sb)
        flops += shape_flops(rows, N, K)
    return flops, time.perf_counter() - t0, oracle.num_threads()


def prepare_oracle_inputs(shapes, rows_per_shape):
    import oracle
    qb_cache = {}
    inputs = {}
    for i, (M, N, K) in enumerate(shapes):
        if (N, K) not in qb_cache:
            B = synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))
            qb_cache[(N, K)] = oracle.quantize(B, oracle.BLOCK_128x128)
        A = synth.normal((min(rows_per_shape, M), K), synth.seed(2, shape_index(M, N, K), 0))
        inputs[(M, N, K)] = (A,) + qb_cache[(N, K)]
    return inputs


def nk_index(N, K):
    return wl.DENSE_NK.index((N, K)) if (N, K) in wl.DENSE_NK else 99


def shape_index(M, N, K):
    sh = wl.dense_shapes()
    return sh.index((M, N, K)) if (M, N, K) in sh else 99


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    shapes = wl.dense_shapes()
    rows = args.ref_rows
    inputs = prepare_oracle_inputs(shapes, rows)
    for _ in range(args.warmup):
        oracle_sample(shapes, rows, inputs)
    tot_f, tot_s, cores = 0.0, 0.0, 1
    for _ in range(args.steps):
        f, s, cores = oracle_sample(shapes, rows, inputs)
        tot_f += f
        tot_s += s
    tflops = tot_f / tot_s / 1e12
    sample = (f"{rows} rows of each of the 18 shapes per step (A rows quantised + those output "
              f"rows of D), weights pre-quantised")
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "shapes": len(shapes), "sample_rows": rows},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- grouped workloads
def run_grouped(args):
    """--workload contiguous | masked | kgrouped: the MoE variants at their
    benchmark sizes (parity cases of the dense sweep's bench line, timed here
    for the record). One step = quantise the activations on the GPU + the
    grouped GEMM, inputs resident in HBM and larger than L2 (no flush needed).
    value = useful TFLOP/s (real rows only); one GPU, rank 0."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    kind = args.workload

    def put(x):
        return torch.from_numpy(x).to(dev)

    if kind == "contiguous":
        w = wl.contiguous()
        A = put(w.A)
        qb, sb = dg.dg_quantize_fp8(put(w.B), dg.DG_QUANT_BLOCK_128x128)
        mi = put(w.m_indices)
        qa = torch.empty(A.shape, dtype=torch.uint8, device=dev)
        sa = torch.zeros((w.K // 128, (w.Mt + 3) // 4 * 4), dtype=torch.float32, device=dev)
        D = torch.empty((w.Mt, w.N), dtype=torch.bfloat16, device=dev)
        flops = 2.0 * w.N * w.K * float(sum(w.rows))
        algo_bytes = w.Mt * w.K + w.G * w.N * w.K + 2 * w.Mt * w.N
        bound = "tensor"
        cfg = {"workload": "m_grouped_contiguous", "G": w.G, "N": w.N, "K": w.K, "Mt": w.Mt,
               "rows": [int(r) for r in w.rows]}

        def quant():
            dg.dg_quantize_fp8(A, dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)

        def gemm():
            dg.dg_m_grouped_fp8_gemm_nt_contiguous(qa, sa, qb, sb, mi, None, D)
    elif kind == "masked":
        NK = wl.MASKED_NK[args.masked_index]
        w = wl.masked(N=NK[0], K=NK[1], shape=args.masked_index)
        A = put(w.A)
        qb, sb = dg.dg_quantize_fp8(put(w.B), dg.DG_QUANT_BLOCK_128x128)
        mm = put(w.masked_m)
        qa = torch.empty(A.shape, dtype=torch.uint8, device=dev)
        sa = torch.zeros((w.G, w.K // 128, (w.max_m + 3) // 4 * 4), dtype=torch.float32, device=dev)
        D = torch.empty((w.G, w.max_m, w.N), dtype=torch.bfloat16, device=dev)
        tot = float(np.sum(w.masked_m))
        flops = 2.0 * w.N * w.K * tot
        algo_bytes = w.G * w.N * w.K + tot * (w.K + 2 * w.N)
        bound = "hbm"
        cfg = {"workload": "m_grouped_masked", "G": w.G, "max_m": w.max_m, "N": w.N, "K": w.K,
               "sum_masked_m": int(tot)}

        def quant():
            dg.dg_quantize_fp8(A, dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)

        def gemm():
            dg.dg_m_grouped_fp8_gemm_nt_masked(qa, sa, qb, sb, mm, D)
    else:
        w = wl.k_grouped()
        A, B = put(w.A), put(w.B)
        qa = torch.empty(A.shape, dtype=torch.uint8, device=dev)
        qb = torch.empty(B.shape, dtype=torch.uint8, device=dev)
        sa = torch.empty((w.sumK // 128, w.M), dtype=torch.float32, device=dev)
        sb = torch.empty((w.sumK // 128, w.N), dtype=torch.float32, device=dev)
        C = put(w.C)
        D = torch.empty_like(C)
        flops = 2.0 * w.M * w.N * w.sumK
        algo_bytes = w.sumK * (w.M + w.N) + 2 * C.numel() * 4
        bound = "tensor"
        cfg = {"workload": "k_grouped_tn_contiguous", "G": w.G, "M": w.M, "N": w.N,
               "ks": [int(k) for k in w.ks]}

        def quant():
            dg.dg_quantize_fp8(A, dg.DG_QUANT_COL_128x1, codes=qa, scales=sa)
            dg.dg_quantize_fp8(B, dg.DG_QUANT_COL_128x1, codes=qb, scales=sb)

        def gemm():
            dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, w.ks, C, D)
    torch.cuda.synchronize()

    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(max(args.warmup, 3)):
        quant()
        gemm()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    launches0 = dg.dg_get_launch_count()
    wall0 = time.time()
    e[0].record()
    for _ in range(args.steps):
        quant()
        gemm()
    e[1].record()
    torch.cuda.synchronize()
    wall1 = time.time()
    launches = dg.dg_get_launch_count() - launches0
    clocks = sampler.stop(wall0, wall1)
    ms_step = e[0].elapsed_time(e[1]) / args.steps
    # GEMM alone (launch-averaged over the same number of launches)
    e[0].record()
    for _ in range(args.steps):
        gemm()
    e[1].record()
    torch.cuda.synchronize()
    ms_gemm = e[0].elapsed_time(e[1]) / args.steps
    if bound == "tensor":
        ach = flops / (ms_gemm * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4), "traffic": None}
    else:
        ach = algo_bytes / (ms_gemm * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4), "traffic": None}
    line = {"metric": METRIC, "value": round(flops / (ms_step * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": round(ms_step, 4), "gemm_ms": round(ms_gemm, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 x e4m3 -> f32 accumulate", "data": "synthetic (seeded N(0,1))",
            "config": dict(cfg, l2="inputs larger than L2, no flush"), "roofline": roof,
            "gpu_launches": int(launches), "clocks": clocks,
            "algorithmic_bytes_per_launch": int(algo_bytes), "flops_per_step": flops}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- UE8M0 comparison
def run_ue8m0(args):
    """--workload ue8m0: the dense sweep with power-of-two scales, timing the
    two GEMM paths on the same quantised inputs: explicit promotion
    (dg_fp8_gemm_nt, FP32 copies of the scales) and the tensor core's
    block-scaled MMA (dg_fp8_gemm_nt_ue8m0, packed UE8M0). One step = per
    shape, quantise A (power-of-two 1x128) + the block-scaled GEMM; L2 flushed
    before every shape as in the main line. One GPU."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    shapes = wl.dense_shapes()
    if args.shape:
        shapes = [tuple(int(x) for x in sh.split(",")) for sh in args.shape.split(";") if sh]
    weights, acts, outs, qbufs = {}, [], [], []
    for (N, K) in sorted(set((s_[1], s_[2]) for s_ in shapes)):
        B = torch.from_numpy(synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))).to(dev)
        weights[(N, K)] = dg.dg_quantize_fp8_ue8m0(B, dg.DG_QUANT_BLOCK_128x128)
        del B
    for (M, N, K) in shapes:
        A = torch.from_numpy(synth.normal((M, K), synth.seed(2, shape_index(M, N, K), 0))).to(dev)
        acts.append(A)
        outs.append(torch.empty((M, N), dtype=torch.bfloat16, device=dev))
        qbufs.append(dg.dg_quantize_fp8_ue8m0(A, dg.DG_QUANT_ROW_1x128))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    n = len(shapes)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]

    def run(kind, record):
        for i, (M, N, K) in enumerate(shapes):
            flush.fill_(i & 0xFF)
            torch.cuda._sleep(100_000)
            qa, sa, pa = qbufs[i]
            qb, sb, pb = weights[(N, K)]
            if record:
                ev[i][0].record()
            if kind == "step":
                dg.dg_quantize_fp8_ue8m0(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa,
                                         packed=pa)
                dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, outs[i])
            elif kind == "mx":
                dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, outs[i])
            else:
                dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, outs[i])
            if record:
                ev[i][1].record()

    res = {}
    for kind in ("step", "mx", "promotion"):
        for _ in range(max(args.warmup, 3)):
            run(kind, False)
        torch.cuda.synchronize()
        t = np.zeros(n)
        for _ in range(args.steps):
            run(kind, True)
            torch.cuda.synchronize()
            for i in range(n):
                t[i] += ev[i][0].elapsed_time(ev[i][1])
        res[kind] = t / args.steps
    flops = [shape_flops(*sh) for sh in shapes]
    big = max(range(n), key=lambda i: flops[i])
    per = [{"M": M, "N": N, "K": K, "mx_us": round(res["mx"][i] * 1e3, 2),
            "promotion_us": round(res["promotion"][i] * 1e3, 2),
            "mx_tflops": round(flops[i] / (res["mx"][i] * 1e-3) / 1e12, 1),
            "promotion_tflops": round(flops[i] / (res["promotion"][i] * 1e-3) / 1e12, 1)}
           for i, (M, N, K) in enumerate(shapes)]
    ach = flops[big] / (res["mx"][big] * 1e-3) / 1e12
    line = {"metric": METRIC, "workload": "dense_fp8_gemm_nt_sweep_ue8m0",
            "value": round(sum(flops) / (res["step"].sum() * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(float(res["step"].sum()), 4), "steps": args.steps,
            "higher_is_better": True, "dtype": "e4m3 x e4m3 (UE8M0 scales) -> f32 accumulate, bf16 out",
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4),
                         "kernel": f"gemm_mx_kernel:{shapes[big][0]}x{shapes[big][1]}x{shapes[big][2]}"},
            "promotion_path_same_scales_tflops": round(
                sum(flops) / (res["promotion"].sum() * 1e-3) / 1e12, 2),
            "mx_path_gemm_only_tflops": round(sum(flops) / (res["mx"].sum() * 1e-3) / 1e12, 2),
            "shapes": per}
    print(json.dumps(line), flush=True)
    return 0


def run_fp8fp4(args):
    """--workload fp8fp4: the dense sweep with E2M1 (FP4) weights, one
    power-of-two scale per 1x32 K-strip, against E4M3 activations with
    power-of-two 1x128 scales, on the block-scaled MMA. One step = per shape,
    quantise A + the FP8 x FP4 GEMM; the FP8 x FP8 block-scaled GEMM on the
    same activations is timed beside it. L2 flushed before every shape. One GPU."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    shapes = wl.dense_shapes()
    if args.shape:
        shapes = [tuple(int(x) for x in sh.split(",")) for sh in args.shape.split(";") if sh]
    w4, w8, acts, outs, qbufs = {}, {}, [], [], []
    for (N, K) in sorted(set((s_[1], s_[2]) for s_ in shapes)):
        B = torch.from_numpy(synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))).to(dev)
        w4[(N, K)] = dg.dg_quantize_fp4_e2m1(B, with_scales=False)
        w8[(N, K)] = dg.dg_quantize_fp8_ue8m0(B, dg.DG_QUANT_BLOCK_128x128, with_scales=False)
        del B
    for (M, N, K) in shapes:
        A = torch.from_numpy(synth.normal((M, K), synth.seed(2, shape_index(M, N, K), 0))).to(dev)
        acts.append(A)
        outs.append(torch.empty((M, N), dtype=torch.bfloat16, device=dev))
        qbufs.append(dg.dg_quantize_fp8_ue8m0(A, dg.DG_QUANT_ROW_1x128, with_scales=False))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    n = len(shapes)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]

    def run(kind, record):
        for i, (M, N, K) in enumerate(shapes):
            flush.fill_(i & 0xFF)
            torch.cuda._sleep(100_000)
            qa, _, pa = qbufs[i]
            if record:
                ev[i][0].record()
            if kind == "step":
                dg.dg_quantize_fp8_ue8m0(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, packed=pa,
                                         with_scales=False)
            if kind in ("step", "fp4"):
                qb, _, pb = w4[(N, K)]
                dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, outs[i])
            else:
                qb, _, pb = w8[(N, K)]
                dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, outs[i])
            if record:
                ev[i][1].record()

    res = {}
    for kind in ("step", "fp4", "fp8"):
        for _ in range(max(args.warmup, 3)):
            run(kind, False)
        torch.cuda.synchronize()
        t = np.zeros(n)
        for _ in range(args.steps):
            run(kind, True)
            torch.cuda.synchronize()
            for i in range(n):
                t[i] += ev[i][0].elapsed_time(ev[i][1])
        res[kind] = t / args.steps
    flops = [shape_flops(*sh) for sh in shapes]
    # algorithmic bytes with FP4 weights: A + B/2 + scales (A 1 per 128, B 1 per 32) + D
    nbytes = [M * K + N * K // 2 + M * (K // 128) + N * (K // 32) + 2 * M * N
              for (M, N, K) in shapes]
    big = max(range(n), key=lambda i: flops[i])
    per = [{"M": M, "N": N, "K": K, "fp4_us": round(res["fp4"][i] * 1e3, 2),
            "fp8_mx_us": round(res["fp8"][i] * 1e3, 2),
            "fp4_tflops": round(flops[i] / (res["fp4"][i] * 1e-3) / 1e12, 1),
            "fp4_gbs": round(nbytes[i] / (res["fp4"][i] * 1e-3) / 1e9, 1),
            "fp8_mx_tflops": round(flops[i] / (res["fp8"][i] * 1e-3) / 1e12, 1)}
           for i, (M, N, K) in enumerate(shapes)]
    ach = flops[big] / (res["fp4"][big] * 1e-3) / 1e12
    line = {"metric": METRIC, "workload": "dense_fp8_fp4_gemm_nt_sweep",
            "value": round(sum(flops) / (res["step"].sum() * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(float(res["step"].sum()), 4), "steps": args.steps,
            "higher_is_better": True,
            "dtype": "e4m3 x e2m1 (UE8M0 scales, 1x128 / 1x32) -> f32 accumulate, bf16 out",
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4),
                         "kernel": f"gemm_mx_kernel<FP4B>:{shapes[big][0]}x{shapes[big][1]}x{shapes[big][2]}",
                         "peak_note": "FP8 x FP4 on kind::mxf8f6f4 runs at the FP8 rate"},
            "fp4_gemm_only_tflops": round(sum(flops) / (res["fp4"].sum() * 1e-3) / 1e12, 2),
            "fp8_mx_gemm_only_tflops": round(sum(flops) / (res["fp8"].sum() * 1e-3) / 1e12, 2),
            "shapes": per}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- ranks
def max_over_ranks(dist, values, device):
    """Element-wise maximum of per-rank timings (ms); every rank calls it in
    the same order. Identity on one process (dist None)."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_tflops(world, flops_per_rank_step, ms_per_step):
    """Whole-job throughput of `world` replicas that each do
    `flops_per_rank_step` per step, timed by the slowest rank."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ----------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import moe_grouped_gemm_07_b200 as dg

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    shapes = wl.dense_shapes()
    if args.shape:
        shapes = [tuple(int(x) for x in sh.split(",")) for sh in args.shape.split(";") if sh]

    # ---- set-up: weights quantised once, activations resident in HBM
    weights = {}
    for (N, K) in sorted(set((s_[1], s_[2]) for s_ in shapes)):
        B = torch.from_numpy(synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))).to(device)
        weights[(N, K)] = dg.dg_quantize_fp8(B, dg.DG_QUANT_BLOCK_128x128)
        del B
    acts, outs, qbufs = [], [], []
    for i, (M, N, K) in enumerate(shapes):
        A = torch.from_numpy(synth.normal((M, K), synth.seed(2, shape_index(M, N, K), 0))).to(device)
        acts.append(A)
        outs.append(torch.empty((M, N), dtype=torch.bfloat16, device=device))
        qbufs.append((torch.empty((M, K), dtype=torch.uint8, device=device),
                      torch.zeros((K // 128, (M + 3) // 4 * 4), dtype=torch.float32,
                                  device=device)))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()

    n = len(shapes)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]

    def step(record=False, split=False):
        """One pass over the shapes. record: events around each shape's
        quantise + GEMM pair (the step time); split: one more event between
        the two kernels (per-kernel times; this can block the overlap of the
        GEMM's prologue with the quantiser, so it is a separate pass)."""
        for i, (M, N, K) in enumerate(shapes):
            flush.fill_(i & 0xFF)
            # ~50 us device spin (outside the per-shape events) so the host has
            # queued the timed launches before the device reaches them: the
            # events then bracket kernel time, not host submission gaps
            torch.cuda._sleep(100_000)
            if record:
                ev[i][0].record()
            qa, sa = qbufs[i]
            dg.dg_quantize_fp8(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)
            if split:
                ev[i][1].record()
            qb, sb = weights[(N, K)]
            dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, outs[i])
            if record:
                ev[i][2].record()

    sampler = None if args.quick else ClockSampler(local)
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()

    # ---- timed region (device-resident inputs)
    t_q = np.zeros(n)
    t_g = np.zeros(n)
    launches0 = dg.dg_get_launch_count()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    outer0 = torch.cuda.Event(enable_timing=True)
    outer1 = torch.cuda.Event(enable_timing=True)
    t_pair = np.zeros(n)
    outer0.record()
    for _ in range(args.steps):
        step(record=True)
        torch.cuda.synchronize()
        for i in range(n):
            t_pair[i] += ev[i][0].elapsed_time(ev[i][2])
    outer1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    wall1 = time.time()
    launches = dg.dg_get_launch_count() - launches0
    clocks = sampler.stop(wall0, wall1) if sampler else None
    t_pair /= args.steps
    ms_step = float(np.sum(t_pair))
    # per-kernel split (separate, untimed-for-value pass)
    split_steps = max(1, min(args.steps, 20))
    for _ in range(split_steps):
        step(record=True, split=True)
        torch.cuda.synchronize()
        for i in range(n):
            t_q[i] += ev[i][0].elapsed_time(ev[i][1])
            t_g[i] += ev[i][1].elapsed_time(ev[i][2])
    t_q /= split_steps
    t_g /= split_steps
    ms_outer = outer0.elapsed_time(outer1) / args.steps
    ms_step, ms_outer = max_over_ranks(dist, [ms_step, ms_outer], device)

    # ---- end to end through the public API with host buffers
    if args.quick:
        if rank == 0:
            print(json.dumps({"quick": True, "shapes": [list(x) for x in shapes],
                              "gemm_us": [round(x * 1e3, 2) for x in t_g],
                              "pair_us": [round(x * 1e3, 2) for x in t_pair],
                              "quant_us": [round(x * 1e3, 2) for x in t_q]}), flush=True)
        if dist:
            dist.destroy_process_group()
        return 0
    host_a = [torch.from_numpy(synth.normal((M, K), synth.seed(2, shape_index(M, N, K), 0))).pin_memory()
              for i, (M, N, K) in enumerate(shapes)]
    host_d = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for (M, N, K) in shapes]
    h2d = sum(a.numel() * 4 for a in host_a)
    d2h = sum(d.numel() * 2 for d in host_d)

    def e2e_step():
        for i, (M, N, K) in enumerate(shapes):
            acts[i].copy_(host_a[i], non_blocking=True)
            qa, sa = qbufs[i]
            dg.dg_quantize_fp8(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)
            qb, sb = weights[(N, K)]
            dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, outs[i])
            host_d[i].copy_(outs[i], non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 10))
    if dist:
        dist.barrier()
    e0.record()
    for _ in range(e2e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / e2e_steps
    ms_e2e, = max_over_ranks(dist, [ms_e2e], device)

    flops_step = sum(shape_flops(*s) for s in shapes)
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]  # nominal FP8:BF16 dense ratio is 2
    per_shape = []
    for i, (M, N, K) in enumerate(shapes):
        tf = shape_flops(M, N, K) / (t_g[i] * 1e-3) / 1e12
        gbs = shape_bytes(M, N, K) / (t_g[i] * 1e-3) / 1e9
        roof_ms = max(shape_flops(M, N, K) / (fp8_peak * 1e12),
                      shape_bytes(M, N, K) / (pk["hbm_gbs"] * 1e9)) * 1e3
        per_shape.append({"M": M, "N": N, "K": K, "step_us": round(t_pair[i] * 1e3, 2),
                          "gemm_us": round(t_g[i] * 1e3, 2),
                          "quant_us": round(t_q[i] * 1e3, 2), "tflops": round(tf, 1),
                          "gbs": round(gbs, 1), "roofline_frac": round(roof_ms / t_g[i], 3)})
    # dominant kernel: the GEMM on its largest shape
    big = max(range(n), key=lambda i: t_g[i])
    Mb, Nb, Kb = shapes[big]
    ach = shape_flops(Mb, Nb, Kb) / (t_g[big] * 1e-3) / 1e12
    key = f"gemm_fp8_kernel:{Mb}x{Nb}x{Kb}"
    roofline = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4),
                "traffic": traffic_from_profile(key),
                "kernel": key,
                "peak_note": f"FP8 dense = 2 x {pk['source']} bf16 burst "
                             f"({pk['bf16_tflops']} TF/s); nominal FP8 {NOMINAL_FP8_TFLOPS} TF/s"}
    dec = [i for i, s in enumerate(shapes) if s[0] <= 128]
    dec_bytes = sum(shape_bytes(*shapes[i]) for i in dec)
    dec_ms = float(sum(t_g[i] for i in dec))
    roofline_hbm = {"bound": "hbm", "achieved": round(dec_bytes / (dec_ms * 1e-3) / 1e9, 1),
                    "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": round(dec_bytes / (dec_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                    "shapes": "M in {64,128} (12 decode shapes), GEMM kernel only"}

    line = {
        "metric": METRIC, "value": round(job_tflops(world, flops_step, ms_step), 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 accumulate, bf16 out",
        "data": "synthetic (seeded N(0,1) float32, quantised on the GPU)",
        "config": {"workload": WORKLOAD, "shapes": n, "M": list(wl.DENSE_M),
                   "NK": [list(x) for x in wl.DENSE_NK],
                   "step": "per shape: quantise A (1x128) + GEMM; B pre-quantised (128x128)",
                   "l2": "flushed (256 MiB write) before every shape, flush excluded from timing",
                   "host_gap": "a ~50 us device spin precedes each shape so events time kernels only",
                   "parallelism": f"replicas x{world}"},
        "ms_per_step_incl_flush": round(ms_outer, 4),
        "fp8_pct_of_measured_peak": round(100 * flops_step / (ms_step * 1e-3) / 1e12 / fp8_peak, 2),
        "fp8_pct_of_nominal_peak": round(100 * flops_step / (ms_step * 1e-3) / 1e12
                                         / NOMINAL_FP8_TFLOPS, 2),
        "roofline": roofline, "roofline_hbm": roofline_hbm,
        "e2e": {"value": round(job_tflops(world, flops_step, ms_e2e), 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e, 3)},
        "gpu_launches": int(launches), "gpu_launches_per_step": int(launches // max(args.steps, 1)),
        "clocks": clocks, "shapes": per_shape,
    }
    if rank == 0 and not args.no_cpu_baseline:
        rows = args.cpu_rows
        inputs = prepare_oracle_inputs(shapes, rows)
        f, s, cores = oracle_sample(shapes, rows, inputs)
        line["cpu_baseline"] = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"{rows} rows of each of the 18 shapes (A rows "
                                          f"quantised + those rows of D), weights pre-quantised; "
                                          f"{s:.1f} s"}
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=1024)
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shape", default="",
                    help="M,N,K[;M,N,K...]: time only these shapes (profiling)")
    ap.add_argument("--quick", action="store_true",
                    help="timed device loop only: no e2e leg, CPU baseline or clock sampling")
    ap.add_argument("--workload", default="dense",
                    choices=["dense", "contiguous", "masked", "kgrouped", "ue8m0", "fp8fp4"],
                    help="dense (the bench line) or one MoE variant at its benchmark size")
    ap.add_argument("--masked-index", type=int, default=0,
                    help="masked workload: index into the (N, K) pairs")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "fp8fp4":
        return run_fp8fp4(args)
    if args.workload == "ue8m0":
        return run_ue8m0(args)
    if args.workload != "dense":
        return run_grouped(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

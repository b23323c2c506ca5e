"""Benchmark: FP8 fine-grained-scaled GEMM on B200 (dense NT projection sweep).

Workload (the dense sweep the pages' headline numbers are quoted on): M in
{64, 128, 4096} x (N, K) in {(2112,7168), (24576,1536), (32768,512),
(7168,16384), (4096,7168), (7168,2048)}; A, B ~ N(0,1) float32 from seeded
streams. Weights B are quantised once at set-up (128x128 blocks, static FP8
weights). One step = for every shape: quantise A (1x128 strips) on the GPU and
run D = A @ B.T (BF16 out), i.e. the whole hot path per shape. K steps run back
to back between two CUDA events; one step streams several GB, so every shape's
operands have left the 126 MB L2 before the shape comes around again (inputs
larger than L2, no flush).

Reported (one JSON line, rank 0):
  value        whole-job TFLOP/s = sum of GEMM FLOPs / device time of a step
  e2e          same metric through the public API with the activations copied
               from pinned host memory and D copied back inside the timed loop
  roofline     dominant kernel (the GEMM on its largest shape): achieved TFLOP/s
               vs the measured-derived FP8 peak, from CUDA events around that
               GEMM inside full steps (its back-to-back time alone beside it);
               roofline_hbm: the
               same for the decode shapes (M <= 128) against HBM bandwidth,
               launches back to back over rotating weight copies (>= 3x L2),
               with the single-launch-after-a-flush figure beside it
  shapes       per shape: GEMM, quantiser and pair launch durations, and the
               isolated single-launch GEMM time
  moe          (one GPU) the MoE workloads: contiguous, masked (two weight
               shapes), K-grouped -- quantise + grouped GEMM steps
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
    """Hash of the dominant kernel's sources: the tile kernel, its PTX helpers
    and the host code that plans and launches it (a recorded DRAM traffic is
    void once any of them changes)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_grouped_gemm_07_b200", "csrc")
    for f in ("dg_api.cu", "gemm.cuh", "ptx.cuh"):
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
L2_BYTES = 126 << 20


def n_copies(nbytes, min_copies=1):
    """Rotating copies so that consecutive launches never find their operand
    in L2: the copies together span at least three times the L2."""
    return max(min_copies, -(-3 * L2_BYTES // max(1, int(nbytes))))


def time_batch(fn, reps, warm=2, graph=False):
    """Average device time (ms) of one call of fn(i) over `reps` calls issued
    back to back on the current stream, CUDA events around the batch. With
    graph=True the batch is captured once into a CUDA graph and the events
    bracket one replay, so the host's per-call cost (Python, argument
    marshalling) cannot starve the device of short kernels."""
    import torch
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(reps):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / reps
    torch.cuda._sleep(200_000)  # the host queues the batch while the device spins
    e0.record()
    for i in range(reps):
        fn(i)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def moe_workload(kind, dev, masked_index=0):
    """Builds one MoE workload at its benchmark size (synth inputs, weights
    quantised once) and returns (quant, gemm, info): quant() quantises the
    activations, gemm() runs the grouped GEMM, info holds FLOPs, algorithmic
    bytes, bound and config."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

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
        info = {"flops": 2.0 * w.N * w.K * float(sum(w.rows)),
                "bytes": w.Mt * w.K + w.G * w.N * w.K + 2 * w.Mt * w.N, "bound": "tensor",
                "config": {"workload": "m_grouped_contiguous", "G": w.G, "N": w.N, "K": w.K,
                           "Mt": w.Mt, "rows": [int(r) for r in w.rows]}}

        def quant():
            dg.dg_quantize_fp8(A, dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)

        def gemm():
            dg.dg_m_grouped_fp8_gemm_nt_contiguous(qa, sa, qb, sb, mi, None, D)
    elif kind == "masked":
        NK = wl.MASKED_NK[masked_index]
        w = wl.masked(N=NK[0], K=NK[1], shape=masked_index)
        A = put(w.A)
        qb, sb = dg.dg_quantize_fp8(put(w.B), dg.DG_QUANT_BLOCK_128x128)
        mm = put(w.masked_m)
        qa = torch.empty(A.shape, dtype=torch.uint8, device=dev)
        sa = torch.zeros((w.G, w.K // 128, (w.max_m + 3) // 4 * 4), dtype=torch.float32, device=dev)
        D = torch.empty((w.G, w.max_m, w.N), dtype=torch.bfloat16, device=dev)
        tot = float(np.sum(w.masked_m))
        info = {"flops": 2.0 * w.N * w.K * tot,
                "bytes": w.G * w.N * w.K + tot * (w.K + 2 * w.N), "bound": "hbm",
                "config": {"workload": "m_grouped_masked", "G": w.G, "max_m": w.max_m, "N": w.N,
                           "K": w.K, "sum_masked_m": int(tot)}}

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
        info = {"flops": 2.0 * w.M * w.N * w.sumK,
                "bytes": w.sumK * (w.M + w.N) + 2 * C.numel() * 4, "bound": "tensor",
                "config": {"workload": "k_grouped_tn_contiguous", "G": w.G, "M": w.M, "N": w.N,
                           "ks": [int(k) for k in w.ks]}}

        def quant():
            dg.dg_quantize_fp8(A, dg.DG_QUANT_COL_128x1, codes=qa, scales=sa)
            dg.dg_quantize_fp8(B, dg.DG_QUANT_COL_128x1, codes=qb, scales=sb)

        def gemm():
            dg.dg_k_grouped_fp8_gemm_tn_contiguous(qa, sa, qb, sb, w.ks, C, D)
    torch.cuda.synchronize()
    return quant, gemm, info


def measure_moe(kind, dev, steps, warmup, pk, masked_index=0):
    """One MoE workload: step = quantise the activations + the grouped GEMM,
    run back to back `steps` times (every operand is larger than L2, so no
    flush is needed); the GEMM alone is timed the same way. Returns a dict."""
    import torch
    fp8_peak = 2.0 * pk["bf16_tflops"]
    quant, gemm, info = moe_workload(kind, dev, masked_index)

    def pair(_):
        quant()
        gemm()
    ms_step = time_batch(pair, steps, warm=max(warmup, 3))
    ms_gemm = time_batch(lambda _: gemm(), steps, warm=2)
    if info["bound"] == "tensor":
        ach = info["flops"] / (ms_gemm * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4)}
    else:
        ach = info["bytes"] / (ms_gemm * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4)}
    out = {"step_ms": round(ms_step, 4), "gemm_ms": round(ms_gemm, 4),
           "step_tflops": round(info["flops"] / (ms_step * 1e-3) / 1e12, 1),
           "gemm_tflops": round(info["flops"] / (ms_gemm * 1e-3) / 1e12, 1),
           "gemm_gbs": round(info["bytes"] / (ms_gemm * 1e-3) / 1e9, 1),
           "algorithmic_bytes": int(info["bytes"]), "flops": info["flops"],
           "roofline": roof, "config": info["config"]}
    del quant, gemm
    torch.cuda.empty_cache()
    return out


def run_grouped(args):
    """--workload contiguous | masked | kgrouped: one MoE variant at its
    benchmark size (the default run reports all of them beside the dense
    line). value = useful TFLOP/s of the quantise + GEMM step; one GPU."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk = peaks()
    sampler = ClockSampler(dev.index)
    launches0 = dg.dg_get_launch_count()
    wall0 = time.time()
    r = measure_moe(args.workload, dev, args.steps, args.warmup, pk, args.masked_index)
    wall1 = time.time()
    clocks = sampler.stop(wall0, wall1)
    line = {"metric": METRIC, "value": r["step_tflops"], "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": r["step_ms"],
            "gemm_ms": r["gemm_ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 accumulate",
            "data": "synthetic (seeded N(0,1))",
            "config": dict(r["config"], l2="inputs larger than L2, steps back to back, no flush"),
            "roofline": r["roofline"], "gpu_launches": int(dg.dg_get_launch_count() - launches0),
            "clocks": clocks, "algorithmic_bytes_per_launch": r["algorithmic_bytes"],
            "flops_per_step": r["flops"]}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- operand layouts
def run_layouts(args):
    """--workload layouts: the dense GEMM in its four operand layouts (NT, NN,
    TN, TT) at M in {64, 128, 4096} on three weight shapes (N = 2112 has a
    ragged last 128x128 block of B in the NN / TN storage), GEMM launches back
    to back over rotating weight copies (>= 3x L2) in a CUDA graph. NT routes
    M <= 128 to the swap-AB decode kernel; NN / TN / TT run the persistent
    kernel at every M. One GPU."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    fns = {"nt": dg.dg_fp8_gemm_nt, "nn": dg.dg_fp8_gemm_nn, "tn": dg.dg_fp8_gemm_tn,
           "tt": dg.dg_fp8_gemm_tt}
    rows = []
    for (N, K) in ((7168, 16384), (4096, 7168), (2112, 7168)):
        Bf = torch.from_numpy(synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))).to(dev)
        for layout in ("nt", "nn", "tn", "tt"):
            b_mn = layout[1] == "n"
            src = Bf.t().contiguous() if b_mn else Bf
            qb, sb = dg.dg_quantize_fp8(src, dg.DG_QUANT_BLOCK_128x128)
            del src
            qbs = [qb] + [qb.clone() for _ in range(n_copies(N * K, 2) - 1)]
            for M in (64, 128, 4096):
                a_mn = layout[0] == "t"
                Af = torch.from_numpy(synth.normal((M, K), synth.seed(2, shape_index(M, N, K), 0))).to(dev)
                A = Af.t().contiguous() if a_mn else Af
                qa, sa = dg.dg_quantize_fp8(
                    A, dg.DG_QUANT_COL_128x1 if a_mn else dg.DG_QUANT_ROW_1x128)
                Ds = [torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                      for _ in range(min(len(qbs), n_copies(2 * M * N, 1)))]
                reps = 16 if M <= 128 else 4
                fn = fns[layout]
                ms = time_batch(lambda j: fn(qa, sa, qbs[j % len(qbs)], sb, None,
                                             Ds[j % len(Ds)]), reps, graph=True)
                roof_ms = max(shape_flops(M, N, K) / (fp8_peak * 1e12),
                              shape_bytes(M, N, K) / (pk["hbm_gbs"] * 1e9)) * 1e3
                rows.append({"layout": layout, "M": M, "N": N, "K": K,
                             "gemm_us": round(ms * 1e3, 2),
                             "tflops": round(shape_flops(M, N, K) / (ms * 1e-3) / 1e12, 1),
                             "gbs": round(shape_bytes(M, N, K) / (ms * 1e-3) / 1e9, 1),
                             "roofline_frac": round(roof_ms / ms, 3)})
                del Af, A, qa, sa, Ds
            del qbs, qb, sb
            torch.cuda.empty_cache()
    print(json.dumps({"metric": METRIC, "workload": "dense_fp8_gemm_layouts",
                      "timing": "GEMM launches back to back in a CUDA graph over rotating "
                                "weight copies (>= 3x L2)", "shapes": rows}), flush=True)
    return 0


# ----------------------------------------------------------------- UE8M0 comparison
def _sweep_inputs(dev, shapes, quant_w, quant_a):
    """Seeded weights (quantised once, rotating copies of the codes spanning
    at least three times the L2) and activations for a dense sweep."""
    import torch
    weights, acts, outs, qbufs = {}, [], [], []
    for (N, K) in sorted(set((s_[1], s_[2]) for s_ in shapes)):
        B = torch.from_numpy(synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))).to(dev)
        qb, sb, pb = quant_w(B)
        del B
        weights[(N, K)] = ([qb] + [qb.clone() for _ in range(n_copies(qb.numel(), 2) - 1)], sb, pb)
    for (M, N, K) in shapes:
        A = torch.from_numpy(synth.normal((M, K), synth.seed(2, shape_index(M, N, K), 0))).to(dev)
        acts.append(A)
        outs.append(torch.empty((M, N), dtype=torch.bfloat16, device=dev))
        qbufs.append(quant_a(A))
    torch.cuda.synchronize()
    return weights, acts, outs, qbufs


def batch_reps(shape):
    """Launches per timed CUDA-graph batch of one GEMM shape."""
    return 32 if shape[0] <= 128 else 8


def _time_steps(step, steps, warmup):
    """Average ms of one step over `steps` steps issued back to back between
    two CUDA events, after `warmup` untimed steps."""
    import torch
    for j in range(max(warmup, 3)):
        step(j)
    torch.cuda.synchronize()
    torch.cuda._sleep(200_000)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for j in range(steps):
        step(j)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_ue8m0(args):
    """--workload ue8m0: the dense sweep with power-of-two scales, timing the
    two GEMM paths on the same quantised inputs: explicit promotion
    (dg_fp8_gemm_nt, FP32 copies of the scales) and the tensor core's
    block-scaled MMA (dg_fp8_gemm_nt_ue8m0, packed UE8M0). One step = per
    shape, quantise A (power-of-two 1x128) + the block-scaled GEMM, steps
    back to back as in the main line; each GEMM is also timed alone, launches
    back to back in a CUDA graph over rotating weight copies. One GPU."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    shapes = wl.dense_shapes()
    if args.shape:
        shapes = [tuple(int(x) for x in sh.split(",")) for sh in args.shape.split(";") if sh]
    weights, acts, outs, qbufs = _sweep_inputs(
        dev, shapes, lambda B: dg.dg_quantize_fp8_ue8m0(B, dg.DG_QUANT_BLOCK_128x128),
        lambda A: dg.dg_quantize_fp8_ue8m0(A, dg.DG_QUANT_ROW_1x128))
    n = len(shapes)

    def gemm(kind, i, j):
        M, N, K = shapes[i]
        qa, sa, pa = qbufs[i]
        qbs, sb, pb = weights[(N, K)]
        qb = qbs[j % len(qbs)]
        if kind == "mx":
            dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, outs[i])
        else:
            dg.dg_fp8_gemm_nt(qa, sa, qb, sb, None, outs[i])

    def step(j):
        for i in range(n):
            qa, sa, pa = qbufs[i]
            dg.dg_quantize_fp8_ue8m0(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa, packed=pa)
            gemm("mx", i, j)

    ms_step = _time_steps(step, args.steps, args.warmup)
    res = {kind: np.array([time_batch(lambda j, i=i: gemm(kind, i, j), batch_reps(shapes[i]),
                                      graph=True) for i in range(n)])
           for kind in ("mx", "promotion")}
    flops = [shape_flops(*sh) for sh in shapes]
    big = max(range(n), key=lambda i: flops[i])
    per = [{"M": M, "N": N, "K": K, "mx_us": round(res["mx"][i] * 1e3, 2),
            "promotion_us": round(res["promotion"][i] * 1e3, 2),
            "mx_tflops": round(flops[i] / (res["mx"][i] * 1e-3) / 1e12, 1),
            "promotion_tflops": round(flops[i] / (res["promotion"][i] * 1e-3) / 1e12, 1)}
           for i, (M, N, K) in enumerate(shapes)]
    ach = flops[big] / (res["mx"][big] * 1e-3) / 1e12
    line = {"metric": METRIC, "workload": "dense_fp8_gemm_nt_sweep_ue8m0",
            "value": round(sum(flops) / (ms_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms_step, 4), "steps": args.steps,
            "higher_is_better": True, "dtype": "e4m3 x e4m3 (UE8M0 scales) -> f32 accumulate, bf16 out",
            "timing": "step: K steps back to back; per shape: GEMM launches back to back in a "
                      "CUDA graph over rotating weight copies (>= 3x L2)",
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
    quantise A + the FP8 x FP4 GEMM, steps back to back; each GEMM (and the
    FP8 x FP8 block-scaled GEMM on the same activations) is also timed alone,
    launches back to back in a CUDA graph over rotating weight copies. One GPU."""
    import torch
    import moe_grouped_gemm_07_b200 as dg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    shapes = wl.dense_shapes()
    if args.shape:
        shapes = [tuple(int(x) for x in sh.split(",")) for sh in args.shape.split(";") if sh]
    w4, acts, outs, qbufs = _sweep_inputs(
        dev, shapes, lambda B: dg.dg_quantize_fp4_e2m1(B, with_scales=False),
        lambda A: dg.dg_quantize_fp8_ue8m0(A, dg.DG_QUANT_ROW_1x128, with_scales=False))
    w8 = {}
    for (N, K) in w4:  # FP8 weights of the same matrices, for the comparison
        B = torch.from_numpy(synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))).to(dev)
        qb, sb, pb = dg.dg_quantize_fp8_ue8m0(B, dg.DG_QUANT_BLOCK_128x128, with_scales=False)
        del B
        w8[(N, K)] = ([qb] + [qb.clone() for _ in range(n_copies(qb.numel(), 2) - 1)], sb, pb)
    torch.cuda.synchronize()
    n = len(shapes)

    def gemm(kind, i, j):
        M, N, K = shapes[i]
        qa, _, pa = qbufs[i]
        qbs, _, pb = (w4 if kind == "fp4" else w8)[(N, K)]
        qb = qbs[j % len(qbs)]
        if kind == "fp4":
            dg.dg_fp8_fp4_gemm_nt(qa, pa, qb, pb, None, outs[i])
        else:
            dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, None, outs[i])

    def step(j):
        for i in range(n):
            qa, _, pa = qbufs[i]
            dg.dg_quantize_fp8_ue8m0(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, packed=pa,
                                     with_scales=False)
            gemm("fp4", i, j)

    ms_step = _time_steps(step, args.steps, args.warmup)
    res = {kind: np.array([time_batch(lambda j, i=i: gemm(kind, i, j), batch_reps(shapes[i]),
                                      graph=True) for i in range(n)])
           for kind in ("fp4", "fp8")}
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
            "value": round(sum(flops) / (ms_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms_step, 4), "steps": args.steps,
            "higher_is_better": True,
            "dtype": "e4m3 x e2m1 (UE8M0 scales, 1x128 / 1x32) -> f32 accumulate, bf16 out",
            "timing": "step: K steps back to back; per shape: GEMM launches back to back in a "
                      "CUDA graph over rotating weight copies (>= 3x L2)",
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
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]  # nominal FP8:BF16 dense ratio is 2

    # ---- set-up: weights quantised once (plus rotating copies for the
    # per-kernel batches), activations resident in HBM
    weights = {}
    for (N, K) in sorted(set((s_[1], s_[2]) for s_ in shapes)):
        B = torch.from_numpy(synth.normal((N, K), synth.seed(2, nk_index(N, K), 1))).to(device)
        qb, sb = dg.dg_quantize_fp8(B, dg.DG_QUANT_BLOCK_128x128)
        del B
        weights[(N, K)] = ([qb] + [qb.clone() for _ in range(n_copies(N * K, 2) - 1)], sb)
    acts, outs, qbufs = [], [], []
    step_bytes = 0
    for i, (M, N, K) in enumerate(shapes):
        A = torch.from_numpy(synth.normal((M, K), synth.seed(2, shape_index(M, N, K), 0))).to(device)
        acts.append(A)
        nd = min(len(weights[(N, K)][0]), n_copies(2 * M * N, 1))
        outs.append([torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(nd)])
        qbufs.append((torch.empty((M, K), dtype=torch.uint8, device=device),
                      torch.zeros((K // 128, (M + 3) // 4 * 4), dtype=torch.float32,
                                  device=device)))
        step_bytes += 4 * M * K + M * K + N * K + 2 * M * N
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()
    n = len(shapes)

    def run_shape(i, copy=0):
        M, N, K = shapes[i]
        qa, sa = qbufs[i]
        qbs, sb = weights[(N, K)]
        dg.dg_quantize_fp8(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)
        dg.dg_fp8_gemm_nt(qa, sa, qbs[copy % len(qbs)], sb, None, outs[i][copy % len(outs[i])])

    def step():
        """One pass of the hot path over the batch: per shape, quantise A
        (1x128) and run the GEMM. Consecutive kernels overlap through PDL."""
        for i in range(n):
            run_shape(i)

    sampler = None if args.quick else ClockSampler(local)
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K whole steps back to back, device-resident inputs.
    # A step streams step_bytes (several GB), so each shape's operands have
    # left L2 before the shape comes around again: no flush is needed.
    launches0 = dg.dg_get_launch_count()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    wall1 = time.time()
    launches = dg.dg_get_launch_count() - launches0
    clocks = sampler.stop(wall0, wall1) if sampler else None
    ms_step = e0.elapsed_time(e1) / args.steps
    ms_step, = max_over_ranks(dist, [ms_step], device)

    # ---- per-kernel launch durations, two ways:
    # (1) in the step: a few more steps with CUDA events around each shape's
    #     GEMM (the events hold the GEMM back from overlapping its
    #     neighbours, so these are not part of the step time);
    # (2) back to back: each kernel launched `reps` times over rotating weight
    #     / output copies (together >= 3x L2, so every launch reads its
    #     weights from DRAM), captured in a CUDA graph, events around a replay
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    t_in = np.zeros(n)
    ctx_steps = max(2, min(args.steps, 10))
    for _ in range(ctx_steps):
        for i in range(n):
            M, N, K = shapes[i]
            qa, sa = qbufs[i]
            qbs, sb = weights[(N, K)]
            dg.dg_quantize_fp8(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa, scales=sa)
            ev[i][0].record()
            dg.dg_fp8_gemm_nt(qa, sa, qbs[0], sb, None, outs[i][0])
            ev[i][1].record()
        torch.cuda.synchronize()
        for i in range(n):
            t_in[i] += ev[i][0].elapsed_time(ev[i][1]) / ctx_steps
    t_g, t_q, t_pair, t_iso = np.zeros(n), np.zeros(n), np.zeros(n), np.zeros(n)
    for i, (M, N, K) in enumerate(shapes):
        qa, sa = qbufs[i]
        qbs, sb = weights[(N, K)]
        reps = batch_reps((M, N, K))
        t_g[i] = time_batch(lambda j: dg.dg_fp8_gemm_nt(qa, sa, qbs[j % len(qbs)], sb, None,
                                                        outs[i][j % len(outs[i])]), reps,
                            graph=True)
        t_q[i] = time_batch(lambda j: dg.dg_quantize_fp8(acts[i], dg.DG_QUANT_ROW_1x128, codes=qa,
                                                         scales=sa), reps, graph=True)
        t_pair[i] = time_batch(lambda j: run_shape(i, j), reps, graph=True)
        # isolated: one launch after a 256 MiB flush write and a device spin
        iso = []
        for j in range(6):
            flush.fill_(j & 0xFF)
            torch.cuda._sleep(100_000)
            e0.record()
            dg.dg_fp8_gemm_nt(qa, sa, qbs[j % len(qbs)], sb, None, outs[i][j % len(outs[i])])
            e1.record()
            torch.cuda.synchronize()
            if j >= 1:
                iso.append(e0.elapsed_time(e1))
        t_iso[i] = float(np.mean(iso))
    t_all = max_over_ranks(dist, list(t_g) + list(t_q) + list(t_pair) + list(t_iso) + list(t_in),
                           device)
    t_g, t_q = np.array(t_all[:n]), np.array(t_all[n:2 * n])
    t_pair, t_iso = np.array(t_all[2 * n:3 * n]), np.array(t_all[3 * n:4 * n])
    t_in = np.array(t_all[4 * n:])

    # ---- end to end through the public API with host buffers
    if args.quick:
        if rank == 0:
            print(json.dumps({"quick": True, "ms_per_step": round(ms_step, 4),
                              "shapes": [list(x) for x in shapes],
                              "gemm_us": [round(x * 1e3, 2) for x in t_g],
                              "pair_us": [round(x * 1e3, 2) for x in t_pair],
                              "quant_us": [round(x * 1e3, 2) for x in t_q],
                              "gemm_isolated_us": [round(x * 1e3, 2) for x in t_iso]}), flush=True)
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
            qbs, sb = weights[(N, K)]
            dg.dg_fp8_gemm_nt(qa, sa, qbs[0], sb, None, outs[i][0])
            host_d[i].copy_(outs[i][0], non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        e2e_step()
    torch.cuda.synchronize()
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

    flops_step = sum(shape_flops(*s_) for s_ in shapes)
    per_shape = []
    for i, (M, N, K) in enumerate(shapes):
        roof_ms = max(shape_flops(M, N, K) / (fp8_peak * 1e12),
                      shape_bytes(M, N, K) / (pk["hbm_gbs"] * 1e9)) * 1e3
        per_shape.append({"M": M, "N": N, "K": K, "gemm_us": round(t_g[i] * 1e3, 2),
                          "gemm_in_step_us": round(t_in[i] * 1e3, 2),
                          "quant_us": round(t_q[i] * 1e3, 2), "pair_us": round(t_pair[i] * 1e3, 2),
                          "gemm_isolated_us": round(t_iso[i] * 1e3, 2),
                          "tflops": round(shape_flops(M, N, K) / (t_g[i] * 1e-3) / 1e12, 1),
                          "gbs": round(shape_bytes(M, N, K) / (t_g[i] * 1e-3) / 1e9, 1),
                          "roofline_frac": round(roof_ms / t_g[i], 3)})
    # dominant kernel: the GEMM on its largest shape, timed in the step
    big = max(range(n), key=lambda i: t_in[i])
    Mb, Nb, Kb = shapes[big]
    ach = shape_flops(Mb, Nb, Kb) / (t_in[big] * 1e-3) / 1e12
    key = f"gemm_fp8_kernel:{Mb}x{Nb}x{Kb}"
    roofline = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4),
                "traffic": traffic_from_profile(key),
                "kernel": key,
                "timing": "CUDA events around this GEMM inside full steps (its neighbours in the "
                          "step are the other shapes' kernels); back to back alone: "
                          f"{t_g[big] * 1e3:.1f} us",
                "peak_note": f"FP8 dense = 2 x {pk['source']} bf16 burst "
                             f"({pk['bf16_tflops']} TF/s); nominal FP8 {NOMINAL_FP8_TFLOPS} TF/s"}
    dec = [i for i, s_ in enumerate(shapes) if s_[0] <= 128]
    roofline_hbm = None
    if dec:
        dec_bytes = sum(shape_bytes(*shapes[i]) for i in dec)
        dec_ms = float(sum(t_g[i] for i in dec))
        dec_iso_ms = float(sum(t_iso[i] for i in dec))
        roofline_hbm = {"bound": "hbm", "achieved": round(dec_bytes / (dec_ms * 1e-3) / 1e9, 1),
                        "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": round(dec_bytes / (dec_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                        "frac_isolated_launch": round(
                            dec_bytes / (dec_iso_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                        "shapes": f"M in {{64,128}} ({len(dec)} decode shapes), GEMM kernel only, "
                                  "average launch duration back to back over rotating weights; "
                                  "frac_isolated_launch: one launch after a flush, events around it"}

    line = {
        "metric": METRIC, "value": round(job_tflops(world, flops_step, ms_step), 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 accumulate, bf16 out",
        "data": "synthetic (seeded N(0,1) float32, quantised on the GPU)",
        "config": {"workload": WORKLOAD, "shapes": n, "M": list(wl.DENSE_M),
                   "NK": [list(x) for x in wl.DENSE_NK],
                   "step": "per shape: quantise A (1x128) + GEMM; B pre-quantised (128x128)",
                   "l2": f"inputs larger than L2: a step streams {step_bytes / 1e9:.2f} GB, so "
                         "every shape's operands leave L2 before it comes around again; no flush",
                   "timing": "K steps back to back between two CUDA events",
                   "parallelism": f"replicas x{world}"},
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
    del weights, outs, flush
    torch.cuda.empty_cache()
    if world == 1 and not args.no_moe:
        moe = {}
        for name, kind, idx in (("contiguous", "contiguous", 0), ("masked_4096x7168", "masked", 0),
                                ("masked_7168x2048", "masked", 1), ("kgrouped", "kgrouped", 0)):
            moe[name] = measure_moe(kind, device, max(3, min(args.steps, 20)), args.warmup, pk, idx)
        line["moe"] = moe
    if rank == 0 and not args.no_cpu_baseline:
        rows = args.cpu_rows
        inputs = prepare_oracle_inputs(shapes, rows)
        f, s_, cores = oracle_sample(shapes, rows, inputs)
        line["cpu_baseline"] = {"value": f / s_ / 1e12, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"{rows} rows of each of the 18 shapes (A rows "
                                          f"quantised + those rows of D), weights pre-quantised; "
                                          f"{s_:.1f} s"}
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def make_parser():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=1024)
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-moe", action="store_true",
                    help="skip the MoE workloads (contiguous, masked, K-grouped) of the default run")
    ap.add_argument("--shape", default="",
                    help="M,N,K[;M,N,K...]: time only these shapes (profiling)")
    ap.add_argument("--quick", action="store_true",
                    help="timed device loop only: no e2e leg, CPU baseline or clock sampling")
    ap.add_argument("--workload", default="dense",
                    choices=["dense", "contiguous", "masked", "kgrouped", "ue8m0", "fp8fp4",
                             "layouts"],
                    help="dense (the bench line) or one MoE variant at its benchmark size")
    ap.add_argument("--masked-index", type=int, default=0,
                    help="masked workload: index into the (N, K) pairs")
    return ap


def main():
    args = make_parser().parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "fp8fp4":
        return run_fp8fp4(args)
    if args.workload == "layouts":
        return run_layouts(args)
    if args.workload == "ue8m0":
        return run_ue8m0(args)
    if args.workload != "dense":
        return run_grouped(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""Benchmark of the SC bipolar XNOR matmul hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
quantise A (+ row statistic), quantise B, assign rows (rung + rung-sorted
order), SC count + decode -- four C-ABI calls on one stream.  The stream
tables are built once before timing (they are built once per layer load).
For the linear layers the weight is static, so by default (--prepare-b auto)
it is quantised and its tensor-core B stages prepared once before timing, as
at layer load (sc_prepare_b; the time is reported as weight_prep_ms), and a
step is three calls: quantise A, assign rows, count + decode.

Default workload (the largest single-GPU configuration): ViT-L MLP fc2 with
K-bands, X [4112 x 4096] = GELU(N(0,1)) times W^T, W [1024 x 4096]
~ N(0, 0.02^2), the contraction split into 16 bands of 256 whose lengths
tilt the ladder {64, 96, 128, 192, 256} linearly (tilt 0.25) under the
iso-compute identity; per-row rungs by thresholds (0.8, 0.6, 0.4, 0.2) on
||X_i||_inf.  The other workloads (--workload) are the attention QK^T and AV
and fc1 configurations and the wider rows' variants.

Multi-GPU (torchrun): every rank runs a whole problem of its own
(workloads.shard: its own (batch, head) groups, or its own tokens against the
replicated weight; weak scaling, no data-path collective); the time is the
max over ranks, the value the bit-ops of all ranks over that time.

Prints ONE JSON line on rank 0.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SC bit-ops/s (Σ L_i·N·D / s) and % of binding roofline on 1 B200"
UNIT = "bit-ops/s"
L2_BYTES = 126 * 1024 * 1024
# DRAM bytes (read + write) of one launch of the dominant count kernel, from
# ncu captures (dram__bytes_read.sum + dram__bytes_write.sum), keyed by
# workload, by whether the second operand was prepared (sc_prepare_b) and by
# the hash of the CUDA sources the capture was taken with
# (kernel_source_hash()); a run whose sources hash differently reports null.
NCU_TRAFFIC = {
    ("fc2", True, "8c1aa6bf520f"): 1709905152 + 344122368,
    ("fc1", True, "8c1aa6bf520f"): 616134656 + 47747328,
    ("qk", False, "8c1aa6bf520f"): 9487616 + 8060928,
    ("av", False, "8c1aa6bf520f"): 22831616 + 0,
}

CONFIG_TEXT = {
    "single": "single SC matmul 64x64x64, uniform L=64",
    "qk": "ViT-L attention QK^T: batch 16 x 16 heads, Q,K [257x64] ~N(0,1), 2% outlier rows x8, "
          "ladder {64,96,128,192,256}, tau (0.8,0.6,0.4,0.2) on ||Q_i||inf",
    "av": "ViT-L attention AV: batch 16 x 16 heads, A = softmax(N(0,2^2)) [257x257], V [257x64], "
          "ladder keyed on max_j A_ij",
    "fc1": "ViT-L MLP fc1: X [4112x1024] Student-t(4) x W^T, W [4096x1024] ~N(0,0.02^2)",
    "fc2": "ViT-L MLP fc2 + 16 K-bands of 256: X [4112x4096] GELU(N(0,1)) x W^T, W [1024x4096], "
           "linear tilt 0.25",
    "fc2_bs": "ViT-L MLP fc2 + 16 K-bands of 256 with one quantisation scale per (row, band): "
              "X [4112x4096] GELU(N(0,1)) x W^T, W [1024x4096], linear tilt 0.25",
    "qk_mp": "ViT-L attention QK^T as qk, fraction-based fixed MP per head: lengths "
             "{256,128,64,32} on 15/57.5/22.5/5 % of the 16 heads of each image by |Q|.amax",
    "av_mp": "ViT-L attention AV as av, fraction-based fixed MP per attention row: lengths "
             "{256,128,64,32} on 15/57.5/22.5/5 % of the rows by max_j A_ij",
    "fc1_mp": "ViT-L MLP fc1 as fc1, fraction-based fixed MP per input row: lengths "
              "{256,128,64,32} on 15/57.5/22.5/5 % of the rows by ||X_i||inf",
    "qk_uni": "ViT-L attention QK^T as qk, unipolar AND mode (sign-magnitude streams, one "
              "enable-gated counter)",
    "qk_gray": "ViT-L attention QK^T as qk, Sobol sequence in Gray-code order",
    "qk_pool": "ViT-L attention QK^T as qk, per-index Sobol pool of width 64 (index d streams "
               "from Sobol dimension d + 1)",
    "fc2_pool": "ViT-L MLP fc2 + 16 K-bands as fc2, per-index Sobol pool of width 4096",
}


def kernel_source_hash() -> str:
    """First 12 hex digits of the SHA-256 of the library's CUDA sources
    (csrc/*.cu, *.cuh, include/sc.h), in name order."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixed_precision_vit_b200", "csrc")
    for p in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))
                    + [os.path.join(ROOT, "include", "sc.h")]):
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def _peaks():
    fallback = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            with open(p) as f:
                d = json.load(f)
        except (OSError, ValueError):
            d = None
        # a measured figure where the file has one, the fallback for the rest
        if isinstance(d, dict) and isinstance(d.get("bf16_tflops"), (int, float)):
            return {**fallback, **{k: v for k, v in d.items() if isinstance(v, (int, float))}}, "measured"
    return fallback, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.idx)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.25)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def combine_ranks(total_ms, e2e_ms, mm_ms, bitops, device):
    """Times: max over ranks; work: sum over ranks (weak scaling, one batch of
    independent groups per rank).  Single process: unchanged."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(total_ms), float(e2e_ms), float(mm_ms), float(bitops)
    times = torch.tensor([total_ms, e2e_ms, mm_ms], dtype=torch.float64, device=device)
    work = torch.tensor([float(bitops)], dtype=torch.float64, device=device)
    dist.all_reduce(times, op=dist.ReduceOp.MAX)
    dist.all_reduce(work, op=dist.ReduceOp.SUM)
    return float(times[0]), float(times[1]), float(times[2]), float(work[0])


def _sub_groups(w, g0: int, n: int):
    """The same workload restricted to groups g0 .. g0 + n - 1."""
    import dataclasses
    return dataclasses.replace(w, a=w.a[g0:g0 + n], b=w.b[g0:g0 + n])


def cpu_baseline(workload: str, budget_s: float = 12.0, steps_cap=None):
    """The oracle as it stands, on all host cores, over whole (batch, head)
    groups (or row blocks) of the same workload until about budget_s of
    work.  Returns (bitops/s, description, cores, per-step samples)."""
    import numpy as np

    import oracle
    from oracle import pipeline
    from mixed_precision_vit_b200 import workloads as W
    oracle.build()
    w = W.make(workload)
    cores = oracle.max_threads()
    # sample unit: one group for batched workloads (one set of heads when the
    # heads are ranked together), a block of 16 rows otherwise
    gs = w.frac_set if w.frac_set > 0 else 1
    if w.batch > 1:
        units = [("group", g) for g in range(0, w.batch, gs)]
    else:
        units = [("rows", r0) for r0 in range(0, w.M, 16)]
    t_all, bits_all, n_done, per = 0.0, 0, 0, []
    for kind, u in units:
        if kind == "group":
            sub = _sub_groups(w, u, gs)
            sel = None
        else:
            sub = w
            sel = None
        t0 = time.perf_counter()
        if kind == "group":
            st, _, _, steps = pipeline.run(sub)
        else:
            st = getattr(cpu_baseline, "_st", None)
            if st is None:
                st = pipeline.prepare(w)
                cpu_baseline._st = st
            rows = np.arange(u, min(u + 16, w.M))
            g, i, j = np.meshgrid([0], rows, np.arange(w.N), indexing="ij")
            sel = np.stack([g.ravel(), i.ravel(), j.ravel()], 1)
            _, _, _, steps = pipeline.run(w, st, sel=sel)
        dt = time.perf_counter() - t0
        t_all += dt
        bits_all += steps
        n_done += 1
        per.append(steps / dt)
        if t_all >= budget_s or (steps_cap and n_done >= steps_cap):
            break
    if kind == "group":
        desc = f"first {n_done * gs} of {w.batch} (batch, head) groups, every output, bit by bit"
    else:
        desc = f"first {n_done * 16} of {w.M} rows x all {w.N} columns, bit by bit"
    return bits_all / t_all, desc, cores, per


def run_reference(args):
    """Reference arm: the CPU oracle on the host cores (bounded samples)."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    from mixed_precision_vit_b200 import workloads as W  # noqa: F401
    import oracle
    from oracle import pipeline
    oracle.build()
    w = W.make(args.workload)
    cores = oracle.max_threads()
    per_step_groups = (w.frac_set if w.frac_set > 0 else 2) if w.batch > 1 else None
    times, bits = [], []
    total = args.warmup + args.steps
    import numpy as np
    st_full = None
    for s in range(total):
        t0 = time.perf_counter()
        if per_step_groups:
            g0 = (s * per_step_groups) % w.batch
            sub = _sub_groups(w, g0, per_step_groups)
            _, _, _, steps = pipeline.run(sub)
        else:
            if st_full is None:
                st_full = pipeline.prepare(w)
            r0 = (s * 4) % w.M
            rows = np.arange(r0, min(r0 + 4, w.M))
            g, i, j = np.meshgrid([0], rows, np.arange(w.N), indexing="ij")
            sel = np.stack([g.ravel(), i.ravel(), j.ravel()], 1)
            _, _, _, steps = pipeline.run(w, st_full, sel=sel)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            bits.append(steps)
    value = sum(bits) / sum(times)
    sample = (f"{per_step_groups} (batch, head) groups per step, every output, bit by bit"
              if per_step_groups else "4 rows x all columns per step, bit by bit")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
            "config": {"workload": args.workload, "text": CONFIG_TEXT[args.workload],
                       "sc_prec": 8},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="fc2", choices=sorted(CONFIG_TEXT))
    ap.add_argument("--engine", default="auto", choices=["auto", "gather", "tc"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--prepare-b", default="auto", choices=["auto", "on", "off"],
                    help="prepare a static second operand once (linear layers; auto: when the "
                         "wide-tile tensor-core kernel runs the problem)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch
    import torch.distributed as dist

    ws, rank, local = _dist()
    if ws > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from mixed_precision_vit_b200 import _lib as L
    from mixed_precision_vit_b200 import workloads as W
    from mixed_precision_vit_b200.sc import ScStep
    L.load()
    engine = {"auto": L.SC_ENGINE_AUTO, "gather": L.SC_ENGINE_GATHER, "tc": L.SC_ENGINE_TC}[args.engine]
    w = W.shard(args.workload, rank)
    prep = args.prepare_b == "on"
    if args.prepare_b == "auto" and w.op == W.OP_LINEAR:
        probe = ScStep(w, device=dev, engine=engine)
        try:
            prep = L.sc_prepare_b_bytes(probe.desc, probe.table.handle) > 0
        except L.ScError:
            prep = False
        probe.close()
    step = ScStep(w, device=dev, engine=engine, prepare_b=prep)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def one(ev=None):
        return step.run(stream=stream, events=ev)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one()
    torch.cuda.synchronize()
    bitops = step.bitops()
    row_L = step.row_lengths()
    launches = step.launches()
    hist = {int(Lv): int((row_L == Lv).sum()) for Lv in w.ladder}

    # -------- timed region: device events per step, L2 flushed between steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    clocks = ClockSampler(ids[local] if local < len(ids) else local)
    clocks.start()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for k in range(args.steps):
            flush.zero_()
            starts[k].record(stream)
            one(ev=mm[k])
            ends[k].record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    t_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    t_mm = [a.elapsed_time(b) for a, b in mm]
    total_ms = sum(t_step)
    mm_ms = sum(t_mm) / len(t_mm)

    # -------- end to end: host (pinned) inputs -> C ABI -> host output, the
    # public HostPipeline: every step uploads its inputs and downloads its
    # output, the copies of neighbouring steps overlapping the compute
    from mixed_precision_vit_b200.sc import HostPipeline
    a_h = w.a.pin_memory()
    b_h = w.b.pin_memory()
    out_h = torch.empty(step.out.shape, dtype=torch.float32).pin_memory()
    pipe = HostPipeline(step)
    st_w, en_w = pipe.run(a_h, b_h, out_h, 2)   # warm-up of the streams
    torch.cuda.synchronize()
    st_e, en_e = pipe.run(a_h, b_h, out_h, args.steps)
    torch.cuda.synchronize()
    e2e_ms = st_e.elapsed_time(en_e)
    h2d, d2h = pipe.bytes_per_step()

    # -------- max over ranks; totals over ranks
    total_ms, e2e_ms, mm_ms, bitops_all = combine_ranks(total_ms, e2e_ms, mm_ms, bitops, dev)

    if rank == 0:
        peaks, src = _peaks()
        value = bitops_all * args.steps / (total_ms / 1e3)
        e2e_value = bitops_all * args.steps / (e2e_ms / 1e3)
        eng = step.engine_used()
        if eng == "tc":
            # algorithmic int8 MACs of the minimal exact folded contraction:
            # sum_i ceil(L_i / 2) * N * D per launch, 2 ops per MAC
            fold = step.fold_macs()
            achieved = 2.0 * fold / (mm_ms / 1e3) / 1e12
            peak = 2.0 * peaks["bf16_tflops"]  # int8 dense = 2 x bf16 dense (nominal ratio)
            src_hash = kernel_source_hash()
            traffic = NCU_TRAFFIC.get((args.workload, bool(prep), src_hash))
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "traffic_source": (f"ncu capture of kernel sources {src_hash}" if traffic
                                       else f"none for kernel sources {src_hash}"),
                    "note": f"int8 tensor ops of the folded exact contraction; peak = 2 x {src} "
                            f"bf16 burst"}
        else:
            # CUDA-core engine: two shared-memory table gathers per (i, j, d)
            # (one in the unipolar AND mode); peak = one 32-lane LDS
            # wavefront per SM per clock
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            gathers = (1.0 if w.unipolar else 2.0) * w.batch * w.M * w.N * w.D
            achieved = gathers / (mm_ms / 1e3) / 1e12
            peak = sms * 32 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tgather/s",
                    "frac": achieved / peak, "traffic": None,
                    "note": "shared-memory gathers / s vs 32 lanes x SMs x max SM clock"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
            "data": "synthetic",
            "config": {"workload": args.workload, "text": CONFIG_TEXT[args.workload],
                       "groups_per_gpu": w.batch, "M": w.M, "N": w.N, "D": w.D,
                       "n_bands": w.n_bands, "engine": eng, "l2": "flushed between steps",
                       "parallelism": f"dp{ws} (independent groups per rank)",
                       "rung_histogram_rank0": hist, "mean_L_rank0": float(row_L.mean()),
                       "equivalent_bits_rank0": float(np.log2(row_L.mean())),
                       "bitops_per_step_rank0": int(bitops),
                       "second_operand": ("static weight, quantised and its B stages prepared once "
                                          "before timing (sc_prepare_b)" if prep
                                          else "quantised in every step")},
            "weight_prep_ms": step.prep_ms if prep else None,
            "sc_matmul_ms": mm_ms,
            "pair_ops_per_s": w.batch * w.M * w.N * w.D * ws * args.steps / (total_ms / 1e3),
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "how": "HostPipeline: every step uploads its inputs from pinned host memory and "
                           "downloads its output; uploads, compute and downloads on three streams, "
                           "neighbouring steps overlapped (inputs arrive by upload, no L2 flush)"},
            "gpu_launches": launches * args.steps,
            "clocks": clk,
            "context": "pages report ~95,000x GPU-over-CPU SC simulation speedup (other GPU)",
        }
        if not args.no_cpu_baseline and ws == 1:
            v, desc, cores, _ = cpu_baseline(args.workload, args.cpu_budget)
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                    "sample": desc}
            line["gpu_over_cpu"] = value / v
        print(json.dumps(line))
    step.close()
    if ws > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""SERQ quantized-linear benchmark on B200.

One step = one decoder layer's worth of the SERQ hot path on one batch of
synthetic activations: per shared input, the per-token quantize-and-pack
kernel, then every projection that reads it through the fused two-accumulator
GEMM (Llama-2-7B shapes: q/k/v/o 4096x4096, gate/up 4096x11008, down
11008x4096; W4A4; r = 128; M = 2048 tokens per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl serq|reference]

For N > 1 it runs under torchrun, one rank per GPU; every rank processes its
own batch (weak scaling, no data-path collective) and the step time is the
maximum over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
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

METRIC = "serq_linear TOPS and tokens/s at Llama-7B shapes; % of INT8-tensor / HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 4.5 / 2.25          # nominal dense ratio (recipe)
N_WEIGHT_COPIES = 8                  # 8 x 101 MB of packed weights > 126 MB L2
N_ACT_COPIES = 2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["serq", "reference"], default="serq")
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--profile", action="store_true",
                    help="short run for a profiler: no e2e, no CPU baseline, no clocks")
    return ap.parse_args()


# --------------------------------------------------------------------------
# workload description (shapes and algorithmic work)
# --------------------------------------------------------------------------
def groups_of(wl):
    """[(input name, [projection, ...]), ...] in the layer's order."""
    out = []
    for p in wl.projections:
        if not out or out[-1][0] != p.input:
            out.append((p.input, []))
        out[-1][1].append(p)
    return out


def ops_of(M, K, N, r):
    return 2.0 * M * N * (K + r)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over the process group (the step time of a
    weak-scaling job is its slowest rank's)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return d, "MEASURED_PEAKS.json"
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for f in ("gemm_tc.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "w4a4_rank_gemm_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per launch of the prefill GEMM from the committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    rec = d.get(workload)
    if not rec or rec.get("kernel_hash") != kernel_hash():
        return None
    return rec.get("bytes_per_launch")


# --------------------------------------------------------------------------
# clock sampling (NVML, read-only) during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.02):
        self.ok = False
        self.samples = []
        self.reasons = set()
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, b in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------
def run_gpu(args, rank, world, local_rank):
    import torch
    from w4a4_rank_gemm_b200 import build as _build
    _build.build()
    from w4a4_rank_gemm_b200 import serq as S
    from w4a4_rank_gemm_b200 import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    M = args.M
    wl = synth.llama2_7b(M=M)
    grp = groups_of(wl)
    r = wl.rank

    # offline: prepare N_WEIGHT_COPIES copies of the layer (untimed)
    layers = [dict() for _ in range(N_WEIGHT_COPIES)]
    flat = {}
    for iname, projs in grp:
        inp = wl.inputs[iname]
        Ws = [torch.from_numpy(p.W).to(dev) for p in projs]
        Xc = torch.from_numpy(inp.X_calib).to(dev)
        for c in range(N_WEIGHT_COPIES):
            for p, L in zip(projs, S.prepare_group(Ws, Xc, r, "w4a4")):
                layers[c][p.name] = L
        L0 = layers[0][projs[0].name]
        Xd = torch.from_numpy(inp.X).to(dev).to(torch.bfloat16)
        flat[iname] = [S.flatten_permute(L0, Xd) for _ in range(N_ACT_COPIES)]
        del Ws, Xc, Xd
    torch.cuda.synchronize()

    Xq = {i: torch.empty((M, wl.inputs[i].K // 2), dtype=torch.uint8, device=dev) for i, _ in grp}
    sx = {i: torch.empty(M, dtype=torch.float32, device=dev) for i, _ in grp}
    Y = {p.name: torch.empty((M, p.W.shape[1]), dtype=torch.bfloat16, device=dev) for p in wl.projections}
    ops_step = sum(ops_of(M, p.W.shape[0], p.W.shape[1], r) for p in wl.projections)
    stream = torch.cuda.current_stream()

    def step(i, gemm_events=None):
        c, a = i % N_WEIGHT_COPIES, i % N_ACT_COPIES
        for iname, projs in grp:
            S.quantize_act(flat[iname][a], "w4a4", Xq=Xq[iname], sx=sx[iname], stream=stream)
            for p in projs:
                if gemm_events is not None:
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                S.linear(layers[c][p.name], Xq[iname], sx[iname], Y=Y[p.name], stream=stream)
                if gemm_events is not None:
                    e1.record(stream)
                    gemm_events.append((p, e0, e1))

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()

    gemm_events = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(i, gemm_events)
        t1.record(stream)
        torch.cuda.synchronize()
    elapsed_ms = t0.elapsed_time(t1)
    if S.device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")

    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    barrier()

    gemm_ms = sum(e0.elapsed_time(e1) for _, e0, e1 in gemm_events)
    gemm_ops = sum(ops_of(M, p.W.shape[0], p.W.shape[1], r) for p, _, _ in gemm_events)
    per_proj = {}
    for p, e0, e1 in gemm_events:
        per_proj.setdefault(p.name, []).append(e0.elapsed_time(e1))
    secs = elapsed_ms / 1e3
    value = ops_step * args.steps * world / secs / 1e12

    pk, pk_src = peaks()
    timed_alone = secs < 2.0
    bf16 = pk.get("bf16_tflops") if timed_alone else pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    peak_int8 = bf16 * INT8_PER_BF16
    achieved = gemm_ops / (gemm_ms / 1e3) / 1e12
    launches_per_step = len(grp) + len(wl.projections)
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4 (W4A4 codes, int32 accumulate)",
        "data": "synthetic (seeded; Llama-2-7B shapes, random-init weights, outlier-channel activations)",
        "tokens_per_s": round(M * args.steps * world / secs, 1),
        "config": {
            "workload": "llama2_7b_prefill_w4a4_r128: one decoder layer's 7 projections "
                        "(q/k/v/o 4096x4096, gate/up 4096x11008, down 11008x4096), 4 shared-input quantizes",
            "tokens_per_gpu": M, "rank": r, "mode": "w4a4",
            "global_batch": M * world, "parallelism": f"dp{world} (independent token batches)",
            "l2": f"inputs larger than L2: {N_WEIGHT_COPIES} prepared weight copies cycled "
                  f"({N_WEIGHT_COPIES} x {sum(p.W.size for p in wl.projections) // 2 / 1e6:.0f} MB packed) "
                  f"and {N_ACT_COPIES} activation copies alternated",
        },
        "roofline": {
            "kernel": "serq::tc::k_gemm (tcgen05 kind::i8 prefill GEMM, main + residual accumulators)",
            "bound": "tensor",
            "achieved": round(achieved, 1),
            "peak": round(peak_int8, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / peak_int8, 4),
            "traffic": recorded_traffic("llama2_7b_prefill"),
            "peak_source": f"{pk_src}: {'bf16_tflops' if timed_alone else 'bf16_tflops_sustained'} "
                           f"x {INT8_PER_BF16} (dense int8 : bf16) -- of measured" if pk_src != "fallback"
                           else "fallback 1.59 PFLOP/s bf16 x 2 -- of fallback",
            "gemm_share_of_step": round(gemm_ms / max(elapsed_ms, 1e-9), 4),
            "per_projection_us": {k: round(1e3 * statistics.median(v), 2) for k, v in per_proj.items()},
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    return res, dict(S=S, torch=torch, wl=wl, grp=grp, layers=layers, flat=flat, Xq=Xq, sx=sx, Y=Y,
                     ops_step=ops_step, dev=dev, stream=stream)


def run_e2e(args, ctx, world):
    """Same step through the public API with the step's inputs copied from
    pinned host memory and every output copied back, inside the timed region."""
    torch, S = ctx["torch"], ctx["S"]
    grp, layers, flat, Xq, sx, Y = ctx["grp"], ctx["layers"], ctx["flat"], ctx["Xq"], ctx["sx"], ctx["Y"]
    stream = ctx["stream"]
    host_in = {i: flat[i][0].cpu().pin_memory() for i, _ in grp}
    dev_in = {i: flat[i][1] for i, _ in grp}
    host_out = {n: torch.empty(y.shape, dtype=y.dtype).pin_memory() for n, y in Y.items()}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    steps = max(3, min(args.steps, 30))

    def step(i):
        c = i % N_WEIGHT_COPIES
        for iname, projs in grp:
            dev_in[iname].copy_(host_in[iname], non_blocking=True)
            S.quantize_act(dev_in[iname], "w4a4", Xq=Xq[iname], sx=sx[iname], stream=stream)
            for p in projs:
                S.linear(layers[c][p.name], Xq[iname], sx[iname], Y=Y[p.name], stream=stream)
                host_out[p.name].copy_(Y[p.name], non_blocking=True)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    ms = max_over_ranks(ms, world, ctx["dev"])
    return {"value": round(ctx["ops_step"] * steps * world / (ms / 1e3) / 1e12, 3), "unit": "TOPS",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3)}


# --------------------------------------------------------------------------
# CPU oracle arm (baseline / reference)
# --------------------------------------------------------------------------
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([d.get("num_threads", 1) for d in info] + [1])
    except Exception:
        return os.cpu_count() or 1


class OracleArm:
    """The oracle as it stands, on a bounded token sample of the workload."""

    def __init__(self, M_sample, wl=None):
        from oracle import serq_oracle as O
        from w4a4_rank_gemm_b200 import synth
        self.O = O
        self.wl = wl if wl is not None else synth.llama2_7b(M=2048)
        self.grp = groups_of(self.wl)
        self.M_s = M_sample
        self.prep = {}
        self.xh = {}
        for iname, projs in self.grp:
            inp = self.wl.inputs[iname]
            _, _, ls = O.prepare_group([p.W for p in projs], inp.X_calib, self.wl.rank)
            for p, L in zip(projs, ls):
                self.prep[p.name] = L
            L0 = ls[0]
            self.xh[iname] = O.flatten_permute(inp.X[:M_sample], L0.s, L0.pi, out_bf16=True)
        self.ops = sum(ops_of(M_sample, p.W.shape[0], p.W.shape[1], self.wl.rank) for p in self.wl.projections)

    def step(self):
        O = self.O
        for iname, projs in self.grp:
            xq, sx = O.quantize_act(self.xh[iname], 4)
            for p in projs:
                L = self.prep[p.name]
                acc0, acc1 = O.linear_accum(xq, L)
                O.linear_epilogue(acc0, acc1, sx, L)


def cpu_baseline(args, wl=None):
    arm = OracleArm(64, wl)
    arm.step()  # warm (allocations)
    n, t = 0, 0.0
    while t < args.cpu_seconds or n < 2:
        t0 = time.perf_counter()
        arm.step()
        t += time.perf_counter() - t0
        n += 1
    return {"value": round(arm.ops * n / t / 1e12, 5), "unit": "TOPS", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"{arm.M_s} tokens of each of the 4 layer inputs through all 7 projections "
                      f"(quantize + two-accumulator integer GEMM + fp64 epilogue), {n} passes in {t:.1f} s"}


def run_reference(args):
    arm = OracleArm(64)
    for _ in range(args.warmup):
        arm.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        arm.step()
    secs = time.perf_counter() - t0
    value = arm.ops * args.steps / secs / 1e12
    cores = cpu_threads()
    sample = f"{arm.M_s} tokens per layer input through all 7 Llama-2-7B projections per step"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int4 codes, int64-exact integer GEMM + fp64 epilogue (CPU oracle)",
        "data": "synthetic (seeded; Llama-2-7B shapes)",
        "config": {"workload": "llama2_7b_prefill_w4a4_r128 (bounded token sample)", "tokens_per_step": arm.M_s,
                   "rank": arm.wl.rank, "mode": "w4a4"},
        "cpu_baseline": {"value": round(value, 5), "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------------
def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        res, ctx = run_gpu(args, rank, world, local_rank)
        if not args.profile and not args.no_e2e:
            res["e2e"] = run_e2e(args, ctx, world)
        if rank == 0 and world == 1 and not args.profile and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args, None)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""SERQ quantized-linear benchmark on B200.

Default workload (the headline): one step = one Llama-2-7B decoder layer's
worth of the SERQ hot path on one batch of synthetic activations: per shared
input the per-token quantize-and-pack kernel, then every projection that reads
it through the fused two-accumulator GEMM (q/k/v/o 4096x4096, gate/up
4096x11008, down 11008x4096; W4A4; r = 128; M = 2048 tokens per GPU).

Other workloads (--workload): llama2_7b_decode (M tokens, default 16, CUDA
graphs, HBM roofline), llama3_8b_w4a8 (M = 4096, INT8 activations),
mlp_block (gate/up -> SiLU*mul + quantize -> down, M = 4096).

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
N_WEIGHT_COPIES = 8                  # 8 x ~100 MB of packed weights > 126 MB L2
N_ACT_COPIES = 2
WORKLOADS = ("llama2_7b_prefill", "llama2_7b_decode", "llama3_8b_w4a8", "mlp_block", "l2qer_compare")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["serq", "reference"], default="serq")
    ap.add_argument("--workload", choices=WORKLOADS, default="llama2_7b_prefill")
    ap.add_argument("--M", type=int, default=None, help="tokens per GPU (default per workload)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--algo", type=int, default=0,
                    help="serq_algo for every linear launch (0 = automatic choice)")
    ap.add_argument("--mode", choices=["w4a4", "w4a8"], default=None,
                    help="override the workload's quantization mode (same shapes)")
    ap.add_argument("--no-group", action="store_true",
                    help="one launch per projection instead of one per shared-input group")
    ap.add_argument("--profile", action="store_true",
                    help="short run for a profiler: no e2e, no CPU baseline")
    a = ap.parse_args()
    if a.M is None:
        a.M = {"llama2_7b_prefill": 2048, "llama2_7b_decode": 16, "llama3_8b_w4a8": 4096,
               "mlp_block": 4096, "l2qer_compare": 2048}[a.workload]
    return a


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


def linear_bytes(M, K, N, r, a_bits):
    """Algorithmic DRAM bytes of one linear launch: packed W, packed R, the
    two scale vectors, the activation codes and scales, the bf16 output."""
    rpad = (r + 31) // 32 * 32
    return N * K / 2 + N * rpad / 2 + 8 * N + M * K * a_bits / 8 + 4 * M + 2 * M * N


def fuses_act_quantize(decode, grouped, M, K):
    """Whether a shared-input group runs as one serq_linear_group_act launch
    whose GEMV CTAs quantize the tokens themselves (decode, grouped, M <= 8,
    K <= 4096); otherwise the quantize is a launch of its own."""
    return bool(decode and grouped and M <= 8 and K <= 4096)


def residual_summary(times):
    """times[(projection, v)] = us per call for v = 0 (main products only),
    1 (SERQ: main + its rank-r compensator in the same launch), 2 (main, then
    the two-factor comparator's products).  Returns the per-projection
    figures, the summed residual times and the comparator / SERQ ratio.
    SERQ's residual rides in the main launch; where its added time is below
    the timings' noise (1% of the main products: run-to-run spread of these
    event timings) the ratio divides by that floor and says so."""
    per = {}
    sum_serq = sum_two = sum_main = 0.0
    for name in dict.fromkeys(n for n, _ in times):
        t0, t1, t2 = (times[(name, v)] for v in range(3))
        per[name] = {"main_us": round(t0, 2), "serq_us": round(t1, 2), "two_factor_us": round(t2, 2),
                     "serq_residual_us": round(t1 - t0, 2), "two_factor_residual_us": round(t2 - t0, 2)}
        sum_main += t0
        sum_serq += t1 - t0
        sum_two += t2 - t0
    floor = 0.01 * sum_main
    return {"per": per, "sum_main": sum_main, "sum_serq": sum_serq, "sum_two": sum_two,
            "ratio": sum_two / max(sum_serq, floor), "at_floor": sum_serq < floor}


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


def kernel_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "w4a4_rank_gemm_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, files):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    rec = d.get(workload)
    if not rec or rec.get("kernel_hash") != kernel_hash(files):
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

    def __init__(self, index, period=0.002):
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

    def _sample(self):
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, b in self.REASONS.items():
                if bits & b and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
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
# GPU workloads
# --------------------------------------------------------------------------
class LayerWorkload:
    """Independent projections grouped by shared input (a decoder layer)."""

    def __init__(self, args, S, torch, dev):
        from w4a4_rank_gemm_b200 import synth
        self.S, self.torch, self.dev = S, torch, dev
        self.algo = args.algo
        self.grouped = not args.no_group
        self.name = args.workload
        M = self.M = args.M
        if args.workload == "llama3_8b_w4a8":
            wl = synth.llama3_8b(M=M)
        else:
            wl = synth.llama2_7b(M=M)
        if args.mode is not None:
            wl.mode = args.mode
        self.wl = wl
        self.mode = wl.mode
        self.a_bits = 4 if wl.mode == "w4a4" else 8
        self.grp = groups_of(wl)
        r = self.r = wl.rank
        self.layers = [dict() for _ in range(N_WEIGHT_COPIES)]
        self.flat = {}
        for iname, projs in self.grp:
            inp = wl.inputs[iname]
            Ws = [torch.from_numpy(p.W).to(dev) for p in projs]
            Xc = torch.from_numpy(inp.X_calib).to(dev)
            for c in range(N_WEIGHT_COPIES):
                for p, L in zip(projs, S.prepare_group(Ws, Xc, r, wl.mode)):
                    self.layers[c][p.name] = L
            L0 = self.layers[0][projs[0].name]
            Xd = torch.from_numpy(inp.X).to(dev).to(torch.bfloat16)
            self.flat[iname] = [S.flatten_permute(L0, Xd) for _ in range(N_ACT_COPIES)]
            del Ws, Xc, Xd
        torch.cuda.synchronize()
        bpr = lambda K: K // 2 if self.a_bits == 4 else K
        self.Xq = {i: torch.empty((M, bpr(wl.inputs[i].K)), dtype=torch.uint8, device=dev) for i, _ in self.grp}
        self.sx = {i: torch.empty(M, dtype=torch.float32, device=dev) for i, _ in self.grp}
        self.Y = {p.name: torch.empty((M, p.W.shape[1]), dtype=torch.bfloat16, device=dev)
                  for p in wl.projections}
        self.gemms = [(p.name, p.W.shape[0], p.W.shape[1]) for p in wl.projections]
        self.ops_step = sum(ops_of(M, K, N, r) for _, K, N in self.gemms)
        self.gemm_bytes_step = sum(linear_bytes(M, K, N, r, self.a_bits) for _, K, N in self.gemms)
        self.decode = M <= S.decode_max_m()
        n_gemm_launches = len(self.grp) if self.grouped else len(self.gemms)
        n_quant = sum(0 if self.fused(i, ps) else 1 for i, ps in self.grp)
        self.launches_per_step = n_quant + n_gemm_launches
        self.weight_mb = sum(p.W.size for p in wl.projections) / 2 / 1e6

    def describe(self):
        shapes = ", ".join(f"{n} {K}x{N}" for n, K, N in self.gemms)
        return (f"{self.name}_{self.mode}_r{self.r}: one decoder layer's {len(self.gemms)} projections "
                f"({shapes}), {len(self.grp)} shared-input quantizes, M = {self.M} tokens per GPU")

    def fused(self, iname, projs):
        return fuses_act_quantize(self.decode, self.grouped, self.M, self.wl.inputs[iname].K)

    def step(self, i, stream, events=None, gemm_only=False):
        S, torch = self.S, self.torch
        c, a = i % N_WEIGHT_COPIES, i % N_ACT_COPIES
        for iname, projs in self.grp:
            if self.fused(iname, projs):
                # one launch, quantize included (also in the GEMM-only graph:
                # it is the GEMV launch of this group)
                S.linear_group_act([self.layers[c][p.name] for p in projs], self.flat[iname][a],
                                   Ys=[self.Y[p.name] for p in projs], Xq=self.Xq[iname], sx=self.sx[iname],
                                   algo=self.algo, stream=stream)
                continue
            if not gemm_only:
                S.quantize_act(self.flat[iname][a], self.mode, Xq=self.Xq[iname], sx=self.sx[iname], stream=stream)
            for name, ps in self._launches(projs):
                if events is not None:
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                self._linear(c, iname, ps, stream)
                if events is not None:
                    e1.record(stream)
                    events.append((name, e0, e1))

    def _launches(self, projs):
        """[(name, [projection, ...]), ...]: one entry per GEMM call."""
        if self.grouped and len(projs) > 1:
            return [("+".join(p.name for p in projs), projs)]
        return [(p.name, [p]) for p in projs]

    def _linear(self, c, iname, ps, stream):
        S = self.S
        if len(ps) > 1:
            S.linear_group([self.layers[c][p.name] for p in ps], self.Xq[iname], self.sx[iname],
                           Ys=[self.Y[p.name] for p in ps], algo=self.algo, stream=stream)
        else:
            S.linear(self.layers[c][ps[0].name], self.Xq[iname], self.sx[iname], Y=self.Y[ps[0].name],
                     algo=self.algo, stream=stream)

    # end-to-end hooks: device inputs and outputs per buffer b (0/1), so that a
    # step's copies overlap its neighbours' compute
    def host_buffers(self):
        torch = self.torch
        self.host_in = {i: self.flat[i][0].cpu().pin_memory() for i, _ in self.grp}
        self.host_out = {n: torch.empty(y.shape, dtype=y.dtype).pin_memory() for n, y in self.Y.items()}
        self.Ybuf = [self.Y, {n: torch.empty_like(y) for n, y in self.Y.items()}]
        return self.host_in, self.host_out

    def e2e_inputs(self, b):
        return [(self.host_in[i], self.flat[i][b]) for i, _ in self.grp]

    def e2e_outputs(self, b):
        return [(self.Ybuf[b][n], self.host_out[n]) for n in self.Y]

    def e2e_compute(self, i, b, stream):
        S = self.S
        c = i % N_WEIGHT_COPIES
        Y = self.Y
        self.Y = self.Ybuf[b]
        try:
            for iname, projs in self.grp:
                if self.fused(iname, projs):
                    S.linear_group_act([self.layers[c][p.name] for p in projs], self.flat[iname][b],
                                       Ys=[self.Y[p.name] for p in projs], Xq=self.Xq[iname], sx=self.sx[iname],
                                       algo=self.algo, stream=stream)
                    continue
                S.quantize_act(self.flat[iname][b], self.mode, Xq=self.Xq[iname], sx=self.sx[iname], stream=stream)
                for _, ps in self._launches(projs):
                    self._linear(c, iname, ps, stream)
        finally:
            self.Y = Y


class MLPWorkload:
    """gate/up (down_proj's order folded into their columns) -> SiLU*mul +
    quantize -> down, one Llama-2-7B MLP block."""

    def __init__(self, args, S, torch, dev):
        from w4a4_rank_gemm_b200 import synth
        self.S, self.torch, self.dev = S, torch, dev
        self.algo = args.algo
        self.grouped = not args.no_group
        self.name = "mlp_block"
        M = self.M = args.M
        blk = synth.mlp_block(M=M)
        self.r = r = blk.rank
        self.mode, self.a_bits = "w4a4", 4
        dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
        Wg, Wu, Wd, Xc, Hc = dv(blk.Wg), dv(blk.Wu), dv(blk.Wd), dv(blk.X_calib), dv(blk.H_calib)
        self.copies = []
        for c in range(N_WEIGHT_COPIES):
            (Ld,) = S.prepare_group([Wd], Hc, r, "w4a4")
            p4, s4 = Ld.perm_smooth()
            Lg, Lu = S.prepare_group([Wg, Wu], Xc, r, "w4a4", out_perm=[dv(p4), dv(p4)], out_div=[None, dv(s4)])
            self.copies.append((Lg, Lu, Ld))
        Lg0 = self.copies[0][0]
        Xd = dv(blk.X).to(torch.bfloat16)
        self.flat = [S.flatten_permute(Lg0, Xd) for _ in range(N_ACT_COPIES)]
        del Wg, Wu, Wd, Xc, Hc, Xd
        K, F = blk.Wg.shape
        self.K, self.F = K, F
        self.Xq = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        self.sx = torch.empty(M, dtype=torch.float32, device=dev)
        self.G = torch.empty((M, F), dtype=torch.bfloat16, device=dev)
        self.U = torch.empty((M, F), dtype=torch.bfloat16, device=dev)
        self.Hq = torch.empty((M, F // 2), dtype=torch.uint8, device=dev)
        self.hsx = torch.empty(M, dtype=torch.float32, device=dev)
        self.Yd = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.gemms = [("gate_proj", K, F), ("up_proj", K, F), ("down_proj", F, K)]
        self.ops_step = sum(ops_of(M, k, n, r) for _, k, n in self.gemms)
        self.gemm_bytes_step = sum(linear_bytes(M, k, n, r, 4) for _, k, n in self.gemms)
        self.launches_per_step = 4 if self.grouped else 5
        self.weight_mb = 3 * K * F / 2 / 1e6
        self.decode = False
        torch.cuda.synchronize()

    def describe(self):
        return (f"mlp_block_w4a4_r{self.r}: Llama-2-7B MLP, gate/up {self.K}x{self.F} with down_proj's saliency "
                f"order folded into their columns -> SiLU*mul + quantize -> down {self.F}x{self.K}, "
                f"M = {self.M} tokens per GPU")

    def step(self, i, stream, events=None, gemm_only=False):
        S, torch = self.S, self.torch
        Lg, Lu, Ld = self.copies[i % N_WEIGHT_COPIES]
        if not gemm_only:
            S.quantize_act(self.flat[i % N_ACT_COPIES], "w4a4", Xq=self.Xq, sx=self.sx, stream=stream)
        if self.grouped:
            calls = (("gate_proj+up_proj", [Lg, Lu], self.Xq, self.sx, [self.G, self.U], None),
                     ("down_proj", [Ld], self.Hq, self.hsx, [self.Yd], "silu"))
        else:
            calls = (("gate_proj", [Lg], self.Xq, self.sx, [self.G], None),
                     ("up_proj", [Lu], self.Xq, self.sx, [self.U], None),
                     ("down_proj", [Ld], self.Hq, self.hsx, [self.Yd], "silu"))
        for name, Ls, xq, sx, ys, pre in calls:
            if pre == "silu" and not gemm_only:
                S.silu_mul_quantize(self.G, self.U, "w4a4", Xq=self.Hq, sx=self.hsx, stream=stream)
            if events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            if len(Ls) > 1:
                S.linear_group(Ls, xq, sx, Ys=ys, algo=self.algo, stream=stream)
            else:
                S.linear(Ls[0], xq, sx, Y=ys[0], algo=self.algo, stream=stream)
            if events is not None:
                e1.record(stream)
                events.append((name, e0, e1))

    def host_buffers(self):
        torch = self.torch
        self.host_in = {"x": self.flat[0].cpu().pin_memory()}
        self.host_out = {"y": torch.empty(self.Yd.shape, dtype=self.Yd.dtype).pin_memory()}
        self.Ydbuf = [self.Yd, torch.empty_like(self.Yd)]
        return self.host_in, self.host_out

    def e2e_inputs(self, b):
        return [(self.host_in["x"], self.flat[b])]

    def e2e_outputs(self, b):
        return [(self.Ydbuf[b], self.host_out["y"])]

    def e2e_compute(self, i, b, stream):
        Yd = self.Yd
        self.Yd = self.Ydbuf[b]
        try:
            self.step(b, stream)  # step(b) reads flat[b % N_ACT_COPIES]
        finally:
            self.Yd = Yd


def run_gpu(args, rank, world, local_rank):
    import torch
    from w4a4_rank_gemm_b200 import build as _build
    _build.build()
    from w4a4_rank_gemm_b200 import serq as S

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    W = MLPWorkload(args, S, torch, dev) if args.workload == "mlp_block" else LayerWorkload(args, S, torch, dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    graphs = None
    if W.decode:
        # decode kernels run for microseconds: replay one captured step per
        # weight copy so host launch overhead does not enter the timing
        for i in range(3):
            W.step(i, stream)
        torch.cuda.synchronize()
        graphs, gemm_graphs = [], []
        for c in range(N_WEIGHT_COPIES):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                W.step(c, torch.cuda.current_stream())
            graphs.append(g)
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2):
                W.step(c, torch.cuda.current_stream(), gemm_only=True)
            gemm_graphs.append(g2)
        run_step = lambda i: graphs[i % N_WEIGHT_COPIES].replay()
    else:
        run_step = lambda i: W.step(i, stream)

    for i in range(args.warmup):
        run_step(i)
    torch.cuda.synchronize()
    barrier()

    # Headline region: whole steps, nothing recorded between kernels (an
    # event between two launches would serialise them and hide the
    # programmatic-dependent-launch overlap of one kernel's tail with the
    # next one's prologue).
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            run_step(i)
        t1.record(stream)
        torch.cuda.synchronize()
        elapsed_ms = t0.elapsed_time(t1)

        # Roofline region, right after: the same steps with CUDA events around
        # every GEMM launch (prefill), or replays of a graph holding only the
        # step's GEMM launches (decode).
        per_proj = {}
        roof_steps = min(args.steps, 100)
        if graphs is None:
            events = []
            for i in range(roof_steps):
                W.step(i, stream, events)
            torch.cuda.synchronize()
            gemm_ms = sum(e0.elapsed_time(e1) for _, e0, e1 in events)
            for n, e0, e1 in events:
                per_proj.setdefault(n, []).append(e0.elapsed_time(e1))
            gemm_note = (f"CUDA events around every GEMM launch, {roof_steps} steps timed right after the "
                         "headline steps")
        else:
            g0 = torch.cuda.Event(enable_timing=True)
            g1 = torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for i in range(roof_steps):
                gemm_graphs[i % N_WEIGHT_COPIES].replay()
            g1.record(stream)
            torch.cuda.synchronize()
            gemm_ms = g0.elapsed_time(g1)
            gemm_note = (f"CUDA events around {roof_steps} replays of a graph holding only the step's GEMM "
                         "launches, timed right after the headline steps")
    if S.device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    barrier()
    secs = elapsed_ms / 1e3

    pk, pk_src = peaks()
    timed_alone = secs < 2.0
    res = {
        "metric": METRIC,
        "value": round(W.ops_step * args.steps * world / secs / 1e12, 3),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4 (W4A4 codes, int32 accumulate)" if W.a_bits == 4 else "int4 weights x int8 activations, int32 accumulate",
        "data": "synthetic (seeded; Llama shapes, random-init weights, outlier-channel activations)",
        "tokens_per_s": round(W.M * args.steps * world / secs, 1),
        "config": {
            "workload": W.describe(),
            "tokens_per_gpu": W.M, "rank": W.r, "mode": W.mode,
            "global_batch": W.M * world, "parallelism": f"dp{world} (independent token batches)",
            "l2": f"inputs larger than L2: {N_WEIGHT_COPIES} prepared weight copies cycled "
                  f"({N_WEIGHT_COPIES} x {W.weight_mb:.0f} MB packed) and {N_ACT_COPIES} activation copies alternated",
            "cuda_graphs": graphs is not None,
            "algo": args.algo,
            "grouped_launches": W.grouped,
        },
        "gpu_launches": W.launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if W.decode:
        peak = pk.get("hbm_gbs")
        achieved = W.gemm_bytes_step * roof_steps / (gemm_ms / 1e3) / 1e9
        res["roofline"] = {
            "kernel": ("decode GEMVs, main + residual accumulators: serq::gs::k_gemv (streaming; at M <= 8 and "
                       "K <= 4096 (q/k/v, o, gate/up) one launch that also quantizes the tokens) and "
                       "serq::decode::k_decode (item ring; o_proj at larger M)"),
            "bound": "hbm", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": recorded_traffic(f"{W.name}_M{W.M}", ["gemv_stream.cuh", "gemv_decode.cuh", "common.cuh"]),
            "peak_source": f"{pk_src}: hbm_gbs" + (" -- of measured" if pk_src != "fallback" else " -- of fallback"),
            "gemm_share_of_step": round(gemm_ms / roof_steps / max(elapsed_ms / args.steps, 1e-9), 4),
            "timing": gemm_note,
        }
    else:
        bf16 = pk.get("bf16_tflops") if timed_alone else pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
        peak_int8 = bf16 * INT8_PER_BF16
        achieved = W.ops_step * roof_steps / (gemm_ms / 1e3) / 1e12
        res["roofline"] = {
            "kernel": "serq::tc::k_gemm (tcgen05 kind::i8 prefill GEMM, main + residual accumulators)",
            "bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak_int8, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak_int8, 4),
            "traffic": recorded_traffic(W.name, ["gemm_tc.cuh", "common.cuh"]),
            "peak_source": (f"{pk_src}: {'bf16_tflops' if timed_alone else 'bf16_tflops_sustained'} x "
                            f"{INT8_PER_BF16} (dense int8 : bf16) -- of measured") if pk_src != "fallback"
                           else "fallback 1.59 PFLOP/s bf16 x 2 -- of fallback",
            "gemm_share_of_step": round(gemm_ms / roof_steps / max(elapsed_ms / args.steps, 1e-9), 4),
            "per_projection_us": {k: round(1e3 * statistics.median(v), 2) for k, v in per_proj.items()},
            "timing": gemm_note,
        }
    return res, dict(S=S, torch=torch, W=W, dev=dev, stream=stream)


def run_e2e(args, ctx, world):
    """Same step through the public API with the step's inputs copied from
    pinned host memory and every output copied back, inside the timed region.
    Steps are pipelined on three streams (host->device copies, compute,
    device->host copies) with two device buffer sets: step i's compute runs
    while step i + 1's inputs go up and step i - 1's outputs come down, and
    events keep a buffer from being refilled before its last reader is done."""
    torch, W, stream = ctx["torch"], ctx["W"], ctx["stream"]
    host_in, host_out = W.host_buffers()
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    steps = max(3, min(args.steps, 30))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]
    in_ready, in_free, out_ready, out_free = ev(), ev(), ev(), ev()
    used = [False, False]

    def one(i):
        b = i % 2
        if used[b]:
            s_in.wait_event(in_free[b])       # the compute that read these inputs is done
        with torch.cuda.stream(s_in):
            for h, d in W.e2e_inputs(b):
                d.copy_(h, non_blocking=True)
        in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if used[b]:
            stream.wait_event(out_free[b])    # these outputs have been copied out
        W.e2e_compute(i, b, stream)
        in_free[b].record(stream)
        out_ready[b].record(stream)
        s_out.wait_event(out_ready[b])
        with torch.cuda.stream(s_out):
            for d, h in W.e2e_outputs(b):
                h.copy_(d, non_blocking=True)
        out_free[b].record(s_out)
        used[b] = True

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        one(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, ctx["dev"])
    return {"value": round(W.ops_step * steps * world / (ms / 1e3) / 1e12, 3), "unit": "TOPS",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "pipelining": "copies of neighbouring steps overlap compute (3 streams, 2 buffer sets)"}


# --------------------------------------------------------------------------
# SERQ's residual path against the two-factor comparator (L2QER)
# --------------------------------------------------------------------------
def run_compare(args):
    """Per Llama-2-7B projection, three variants on the same activation codes:
    the main 4-bit product alone (rank 0), SERQ (main + the single r x N
    residual on the salient columns, one launch) and the comparator (the
    same main product, plus X_q L1 -> on-the-fly quantization -> L2, three
    launches).  The residual path's cost is each variant's time minus the
    main product's.  Decode sizes replay each variant as a CUDA graph."""
    import torch
    from w4a4_rank_gemm_b200 import build as _build
    _build.build()
    from w4a4_rank_gemm_b200 import serq as S
    from w4a4_rank_gemm_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    M, copies = args.M, 4
    wl = synth.llama2_7b(M=M)
    r = wl.rank
    projs = []
    for iname, ps in groups_of(wl):
        inp = wl.inputs[iname]
        Xc = torch.from_numpy(inp.X_calib).to(dev)
        for p in ps:
            W = torch.from_numpy(p.W).to(dev)
            K, N = p.W.shape
            L1, L2 = synth.factor_pair(K, N, r, seed=len(projs) + 31)
            L1d, L2d = torch.from_numpy(L1).to(dev), torch.from_numpy(L2).to(dev)
            var = []
            for _ in range(copies):
                L0 = S.prepare(W, Xc, 0)
                Lr = S.prepare(W, Xc, r)
                var.append((L0, Lr, S.L2QER(L0, L1d, L2d)))
            Xh = S.flatten_permute(var[0][0], torch.from_numpy(inp.X).to(dev).to(torch.bfloat16))
            Xq, sx = S.quantize_act(Xh, "w4a4")
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            projs.append(dict(name=p.name, K=K, N=N, var=var, Xq=Xq, sx=sx, Y=Y,
                              bufs=var[0][2].buffers(M, dev)))
            del W
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    decode = M <= S.decode_max_m()

    def call(pr, v, c):
        L0, Lr, Q = pr["var"][c]
        # the current stream: the timing stream, or the capture stream of a graph
        if v == 0:
            S.linear(L0, pr["Xq"], pr["sx"], Y=pr["Y"])
        elif v == 1:
            S.linear(Lr, pr["Xq"], pr["sx"], Y=pr["Y"])
        else:
            Q.linear(pr["Xq"], pr["sx"], Y=pr["Y"], bufs=pr["bufs"])

    reps = max(10, min(args.steps, 200))
    times = {}
    for pr in projs:
        for v in range(3):
            for c in range(copies):
                call(pr, v, c)
            torch.cuda.synchronize()
            if decode:
                gs = []
                for c in range(copies):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        call(pr, v, c)
                    gs.append(g)
                run = lambda i, gs=gs: gs[i % copies].replay()
            else:
                run = lambda i, pr=pr, v=v: call(pr, v, i % copies)
            for i in range(3):
                run(i)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for i in range(reps):
                run(i)
            e1.record(stream)
            torch.cuda.synchronize()
            times[(pr["name"], v)] = e0.elapsed_time(e1) * 1e3 / reps   # us per call
            if decode:
                del gs
    if S.device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")
    rs = residual_summary(times)
    per, sum_main, sum_serq, sum_two, ratio = rs["per"], rs["sum_main"], rs["sum_serq"], rs["sum_two"], rs["ratio"]
    return {
        "metric": "residual-path latency: two-factor comparator (L2QER) / SERQ, one Llama-2-7B layer",
        "value": round(ratio, 3), "unit": "x", "higher_is_better": True, "n_gpus": 1,
        "serq_residual_at_noise_floor": rs["at_floor"],
        "steps": reps, "warmup": 3, "ms_per_step": round((sum_main + sum_serq) / 1e3, 4),
        "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 (W4A4 codes, int32 accumulate)",
        "data": "synthetic (seeded; Llama shapes, random-init weights and factors, outlier-channel activations)",
        "config": {"workload": f"l2qer_compare: 7 projections of one Llama-2-7B layer, M = {M}, r = {r}, "
                               f"{copies} weight copies cycled; {'CUDA graphs' if decode else 'stream launches'}",
                   "tokens_per_gpu": M, "rank": r},
        "residual_us": {"serq": round(sum_serq, 2), "two_factor": round(sum_two, 2), "main_only": round(sum_main, 2)},
        "per_projection": per,
        "gpu_launches": 7 * reps * 5,
    }


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

    def __init__(self, workload, M_sample):
        from oracle import serq_oracle as O
        from w4a4_rank_gemm_b200 import synth
        self.O = O
        self.workload = workload
        self.M_s = M_sample
        if workload == "mlp_block":
            blk = synth.mlp_block(M=max(M_sample, 16))
            self.blk = blk
            self.prep = O.prepare_mlp(blk.Wg, blk.Wu, blk.Wd, blk.X_calib, blk.H_calib, blk.rank)
            self.X = blk.X[:M_sample]
            K, F = blk.Wg.shape
            self.ops = 2 * ops_of(M_sample, K, F, blk.rank) + ops_of(M_sample, F, K, blk.rank)
            self.rank = blk.rank
            return
        wl = synth.llama3_8b(M=max(M_sample, 16)) if workload == "llama3_8b_w4a8" else \
            synth.llama2_7b(M=max(M_sample, 16))
        self.wl, self.grp = wl, groups_of(wl)
        self.bits = 4 if wl.mode == "w4a4" else 8
        self.rank = wl.rank
        self.prep, self.xh = {}, {}
        for iname, projs in self.grp:
            inp = wl.inputs[iname]
            _, _, ls = O.prepare_group([p.W for p in projs], inp.X_calib, wl.rank)
            for p, L in zip(projs, ls):
                self.prep[p.name] = L
            self.xh[iname] = O.flatten_permute(inp.X[:M_sample], ls[0].s, ls[0].pi, out_bf16=True)
        self.ops = sum(ops_of(M_sample, p.W.shape[0], p.W.shape[1], wl.rank) for p in wl.projections)

    def step(self):
        O = self.O
        if self.workload == "mlp_block":
            O.mlp_forward(self.X, self.prep)
            return
        for iname, projs in self.grp:
            xq, sx = O.quantize_act(self.xh[iname], self.bits)
            for p in projs:
                L = self.prep[p.name]
                acc0, acc1 = O.linear_accum(xq, L)
                O.linear_epilogue(acc0, acc1, sx, L)


def oracle_sample(args):
    return min(args.M, 64)


def cpu_baseline(args):
    arm = OracleArm(args.workload, oracle_sample(args))
    arm.step()  # warm (allocations)
    n, t = 0, 0.0
    while t < args.cpu_seconds or n < 2:
        t0 = time.perf_counter()
        arm.step()
        t += time.perf_counter() - t0
        n += 1
    return {"value": round(arm.ops * n / t / 1e12, 5), "unit": "TOPS", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"{arm.M_s} tokens through the workload's quantize + two-accumulator integer GEMM + "
                      f"fp64 epilogue ({args.workload}), {n} passes in {t:.1f} s"}


def run_reference(args):
    arm = OracleArm(args.workload, oracle_sample(args))
    for _ in range(args.warmup):
        arm.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        arm.step()
    secs = time.perf_counter() - t0
    value = arm.ops * args.steps / secs / 1e12
    cores = cpu_threads()
    sample = f"{arm.M_s} tokens per step through the {args.workload} workload"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "integer codes, exact integer GEMM + fp64 epilogue (CPU oracle)",
        "data": "synthetic (seeded; Llama shapes)",
        "config": {"workload": f"{args.workload} (bounded token sample)", "tokens_per_step": arm.M_s,
                   "rank": arm.rank},
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
    if args.workload == "l2qer_compare":
        if world == 1:
            print(json.dumps(run_compare(args)), flush=True)
        return
    try:
        res, ctx = run_gpu(args, rank, world, local_rank)
        if not args.profile and not args.no_e2e:
            res["e2e"] = run_e2e(args, ctx, world)
        if rank == 0 and world == 1 and not args.profile and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

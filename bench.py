#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 (NVFP4) linear layer and the AWQ W4A16 linear layer.

One step is one pass of the whole hot path over one batch of synthetic input:
  * the SVDQ W4A4 NVFP4 attention projection, M=4096, K=N=3072, rank 32, group 16
    (kernel 1: smoothing + NVFP4 quantization + low-rank down; kernel 2: the
    block-scaled tcgen05 GEMM with the low-rank-up/bias epilogue);
  * the AWQ W4A16 adaLN linear, K=3072, N=18432, group 64, at M = 1, 2, 4, 8, 16, 32, 64.
`value` is the SVDQ layer throughput in TFLOP/s (2MNK per step over the device
time of kernels 1+2); the AWQ throughput in GB/s is reported under "awq".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: the layers do not need to shard (every GPU runs its own replica),
so N ranks run N independent replicas; `value` sums all ranks' work over the
slowest rank's time ("scaling": "weak").  Inputs and weights are rotated over
8 resident copies so that every step reads from HBM, not from L2.
"""

import argparse
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 SVDQ W4A4 linear TFLOPS (% FP4 peak); AWQ W4A16 GB/s (% HBM)"
SVDQ_SHAPE = (4096, 3072, 3072)              # M, K, N: DiT attention projection, 64x64 latent tokens
AWQ_K, AWQ_N, AWQ_MS = 3072, 18432, (1, 2, 4, 8, 16, 32, 64)
RANK = 32
NSETS = 8                                    # rotating copies (> 2x L2 per cycle)
NREP = 3                                     # passes over the copies per CUDA-graph batch (24 launches)
FP4_OVER_BF16 = 4.0                          # nominal dense ratio (9 / 2.25 PFLOP/s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=384)       # 16 graph batches of 24
    ap.add_argument("--warmup", type=int, default=24)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly (for profilers)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", action="store_true",
                    help="one resident copy, eager launches of every kernel (for ncu captures); prints timings")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- distributed plumbing

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "ours" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available() and args.impl == "ours":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def time_dynamic_variant(P, wl, stream, use_graph, reps=5):
    """The dynamic-activation-scale layer (a variant, timed after the main region): kernel 5
    alone and the whole layer (kernels 5, 1, 2), each as CUDA-graph batches over the copies."""
    import torch
    out = {}
    for name, fn in (("amax", wl.amax), ("layer", wl.dyn_layer)):
        def batch():
            for _ in range(NREP):
                for i in range(NSETS):
                    fn(P, i)
        with torch.cuda.stream(stream):
            batch()                                  # warm-up (eager)
        torch.cuda.synchronize()
        if use_graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                batch()
            run = g.replay
        else:
            run = batch
        best = None
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            with torch.cuda.stream(stream):
                run()
            e1.record(stream)
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / (NSETS * NREP)
            best = t if best is None else min(best, t)
        out[name + "_us"] = best * 1e3
    M, K, N = SVDQ_SHAPE
    out["amax_gbs"] = 2.0 * M * K / (out["amax_us"] * 1e-6) / 1e9
    out["layer_tflops"] = svdq_flops() / (out["layer_us"] * 1e-6) / 1e12
    out["note"] = "g_a from the batch's amax (kernel 5) instead of calibration; best of 5 graph batches of 24"
    return out


def job_rate(world, steps, units_per_step, slowest_ms):
    """Whole-job throughput in units per second: the units all ranks processed (each rank ran
    `steps` steps of `units_per_step`) over the slowest rank's device time."""
    return world * steps * units_per_step / (slowest_ms * 1e-3)


def allreduce_max(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks during the timed region

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Samples the SM clock and the clock-event reasons of one GPU through NVML."""

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()
            self._run_once()

    def _run_once(self):
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
        except Exception:
            pass

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        names = [n for bit, n in REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------- our implementation

def bf16_dev(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).to(dev)


class Workload:
    """Resident inputs, weights and outputs of one step, in NSETS rotating copies."""

    def __init__(self, P, dev):
        import torch
        import synth
        M, K, N = SVDQ_SHAPE
        w = synth.svdq_workload(M, K, N)
        blob, self.g_w = P.svdq_pack_weights(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2),
                                             synth.bf16_bits(w.bias), synth.bf16_bits(w.smooth_inv))
        self.g_a = w.g_a
        self.M, self.K, self.N = M, K, N
        X = bf16_dev(w.X, dev)
        self.smooth = bf16_dev(w.smooth_inv, dev)
        blob_d = torch.from_numpy(blob).to(dev)
        self.host_X = w.X                                   # for the end-to-end leg
        self.sets = []
        for _ in range(NSETS):
            self.sets.append({
                "X": X.clone(), "W": blob_d.clone(),
                "codes": torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                "scales": torch.empty((P.svdq_act_scale_bytes(M, K),), dtype=torch.uint8, device=dev),
                "U": torch.empty((M, 2 * RANK), dtype=torch.bfloat16, device=dev),
                "Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                "amax": torch.zeros((4,), dtype=torch.int32, device=dev),
            })
        a = synth.awq_workload(max(AWQ_MS), AWQ_K, AWQ_N)
        ax = bf16_dev(a.X, dev)
        qw = torch.from_numpy(a.qweight).to(dev)
        sc, zr = bf16_dev(a.scales, dev), bf16_dev(a.zeros, dev)
        self.awq_sets = []
        for _ in range(NSETS):
            s = {"qw": qw.clone(), "s": sc.clone(), "z": zr.clone(), "X": {}, "Y": {}}
            for m in AWQ_MS:
                s["X"][m] = ax[:m].clone()
                s["Y"][m] = torch.empty((m, AWQ_N), dtype=torch.bfloat16, device=dev)
            self.awq_sets.append(s)

    def k1(self, P, i):
        s = self.sets[i]
        P.svdq_quantize_act_lowrank_down(s["X"], self.smooth, s["W"], self.g_a, RANK, s["codes"], s["scales"], s["U"])

    def k2(self, P, i):
        s = self.sets[i]
        P.svdq_w4a4_nvfp4_linear(s["codes"], s["scales"], s["U"], self.g_a, s["W"], self.g_w,
                                 self.M, self.N, self.K, RANK, s["Y"])

    def amax(self, P, i):
        s = self.sets[i]
        P.svdq_act_amax(s["X"], self.smooth, s["amax"])

    def dyn_layer(self, P, i):
        """The layer with the dynamic activation scale: kernel 5, then kernels 1 and 2 reading it."""
        s = self.sets[i]
        P.svdq_act_amax(s["X"], self.smooth, s["amax"])
        P.svdq_quantize_act_lowrank_down_dyn(s["X"], self.smooth, s["W"], s["amax"], RANK, s["codes"], s["scales"],
                                             s["U"])
        P.svdq_w4a4_nvfp4_linear_dyn(s["codes"], s["scales"], s["U"], s["amax"], s["W"], self.g_w,
                                     self.M, self.N, self.K, RANK, s["Y"])

    def awq(self, P, i, m):
        s = self.awq_sets[i]
        P.awq_w4a16_linear(s["X"][m], s["qw"], s["s"], s["z"], None, s["Y"][m])


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one nvfp4_gemm_kernel<256>
# launch at the attention shape, from an ncu capture with cold caches (13.15 MB read = the
# algorithmic input bytes; the bf16 output stays in L2 within the launch).  Must be
# re-measured whenever the GEMM kernel changes.
GEMM_DRAM_BYTES_PER_LAUNCH = 13154560


def svdq_flops():
    M, K, N = SVDQ_SHAPE
    return 2.0 * M * N * K


def k1_bytes():
    M, K, N = SVDQ_SHAPE
    return 2 * M * K + 2 * K + 4 * K * RANK + M * K / 2 + M * K / 16 + 4 * M * RANK


def k2_bytes():
    M, K, N = SVDQ_SHAPE
    return (N + M) * K * (0.5 + 1 / 16) + 2 * RANK * N + 2 * N + 4 * M * RANK + 2 * M * N


def awq_bytes(m):
    return AWQ_N * AWQ_K / 2 + 4 * AWQ_N * AWQ_K / 64 + 2 * m * AWQ_K + 2 * m * AWQ_N


def run_ours(args, world, rank, local):
    import torch
    import bit_diffusion_transformer_act_b200 as P
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    wl = Workload(P, dev)
    stream = torch.cuda.Stream()
    names = ["k1", "k2"] + ["awq%d" % m for m in AWQ_MS]

    def launch(name, i):
        if name == "k1":
            wl.k1(P, i)
        elif name == "k2":
            wl.k2(P, i)
        else:
            wl.awq(P, i, int(name[3:]))

    # one graph per kernel kind: NREP passes over the NSETS rotating copies (a batch of 24 launches),
    # plus single-set graphs for remainders
    with torch.cuda.stream(stream):
        for i in range(NSETS):                       # eager warm-up (sets attributes, loads modules)
            for n in names:
                launch(n, i)
    torch.cuda.synchronize()
    graphs, singles = {}, {}
    use_graph = not args.no_graph
    if use_graph:
        for n in names:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(NREP):
                    for i in range(NSETS):
                        launch(n, i)
            graphs[n] = g
            singles[n] = []
            for i in range(NSETS):
                g1 = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g1, stream=stream):
                    launch(n, i)
                singles[n].append(g1)
    torch.cuda.synchronize()

    def run_steps(nsteps, events):
        """Runs nsteps steps on `stream`; appends (name, start, end, launches) event records."""
        done = 0
        while done < nsteps:
            chunk = min(NSETS * NREP, nsteps - done)
            for n in names:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                if use_graph and chunk == NSETS * NREP:
                    graphs[n].replay()
                elif use_graph:
                    for i in range(chunk):
                        singles[n][i % NSETS].replay()
                else:
                    with torch.cuda.stream(stream):
                        for i in range(chunk):
                            launch(n, i % NSETS)
                e1.record(stream)
                if events is not None:
                    events.append((n, e0, e1, chunk))
            done += chunk

    with torch.cuda.stream(stream):
        run_steps(max(args.warmup, 3), None)
    torch.cuda.synchronize()

    events = []
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        with torch.cuda.stream(stream):
            run_steps(args.steps, events)
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = start.elapsed_time(end)
    per = {n: [0.0, 0] for n in names}
    for n, e0, e1, c in events:
        per[n][0] += e0.elapsed_time(e1)
        per[n][1] += c
    avg_ms = {n: per[n][0] / max(per[n][1], 1) for n in names}
    svdq_ms = per["k1"][0] + per["k2"][0]
    svdq_ms_max = allreduce_max(svdq_ms, world)
    total_ms_max = allreduce_max(total_ms, world)
    awq_ms = {m: per["awq%d" % m][0] for m in AWQ_MS}
    awq_ms_max = {m: allreduce_max(awq_ms[m], world) for m in AWQ_MS}
    status = P.svdq_device_status()
    if status:
        raise RuntimeError("device status %d after the timed region" % status)
    variants = {"svdq_dynamic_act_scale": time_dynamic_variant(P, wl, stream, use_graph)}

    value = job_rate(world, args.steps, svdq_flops(), svdq_ms_max) / 1e12
    fp4_peak = FP4_OVER_BF16 * peaks["bf16_tflops"]
    k2_tflops = svdq_flops() / (avg_ms["k2"] * 1e-3) / 1e12
    k1_gbs = k1_bytes() / (avg_ms["k1"] * 1e-3) / 1e9
    awq_per_m = {}
    for m in AWQ_MS:
        gbs = awq_bytes(m) / (avg_ms["awq%d" % m] * 1e-3) / 1e9
        agg = job_rate(world, args.steps, awq_bytes(m), awq_ms_max[m]) / 1e9
        awq_per_m[str(m)] = {"us": avg_ms["awq%d" % m] * 1e3, "gbs": gbs, "gbs_all_ranks": agg,
                             "frac_hbm": gbs / peaks["hbm_gbs"]}
    awq_all = job_rate(world, args.steps, sum(awq_bytes(m) for m in AWQ_MS), sum(awq_ms_max.values())) / 1e9

    result = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 codes, e4m3 scales per 16, fp32 accumulate); awq int4 x bf16",
        "data": "synthetic",
        "config": {
            "workload": "SVDQ W4A4 NVFP4 DiT attention projection M=4096 K=3072 N=3072 rank 32 group 16 "
                        "+ AWQ W4A16 adaLN K=3072 N=18432 group 64 at M=1,2,4,8,16,32,64",
            "svdq": {"M": SVDQ_SHAPE[0], "K": SVDQ_SHAPE[1], "N": SVDQ_SHAPE[2], "rank": RANK, "group": 16},
            "awq": {"M": list(AWQ_MS), "K": AWQ_K, "N": AWQ_N, "group": 64},
            "l2": "inputs, weights and outputs rotate over 8 resident copies (> 2x L2 per cycle); no flush",
            "launch": "CUDA graphs of 24 launches per kernel (3 passes over the 8 copies)" if use_graph else "eager",
            "parallelism": "replicas x%d" % world,
            "seed": 0,
        },
        "svdq_ms_per_step": svdq_ms_max / args.steps,
        "roofline": {
            "bound": "tensor", "achieved": k2_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
            "frac": k2_tflops / fp4_peak, "traffic": GEMM_DRAM_BYTES_PER_LAUNCH,
            "traffic_unit": "bytes per launch (dram read + write, ncu, cold caches)",
            "traffic_source": "profiles/nvfp4_gemm_attention_4096x3072x3072.md",
            "kernel": "nvfp4_gemm_kernel<256>",
            "peak_note": "dense FP4 = 4 x measured bf16 burst (%s), nominal 9/2.25 ratio" % peaks["source"],
        },
        "kernels": {
            "quant_act_lowrank_kernel": {"us": avg_ms["k1"] * 1e3, "bound": "hbm", "gbs": k1_gbs,
                                         "frac": k1_gbs / peaks["hbm_gbs"], "bytes": k1_bytes()},
            "nvfp4_gemm_kernel": {"us": avg_ms["k2"] * 1e3, "bound": "tensor", "tflops": k2_tflops,
                                  "frac": k2_tflops / fp4_peak, "flops": svdq_flops(),
                                  "frac_of_9pf_datasheet": k2_tflops / 9000.0},
            "layer": {"us": (avg_ms["k1"] + avg_ms["k2"]) * 1e3,
                      "tflops": svdq_flops() / ((avg_ms["k1"] + avg_ms["k2"]) * 1e-3) / 1e12},
        },
        "variants": variants,
        "awq": {"value": awq_all, "unit": "GB/s", "frac_hbm": awq_all / peaks["hbm_gbs"], "per_m": awq_per_m,
                "hbm_peak_gbs": peaks["hbm_gbs"]},
        "gpu_launches": (2 + len(AWQ_MS)) * args.steps,
        "clocks": clocks.summary(),
    }
    result["e2e"] = e2e_ours(args, P, wl, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline()
    return result


def e2e_ours(args, P, wl, dev, world):
    """The same layer through the public API with the input in pinned host memory and the
    output read back to pinned host memory, every step inside the timed region."""
    import torch
    M, K, N = SVDQ_SHAPE
    hX = torch.from_numpy(wl.host_X).to(torch.bfloat16).pin_memory()
    hY = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    s0 = wl.sets[0]
    dX = torch.empty_like(s0["X"])

    def step():
        dX.copy_(hX, non_blocking=True)
        codes, scales, U = P.svdq_quantize_act_lowrank_down(dX, wl.smooth, s0["W"], wl.g_a, RANK,
                                                            s0["codes"], s0["scales"], s0["U"])
        P.svdq_w4a4_nvfp4_linear(codes, scales, U, wl.g_a, s0["W"], wl.g_w, M, N, K, RANK, s0["Y"])
        hY.copy_(s0["Y"], non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.e2e_steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = allreduce_max(e0.elapsed_time(e1), world)
    val = world * args.e2e_steps * svdq_flops() / (ms * 1e-3) / 1e12
    return {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": hX.numel() * 2,
            "d2h_bytes_per_step": hY.numel() * 2, "steps": args.e2e_steps,
            "note": "SVDQ layer via the C ABI; pinned host X in, pinned host Y out, per step"}


# ---------------------------------------------------------------- CPU oracle legs

def _oracle_layer_prepared():
    import synth
    from oracle import awq, nvfp4, svdq
    M, K, N = SVDQ_SHAPE
    w = synth.svdq_workload(M, K, N)
    cw, sw, gw = svdq.quantize_weights(w.R)                 # offline, like packing (untimed)
    wq = nvfp4.dequantize(cw, sw, gw)
    a = synth.awq_workload(max(AWQ_MS), AWQ_K, AWQ_N)
    return w, wq, a


def _oracle_svdq_rows(w, wq, rows):
    import numpy as np
    from oracle import nvfp4, svdq
    X = w.X[:rows]
    cx, sx = svdq.quantize_activations(X, w.smooth_inv, w.g_a)
    y = nvfp4.dequantize(cx, sx, w.g_a) @ wq.T
    y = y + svdq.lowrank_down(X, w.smooth_inv, w.L1) @ w.L2.astype(np.float64) + w.bias
    return y


def _oracle_awq_rows(a, m, nrows):
    from oracle import awq
    return awq.forward(a.X[:m], a.q[:nrows], a.scales[:nrows], a.zeros[:nrows])


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline():
    """The oracle as it stands on this host's cores: the full attention layer and the full
    AWQ weight at M=64 (weights quantized once beforehand, as the packer does offline)."""
    w, wq, a = _oracle_layer_prepared()
    M, K, N = SVDQ_SHAPE
    t = time.perf_counter()
    _oracle_svdq_rows(w, wq, M)
    dt = time.perf_counter() - t
    t = time.perf_counter()
    _oracle_awq_rows(a, 64, AWQ_N)
    da = time.perf_counter() - t
    return {"value": svdq_flops() / dt / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": "whole attention layer M=4096 K=N=3072 in float64 NumPy (activation quantization, "
                      "dequantize, matmul, low-rank, bias), %.2f s; weights quantized beforehand" % dt,
            "awq": {"value": awq_bytes(64) / da / 1e9, "unit": "GB/s", "sample": "M=64, whole N=18432 (%.2f s)" % da}}


def run_reference(args, world, rank):
    """The oracle on the host cores, the same metric and workload, each step a row sample."""
    if rank != 0:
        return None
    w, wq, a = _oracle_layer_prepared()
    t = time.perf_counter()
    _oracle_svdq_rows(w, wq, 64)
    per_row = (time.perf_counter() - t) / 64
    budget = 120.0 / max(args.steps + args.warmup, 1)       # whole run within a few minutes
    rows = int(max(1, min(SVDQ_SHAPE[0], budget / per_row)))
    for _ in range(args.warmup):
        _oracle_svdq_rows(w, wq, rows)
    t = time.perf_counter()
    for _ in range(args.steps):
        _oracle_svdq_rows(w, wq, rows)
    dt = time.perf_counter() - t
    M, K, N = SVDQ_SHAPE
    val = args.steps * 2.0 * rows * N * K / dt / 1e12
    return {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "SVDQ W4A4 NVFP4 DiT attention projection M=4096 K=3072 N=3072 rank 32 "
                                   "group 16 (row sample per step)", "rows_per_step": rows},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                             "sample": "%d of 4096 rows per step, float64 NumPy oracle" % rows},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_profile_case(args):
    """Each kernel launched eagerly `steps` times on one resident copy of the workload."""
    import torch
    import bit_diffusion_transformer_act_b200 as P
    global NSETS
    NSETS = 1
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = Workload(P, dev)
    out = {}
    jobs = [("k1", lambda: wl.k1(P, 0)), ("k2", lambda: wl.k2(P, 0))] + \
           [("awq%d" % m, (lambda m=m: wl.awq(P, 0, m))) for m in AWQ_MS]
    for name, fn in jobs:
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out[name + "_us"] = e0.elapsed_time(e1) * 1e3 / args.steps
    out["device_status"] = P.svdq_device_status()
    return out


def main():
    args = parse()
    if args.profile_case:
        print(json.dumps({"profile_case": run_profile_case(args)}))
        return
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        out = run_reference(args, world, rank)
    else:
        out = run_ours(args, world, rank, local)
    if rank == 0 and out is not None:
        print(json.dumps(out))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

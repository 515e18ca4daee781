#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 (NVFP4) linear layer and the AWQ W4A16 linear layer.

One step is one pass of the whole hot path over one batch of synthetic input, on every
seeded configuration:
  * the SVDQ W4A4 NVFP4 DiT attention projection, M=4096, K=N=3072, rank 32, group 16, as the
    layer runs it (kernel 1: smoothing + NVFP4 quantization + low-rank down, chained with
    programmatic dependent launch into kernel 2: the block-scaled tcgen05 GEMM with the
    low-rank-up/bias epilogue), then each of its two kernels on its own;
  * the AWQ W4A16 adaLN linear, K=3072, N=18432, group 64, at M = 1, 2, 4, 8, 16, 32, 64;
  * the SVDQ fused-QKV sweep, K=3072, N=9216, M = 64, 256, 1024, 4608, 18432 (layer);
  * the SVDQ DiT MLP pair: up 4608x3072->12288, down 4608x12288->3072 on GELU-shaped inputs.
`value` is the attention layer's throughput in TFLOP/s (2MNK per step over the device time
of its chained kernels); every other figure is reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Timing: each segment (a layer or kernel of one configuration) is one CUDA graph holding
exactly K launches (or K layers) over rotating resident copies of its inputs, weights and
outputs (more than twice the L2 size per cycle, so every launch reads from HBM); CUDA events
on the launching stream bracket every graph, and the timed region is all segments back to
back.  The SM clock is sampled through NVML throughout the timed region.

Multi-GPU: the layers do not need to shard (every GPU runs its own replica), so N ranks run N
independent replicas; `value` sums all ranks' work over the slowest rank's time ("scaling":
"weak").
"""

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 SVDQ W4A4 linear TFLOPS (% FP4 peak); AWQ W4A16 GB/s (% HBM)"
ATTN = (4096, 3072, 3072)                    # M, K, N: DiT attention projection, 64x64 latent tokens
QKV_K, QKV_N, QKV_MS = 3072, 9216, (64, 256, 1024, 4608, 18432)
QKV_HEADS, QKV_FUSED_MS, QKV_EPS = 24, (64, 4608), 1e-6   # 24 heads of 128; the fused-epilogue rows
MLP_UP = (4608, 3072, 12288)
MLP_DOWN = (4608, 12288, 3072)
AWQ_K, AWQ_N, AWQ_MS = 3072, 18432, (1, 2, 4, 8, 16, 32, 64)
RANK = 32
FP4_OVER_BF16 = 4.0                          # nominal dense ratio (9 / 2.25 PFLOP/s)
# Nominal dense FP4 rate of one SM per clock: one kind::mxf4nvf4 MMA of M=128 (per SM),
# N=256, K=64 every 128 cycles.  Times the SM count and the sampled clock it gives the
# clock-matched peak beside the measured-derived one.
FP4_FLOP_PER_SM_CLK = 2 * 128 * 256 * 64 / 128
GEMM_SOURCES = ("gemm_nvfp4.cuh", "ptx.cuh", "act_amax.cuh", "libsvdq.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "nvfp4_gemm_kernel_attention_4096x3072x3072_dram.txt")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=48)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly (for profilers)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", action="store_true",
                    help="one resident copy, eager launches of every kernel (for ncu captures); prints timings")
    ap.add_argument("--case", default="attention",
                    choices=["attention", "qkv64", "qkv4608_fused", "mlp_fused", "int4"],
                    help="workload of --profile-case")
    return ap.parse_args(argv)


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


def gemm_sources_sha():
    """sha256 over the GEMM kernel's sources: a DRAM capture is valid only for the build it
    was taken on."""
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "bit_diffusion_transformer_act_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def captured_traffic():
    """DRAM bytes (read + write) per launch of the attention GEMM from the ncu capture summary,
    or None when there is none or it was taken on other kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            kv = dict(line.split(":", 1) for line in f if ":" in line and not line.startswith("#"))
    except OSError:
        return None, "no capture"
    kv = {k.strip(): v.strip() for k, v in kv.items()}
    if kv.get("sources_sha256") != gemm_sources_sha():
        return None, "capture taken on other kernel sources (stale)"
    return int(kv["dram_bytes_read"]) + int(kv["dram_bytes_write"]), "ncu capture of this build, cold caches"


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
    """Samples the SM clock and the clock-event reasons of one GPU through NVML, as often as
    NVML answers (a fraction of a millisecond), while the timed region runs."""

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

    def _sample(self):
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.0001)

    def __enter__(self):
        if self._h is not None:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        names = [n for bit, n in REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": float(np.min(self.samples)) if self.samples else None,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------- work per configuration

def bf16_dev(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).to(dev)


def n_sets(footprint_bytes, l2_bytes):
    """Rotating copies so that one pass over them touches more than twice the L2 size."""
    return int(min(16, max(2, math.ceil(2 * l2_bytes / footprint_bytes))))


def svdq_flops(M, K, N):
    return 2.0 * M * N * K


def k1_bytes(M, K):
    """Kernel 1: X, smooth_inv, the packed low-rank down factor (hi + lo), codes, scales, U (hi + lo)."""
    return 2 * M * K + 2 * K + 4 * K * RANK + M * K / 2 + M * K / 16 + 4 * M * RANK


def k2_bytes(M, K, N):
    """Kernel 2: codes and scales of both operands, L2, bias, U (hi + lo) and the bf16 output."""
    return (N + M) * K * (0.5 + 1 / 16) + 2 * RANK * N + 2 * N + 4 * M * RANK + 2 * M * N


def awq_bytes(m):
    return AWQ_N * AWQ_K / 2 + 4 * AWQ_N * AWQ_K / 64 + 2 * m * AWQ_K + 2 * m * AWQ_N


class SvdqCase:
    """One SVDQ layer (M, K, N) with its weights packed once and `nsets` rotating resident
    copies of input, weights, intermediates and output."""

    def __init__(self, P, dev, w, M, l2_bytes, nsets=None):
        import torch
        import synth
        K, N = w.K, w.N
        blob, self.g_w = P.svdq_pack_weights(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2),
                                             synth.bf16_bits(w.bias), synth.bf16_bits(w.smooth_inv))
        self.g_a = w.g_a
        self.M, self.K, self.N = M, K, N
        self.smooth = bf16_dev(w.smooth_inv, dev)
        X = bf16_dev(w.X[:M], dev)
        blob_d = torch.from_numpy(blob).to(dev)
        per_set = blob.nbytes + k1_bytes(M, K) + 2 * M * N
        self.nsets = nsets or n_sets(per_set, l2_bytes)
        self.sets = []
        for _ in range(self.nsets):
            self.sets.append({
                "X": X.clone(), "W": blob_d.clone(),
                "codes": torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                "scales": torch.empty((P.svdq_act_scale_bytes(M, K),), dtype=torch.uint8, device=dev),
                "U": torch.empty((M, 2 * RANK), dtype=torch.bfloat16, device=dev),
                "Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                "amax": torch.zeros((4,), dtype=torch.int32, device=dev),
            })

    def k1(self, P, i):
        s = self.sets[i % self.nsets]
        P.svdq_quantize_act_lowrank_down(s["X"], self.smooth, s["W"], self.g_a, RANK, s["codes"], s["scales"], s["U"])

    def k2(self, P, i):
        s = self.sets[i % self.nsets]
        P.svdq_w4a4_nvfp4_linear(s["codes"], s["scales"], s["U"], self.g_a, s["W"], self.g_w,
                                 self.M, self.N, self.K, RANK, s["Y"])

    def layer(self, P, i):
        self.k1(P, i)
        self.k2(P, i)

    def set_qkv(self, dev, heads, eps):
        """Norm weights and RoPE tables of a fused Q/K/V projection over this case's N."""
        import torch
        rng = np.random.default_rng(7)
        D = 128
        self.heads, self.eps = heads, eps
        self.wq = bf16_dev(1.0 + 0.2 * rng.standard_normal(D), dev)
        self.wk = bf16_dev(1.0 + 0.2 * rng.standard_normal(D), dev)
        ang = np.arange(self.M)[:, None] * 10000.0 ** (-np.arange(D // 2) / (D // 2))[None, :]
        self.cos = torch.from_numpy(np.ascontiguousarray(np.cos(ang).T, dtype=np.float32)).to(dev)   # [64, M]
        self.sin = torch.from_numpy(np.ascontiguousarray(np.sin(ang).T, dtype=np.float32)).to(dev)

    def qkv_fused(self, P, i):
        """Kernel 1, then the GEMM whose epilogue RMS-normalises and rotates q and k."""
        s = self.sets[i % self.nsets]
        self.k1(P, i)
        P.svdq_w4a4_nvfp4_linear_qkv(s["codes"], s["scales"], s["U"], self.g_a, s["W"], self.g_w, self.M, self.N,
                                     self.K, self.heads, self.wq, self.wk, self.eps, self.cos, self.sin, Y=s["Y"])

    def qkv_torch_norm_rope(self, P, i):
        """The unfused pipeline's second half, for comparison only: RMSNorm and RoPE of q and k
        as separate PyTorch operations on the plain layer's bf16 output (not this library)."""
        import torch
        s = self.sets[i % self.nsets]
        M, HD = self.M, self.heads * 128
        x = s["Y"][:, :2 * HD].view(M, 2, self.heads, 128).float()
        w = torch.stack([self.wq, self.wk]).float().view(1, 2, 1, 128)
        x = x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + self.eps) * w
        x0, x1 = x[..., 0::2], x[..., 1::2]
        c, sn = self.cos.t().reshape(M, 1, 1, 64), self.sin.t().reshape(M, 1, 1, 64)
        out = torch.stack([x0 * c - x1 * sn, x0 * sn + x1 * c], dim=-1).flatten(-2)
        s["Y"][:, :2 * HD].copy_(out.reshape(M, 2 * HD).to(torch.bfloat16))

    def amax(self, P, i):
        s = self.sets[i % self.nsets]
        P.svdq_act_amax(s["X"], self.smooth, s["amax"])

    def dyn_layer(self, P, i):
        """The layer with the dynamic activation scale: kernel 5, then kernels 1 and 2 reading it."""
        s = self.sets[i % self.nsets]
        P.svdq_act_amax(s["X"], self.smooth, s["amax"])
        P.svdq_quantize_act_lowrank_down_dyn(s["X"], self.smooth, s["W"], s["amax"], RANK, s["codes"], s["scales"],
                                             s["U"])
        P.svdq_w4a4_nvfp4_linear_dyn(s["codes"], s["scales"], s["U"], s["amax"], s["W"], self.g_w,
                                     self.M, self.N, self.K, RANK, s["Y"])


class Int4Case:
    """The attention layer in the int4 / group-64 row (the same seeded workload), rotating sets."""

    def __init__(self, P, dev, w, M, l2_bytes):
        import torch
        import synth
        K, N = w.K, w.N
        blob = P.svdq_int4_pack_weights(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2), synth.bf16_bits(w.bias),
                                        synth.bf16_bits(w.smooth_inv))
        self.M, self.K, self.N = M, K, N
        self.smooth = bf16_dev(w.smooth_inv, dev)
        X = bf16_dev(w.X[:M], dev)
        blob_d = torch.from_numpy(blob).to(dev)
        self.nsets = n_sets(blob.nbytes + 2 * M * K + M * K + 2 * M * N, l2_bytes)
        self.sets = [{"X": X.clone(), "W": blob_d.clone(),
                      "codes": torch.empty((M, K), dtype=torch.uint8, device=dev),
                      "scales": torch.empty((K // 64, P.int4_padded_rows(M)), dtype=torch.bfloat16, device=dev),
                      "U": torch.empty((M, 2 * RANK), dtype=torch.bfloat16, device=dev),
                      "Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev)} for _ in range(self.nsets)]

    def k1(self, P, i):
        s = self.sets[i % self.nsets]
        P.svdq_int4_quantize_act_lowrank_down(s["X"], self.smooth, s["W"], RANK, s["codes"], s["scales"], s["U"])

    def k2(self, P, i):
        s = self.sets[i % self.nsets]
        P.svdq_w4a4_int4_linear(s["codes"], s["scales"], s["U"], s["W"], self.M, self.N, self.K, RANK, s["Y"])

    def layer(self, P, i):
        self.k1(P, i)
        self.k2(P, i)


class MlpFused:
    """The MLP pair with the up projection's fused epilogue (GELU + the down projection's
    activation pass): kernel 1 on X, kernels 6 and 7, then the down projection's GEMM on their
    outputs; buffers per rotating set of the two layers."""

    def __init__(self, P, dev, up, down):
        import torch
        self.up, self.down = up, down
        M, F = up.M, up.N
        self.ws_bytes = P.svdq_gelu_quant_workspace_bytes(M, F)
        self.gelu = P.svdq_gelu_table_fill(device=dev)
        self.nsets = min(up.nsets, down.nsets)
        self.sets = [{"codes": torch.empty((M, F // 2), dtype=torch.uint8, device=dev),
                      "scales": torch.empty((P.svdq_act_scale_bytes(M, F),), dtype=torch.uint8, device=dev),
                      "U": torch.empty((M, 2 * RANK), dtype=torch.bfloat16, device=dev),
                      "ws": torch.empty((self.ws_bytes,), dtype=torch.uint8, device=dev)} for _ in range(self.nsets)]

    def up_fused(self, P, i):
        u, d, s = self.up.sets[i % self.nsets], self.down.sets[i % self.nsets], self.sets[i % self.nsets]
        self.up.k1(P, i % self.nsets)
        P.svdq_w4a4_nvfp4_linear_gelu_quant(u["codes"], u["scales"], u["U"], self.up.g_a, u["W"], self.up.g_w,
                                            self.up.M, self.up.N, self.up.K, self.down.smooth, d["W"], self.down.g_a,
                                            RANK, s["codes"], s["scales"], s["U"], s["ws"], gelu_table=self.gelu)

    def down_gemm(self, P, i):
        d, s = self.down.sets[i % self.nsets], self.sets[i % self.nsets]
        P.svdq_w4a4_nvfp4_linear(s["codes"], s["scales"], s["U"], self.down.g_a, d["W"], self.down.g_w,
                                 self.down.M, self.down.N, self.down.K, RANK, d["Y"])


class AwqCase:
    """The AWQ adaLN weight in rotating copies, with inputs and outputs for every M."""

    def __init__(self, P, dev, l2_bytes, nsets=None):
        import torch
        import synth
        a = synth.awq_workload(max(AWQ_MS), AWQ_K, AWQ_N)
        ax = bf16_dev(a.X, dev)
        qw = torch.from_numpy(a.qweight).to(dev)
        sc, zr = bf16_dev(a.scales, dev), bf16_dev(a.zeros, dev)
        self.nsets = nsets or n_sets(awq_bytes(1), l2_bytes)
        self.sets = []
        for _ in range(self.nsets):
            s = {"qw": qw.clone(), "s": sc.clone(), "z": zr.clone(), "X": {}, "Y": {}}
            for m in AWQ_MS:
                s["X"][m] = ax[:m].clone()
                s["Y"][m] = torch.empty((m, AWQ_N), dtype=torch.bfloat16, device=dev)
            self.sets.append(s)

    def run(self, P, i, m):
        s = self.sets[i % self.nsets]
        P.awq_w4a16_linear(s["X"][m], s["qw"], s["s"], s["z"], None, s["Y"][m])


class Workloads:
    def __init__(self, P, dev, l2_bytes, extra=True):
        import synth
        wa = synth.svdq_workload(*ATTN)
        self.attn = SvdqCase(P, dev, wa, ATTN[0], l2_bytes)
        self.int4 = Int4Case(P, dev, wa, ATTN[0], l2_bytes) if extra else None
        self.awq = AwqCase(P, dev, l2_bytes)
        self.qkv, self.mlp_up, self.mlp_down = {}, None, None
        if extra:
            wq = synth.svdq_workload(max(QKV_MS), QKV_K, QKV_N)      # one layer; batches are row prefixes
            self.qkv = {m: SvdqCase(P, dev, wq, m, l2_bytes) for m in QKV_MS}
            del wq
            for m in QKV_FUSED_MS:
                self.qkv[m].set_qkv(dev, QKV_HEADS, QKV_EPS)
            self.mlp_up = SvdqCase(P, dev, synth.svdq_workload(*MLP_UP), MLP_UP[0], l2_bytes)
            self.mlp_down = SvdqCase(P, dev, synth.svdq_workload(*MLP_DOWN, gelu_input=True), MLP_DOWN[0], l2_bytes)
            self.mlp_fused = MlpFused(P, dev, self.mlp_up, self.mlp_down)

    def mlp_gelu_torch(self, i):
        """The unfused pipeline's GELU: the up layer's bf16 output through PyTorch's erf-form
        GELU into the down layer's input (the rotating sets of the two layers)."""
        import torch
        n = min(self.mlp_up.nsets, self.mlp_down.nsets)
        u, d = self.mlp_up.sets[i % n], self.mlp_down.sets[i % n]
        torch.ops.aten.gelu.out(u["Y"], approximate="none", out=d["X"])

    def segments(self, P):
        """(name, launches per step, fn(i)) of every segment of one step, in timing order."""
        seg = [("attn_layer", 2, lambda i: self.attn.layer(P, i)),
               ("attn_k1", 1, lambda i: self.attn.k1(P, i)),
               ("attn_k2", 1, lambda i: self.attn.k2(P, i))]
        seg += [("awq%d" % m, 1, (lambda i, m=m: self.awq.run(P, i, m))) for m in AWQ_MS]
        if self.int4 is not None:
            seg += [("int4_layer", 2, lambda i: self.int4.layer(P, i)),
                    ("int4_k1", 1, lambda i: self.int4.k1(P, i)),
                    ("int4_k2", 1, lambda i: self.int4.k2(P, i))]
        seg += [("qkv%d" % m, 2, (lambda i, c=c: c.layer(P, i))) for m, c in self.qkv.items()]
        seg += [("qkv%d_k1" % m, 1, (lambda i, c=c: c.k1(P, i))) for m, c in self.qkv.items()]
        seg += [("qkv%d_k2" % m, 1, (lambda i, c=c: c.k2(P, i))) for m, c in self.qkv.items()]
        for m in QKV_FUSED_MS:
            if m in self.qkv:
                c = self.qkv[m]
                seg += [("qkv%d_fused" % m, 2, (lambda i, c=c: c.qkv_fused(P, i))),
                        ("qkv%d_torch_norm_rope" % m, 0, (lambda i, c=c: c.qkv_torch_norm_rope(P, i)))]
        if self.mlp_up is not None:
            seg += [("mlp_up", 2, lambda i: self.mlp_up.layer(P, i)),
                    ("mlp_gelu_torch", 0, lambda i: self.mlp_gelu_torch(i)),
                    ("mlp_down", 2, lambda i: self.mlp_down.layer(P, i)),
                    ("mlp_up_fused", 3, lambda i: self.mlp_fused.up_fused(P, i)),
                    ("mlp_down_gemm", 1, lambda i: self.mlp_fused.down_gemm(P, i))]
        return seg


# ---------------------------------------------------------------- timing

def capture(fn, steps, stream, use_graph):
    """A callable that runs fn(0..steps-1) on `stream`: one CUDA graph holding all of them, or
    eager launches."""
    import torch
    if not use_graph:
        def run():
            with torch.cuda.stream(stream):
                for i in range(steps):
                    fn(i)
        return run
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            fn(i)
    return g.replay


def time_segments(runs, stream):
    """Replays every segment once on `stream` with CUDA events around each; returns the
    milliseconds of each segment and of the whole region."""
    import torch
    ev = []
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for name, run in runs:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            run()
        e1.record(stream)
        ev.append((name, e0, e1))
    end.record(stream)
    torch.cuda.synchronize()
    return {n: e0.elapsed_time(e1) for n, e0, e1 in ev}, start.elapsed_time(end)


def time_dynamic_variant(P, wl, stream, steps, use_graph, reps=3):
    """The dynamic-activation-scale layer (a variant, timed after the main region): kernel 5
    alone and the whole layer (kernels 5, 1, 2), each a graph of `steps` launches or layers."""
    import torch
    out = {}
    for name, fn in (("amax", wl.attn.amax), ("layer", wl.attn.dyn_layer)):
        with torch.cuda.stream(stream):
            for i in range(wl.attn.nsets):
                fn(P, i)                              # warm-up (eager)
        torch.cuda.synchronize()
        run = capture(lambda i, fn=fn: fn(P, i), steps, stream, use_graph)
        run()
        best = None
        for _ in range(reps):
            ms, _ = time_segments([(name, run)], stream)
            best = ms[name] if best is None else min(best, ms[name])
        out[name + "_us"] = best * 1e3 / steps
    M, K, N = ATTN
    out["amax_gbs"] = 2.0 * M * K / (out["amax_us"] * 1e-6) / 1e9
    out["layer_tflops"] = svdq_flops(M, K, N) / (out["layer_us"] * 1e-6) / 1e12
    out["note"] = "g_a from the batch's amax (kernel 5) instead of calibration; best of %d graphs of %d" % (reps, steps)
    return out


def run_ours(args, world, rank, local):
    import torch
    import bit_diffusion_transformer_act_b200 as P
    dev = torch.device("cuda", torch.cuda.current_device())
    props = torch.cuda.get_device_properties(dev)
    l2_bytes = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    sms = props.multi_processor_count
    peaks = load_peaks()
    wl = Workloads(P, dev, l2_bytes)
    stream = torch.cuda.Stream()
    segs = wl.segments(P)
    use_graph = not args.no_graph
    K = args.steps

    # warm-up: W steps of every segment, eager (sets kernel attributes, loads modules)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            for _, _, fn in segs:
                fn(i)
    torch.cuda.synchronize()
    runs = [(name, capture(fn, K, stream, use_graph)) for name, _, fn in segs]
    for _, run in runs:                              # one untimed replay (graph upload)
        with torch.cuda.stream(stream):
            run()
    torch.cuda.synchronize()

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        seg_ms, total_ms = time_segments(runs, stream)
    barrier(world)
    status = P.svdq_device_status()
    if status:
        raise RuntimeError("device status %d after the timed region" % status)
    seg_ms_max = {n: allreduce_max(v, world) for n, v in seg_ms.items()}
    total_ms_max = allreduce_max(total_ms, world)
    launches = K * sum(c for _, c, _ in segs)
    clk = clocks.summary()

    fp4_peak = FP4_OVER_BF16 * peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    mhz = clk["sm_mhz"] or 1965.0
    fp4_clock_peak = FP4_FLOP_PER_SM_CLK * sms * mhz * 1e6 / 1e12

    def us(name):
        return seg_ms[name] * 1e3 / K

    M, Kd, N = ATTN
    fl = svdq_flops(M, Kd, N)
    value = job_rate(world, K, fl, seg_ms_max["attn_layer"]) / 1e12
    k2_tflops = fl / (us("attn_k2") * 1e-6) / 1e12
    k1_gbs = k1_bytes(M, Kd) / (us("attn_k1") * 1e-6) / 1e9
    traffic, traffic_note = captured_traffic()

    def layer_row(name, M_, K_, N_):
        t = us(name)
        fl_ = svdq_flops(M_, K_, N_)
        by = k1_bytes(M_, K_) + k2_bytes(M_, K_, N_)
        t_math = fl_ / (fp4_peak * 1e12) * 1e6
        t_mem = by / (hbm * 1e9) * 1e6
        return {"M": M_, "K": K_, "N": N_, "us": t, "tflops": fl_ / (t * 1e-6) / 1e12,
                "frac_fp4": fl_ / (t * 1e-6) / 1e12 / fp4_peak, "gbs": by / (t * 1e-6) / 1e9,
                "frac_hbm": by / (t * 1e-6) / 1e9 / hbm, "bound": "tensor" if t_math >= t_mem else "hbm",
                "roofline_frac": max(t_math, t_mem) / t, "algorithmic_bytes": by, "flops": fl_}

    awq_per_m = {}
    for m in AWQ_MS:
        t = us("awq%d" % m)
        gbs = awq_bytes(m) / (t * 1e-6) / 1e9
        awq_per_m[str(m)] = {"us": t, "gbs": gbs, "frac_hbm": gbs / hbm,
                             "gbs_all_ranks": job_rate(world, K, awq_bytes(m), seg_ms_max["awq%d" % m]) / 1e9}
    awq_all = job_rate(world, K, sum(awq_bytes(m) for m in AWQ_MS),
                       sum(seg_ms_max["awq%d" % m] for m in AWQ_MS)) / 1e9

    def qkv_row(m):
        row = layer_row("qkv%d" % m, m, QKV_K, QKV_N)
        t1, t2 = us("qkv%d_k1" % m), us("qkv%d_k2" % m)
        g_bytes = k2_bytes(m, QKV_K, QKV_N)
        row["kernels"] = {"quant_act_lowrank_kernel": {"us": t1, "frac_hbm": k1_bytes(m, QKV_K) / (t1 * 1e-6) / 1e9 / hbm},
                          "nvfp4_gemm_kernel": {"us": t2, "tflops": svdq_flops(m, QKV_K, QKV_N) / (t2 * 1e-6) / 1e12,
                                                "frac_hbm": g_bytes / (t2 * 1e-6) / 1e9 / hbm,
                                                "roofline_frac": max(svdq_flops(m, QKV_K, QKV_N) / (fp4_peak * 1e12),
                                                                     g_bytes / (hbm * 1e9)) / (t2 * 1e-6)}}
        return row

    configs = {"qkv_sweep": [qkv_row(m) for m in wl.qkv]}
    if "int4_layer" in seg_ms:
        configs["int4_attention"] = {
            "M": M, "K": Kd, "N": N, "layer_us": us("int4_layer"),
            "layer_tflops": fl / (us("int4_layer") * 1e-6) / 1e12,
            "quant_act_us": us("int4_k1"), "gemm_us": us("int4_k2"),
            "gemm_tops": fl / (us("int4_k2") * 1e-6) / 1e12,
            "gemm_frac_fp8_peak": fl / (us("int4_k2") * 1e-6) / 1e12 / (2.0 * peaks["bf16_tflops"]),
            "vs_nvfp4_layer": us("attn_layer") / us("int4_layer"),
            "note": "the int4 / group-64 row: codes carried as E4M3 bytes through the fp8 MMA, per-group scales "
                    "in the epilogue; frac against the measured-derived dense fp8 peak (2 x bf16)"}
    fused = {}
    for m in QKV_FUSED_MS:
        if "qkv%d_fused" % m not in seg_ms:
            continue
        row = layer_row("qkv%d_fused" % m, m, QKV_K, QKV_N)
        t_plain, t_torch = us("qkv%d" % m), us("qkv%d_torch_norm_rope" % m)
        row.update({"plain_layer_us": t_plain, "unfused_us": t_plain + t_torch, "torch_norm_rope_us": t_torch,
                    "speedup_vs_unfused": (t_plain + t_torch) / row["us"],
                    "epilogue_cost_vs_plain": row["us"] / t_plain})
        fused[str(m)] = row
    configs["qkv_fused_rmsnorm_rope"] = {
        "heads": QKV_HEADS, "head_dim": 128, "per_m": fused,
        "note": "kernel 1 + the GEMM with the RMSNorm + RoPE epilogue, against the plain layer and the plain "
                "layer followed by RMSNorm + RoPE as separate PyTorch operations (the unfused pipeline)"}
    if wl.mlp_up is not None:
        configs["mlp_pair"] = {"up": layer_row("mlp_up", *MLP_UP), "down_gelu_input": layer_row("mlp_down", *MLP_DOWN)}
        t_pair = us("mlp_up") + us("mlp_down")
        configs["mlp_pair"]["pair"] = {"us": t_pair, "tflops": (svdq_flops(*MLP_UP) + svdq_flops(*MLP_DOWN))
                                       / (t_pair * 1e-6) / 1e12}
        t_fused = us("mlp_up_fused") + us("mlp_down_gemm")
        t_gelu = us("mlp_gelu_torch")
        configs["mlp_pair"]["pair_with_gelu"] = {
            "us": t_pair + t_gelu, "gelu_torch_us": t_gelu,
            "note": "the unfused pipeline as a model runs it: the up layer, GELU (erf form) of its bf16 output "
                    "as a PyTorch operation into the down layer's input, the down layer"}
        configs["mlp_pair"]["fused_gelu_requant"] = {
            "up_fused_us": us("mlp_up_fused"), "down_gemm_us": us("mlp_down_gemm"), "pair_us": t_fused,
            "tflops": (svdq_flops(*MLP_UP) + svdq_flops(*MLP_DOWN)) / (t_fused * 1e-6) / 1e12,
            "speedup_vs_unfused_pair": t_pair / t_fused,
            "speedup_vs_unfused_pair_with_gelu": (t_pair + t_gelu) / t_fused,
            "note": "kernel 1 on X, the up GEMM with GELU and the down projection's activation pass in its "
                    "epilogue (kernels 6, 7), then the down GEMM: the 4608 x 12288 hidden state is never stored"}

    result = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms_max / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 codes, e4m3 scales per 16, fp32 accumulate); awq int4 x bf16",
        "data": "synthetic",
        "config": {
            "workload": "SVDQ W4A4 NVFP4 DiT attention projection M=4096 K=3072 N=3072 rank 32 group 16 "
                        "(kernel 1 chained into kernel 2)",
            "also_per_step": "each kernel of that layer alone; AWQ W4A16 adaLN K=3072 N=18432 group 64 at "
                             "M=1,2,4,8,16,32,64; SVDQ QKV K=3072 N=9216 at M=64,256,1024,4608,18432; "
                             "SVDQ MLP up 4608x3072->12288 and down 4608x12288->3072 (GELU inputs)",
            "l2": "every segment rotates over resident copies of inputs, weights and outputs touching "
                  "more than 2x L2 per cycle; no flush",
            "launch": ("one CUDA graph per segment holding exactly `steps` launches (or layers)" if use_graph
                       else "eager"),
            "parallelism": "replicas x%d" % world,
            "seed": 0,
        },
        "roofline": {
            "bound": "tensor", "achieved": k2_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
            "frac": k2_tflops / fp4_peak, "traffic": traffic,
            "traffic_unit": "bytes per launch (dram read + write)", "traffic_note": traffic_note,
            "kernel": "nvfp4_gemm_kernel<256> (attention M=4096 K=N=3072)",
            "peak_note": "dense FP4 = 4 x measured bf16 burst (%s), the nominal 9/2.25 ratio" % peaks["source"],
            "frac_clock_matched": k2_tflops / fp4_clock_peak,
            "clock_matched_peak": fp4_clock_peak,
            "clock_matched_note": "nominal dense FP4 issue rate (32768 FLOP per SM per clock) x %d SMs at the "
                                  "median sampled SM clock" % sms,
            "frac_of_9pf_datasheet": k2_tflops / 9000.0,
        },
        "kernels": {
            "quant_act_lowrank_kernel": {"us": us("attn_k1"), "bound": "hbm", "gbs": k1_gbs, "frac": k1_gbs / hbm,
                                         "bytes": k1_bytes(M, Kd)},
            "nvfp4_gemm_kernel": {"us": us("attn_k2"), "bound": "tensor", "tflops": k2_tflops,
                                  "frac": k2_tflops / fp4_peak, "flops": fl},
            "layer_chained": {"us": us("attn_layer"), "tflops": fl / (us("attn_layer") * 1e-6) / 1e12,
                              "frac_fp4": fl / (us("attn_layer") * 1e-6) / 1e12 / fp4_peak},
        },
        "configs": configs,
        "awq": {"value": awq_all, "unit": "GB/s", "frac_hbm": awq_all / hbm, "per_m": awq_per_m,
                "hbm_peak_gbs": hbm},
        "variants": {"svdq_dynamic_act_scale": time_dynamic_variant(P, wl, stream, K, use_graph)},
        "gpu_launches": launches,
        "clocks": clk,
    }
    del runs
    result["e2e"] = e2e_ours(args, P, wl.attn, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline()
    return result


def e2e_ours(args, P, case, dev, world, chunks=1):
    """The attention layer through the public API with the input in pinned host memory and
    the output read back to pinned host memory, every step inside the timed region.  The rows
    go in `chunks` pieces (one by default: each copy node of a graph has a fixed cost, and the
    overlap comes from consecutive steps) through three streams -- host-to-device copies, the
    two kernels, device-to-host copies -- so that both copy directions and the kernels overlap;
    consecutive steps alternate between two sets of device buffers, so a step's copy-in waits
    only for the kernels of the step before last.  The `e2e_steps` steps (copies, calls and their
    cross-stream order) are captured once into a CUDA graph and replayed: eager, the ≈ 80 host
    calls per step take longer than the step's transfers on the GPU."""
    import torch
    M, K, N = case.M, case.K, case.N
    assert case.nsets >= 2
    hX = case.sets[0]["X"].cpu().pin_memory()
    hY = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    rows = M // chunks
    assert rows % 128 == 0 and rows * chunks == M
    sc_per_row_block = (K // 64) * 512
    s_in, s_k, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [[torch.cuda.Event() for _ in range(chunks)] for _ in range(2)]
    ev_k1 = [[torch.cuda.Event() for _ in range(chunks)] for _ in range(2)]
    ev_k2 = [[torch.cuda.Event() for _ in range(chunks)] for _ in range(2)]
    ev_out = [[torch.cuda.Event() for _ in range(chunks)] for _ in range(2)]
    used = [False, False]                            # buffer set used by an earlier step (of this sequence)
    count = [0]

    def step():
        par = count[0] % 2
        s = case.sets[par]
        dX, codes, scales, U, Y = s["X"], s["codes"], s["scales"], s["U"], s["Y"]
        for c in range(chunks):
            r0, r1 = c * rows, (c + 1) * rows
            b0, b1 = (r0 // 128) * sc_per_row_block, (r1 // 128) * sc_per_row_block
            with torch.cuda.stream(s_in):
                if used[par]:
                    s_in.wait_event(ev_k1[par][c])    # kernel 1 of the step before last has read this chunk
                dX[r0:r1].copy_(hX[r0:r1], non_blocking=True)
                ev_in[par][c].record(s_in)
            with torch.cuda.stream(s_k):
                s_k.wait_event(ev_in[par][c])
                P.svdq_quantize_act_lowrank_down(dX[r0:r1], case.smooth, s["W"], case.g_a, RANK,
                                                 codes[r0:r1], scales[b0:b1], U[r0:r1])
                ev_k1[par][c].record(s_k)
                if used[par]:
                    s_k.wait_event(ev_out[par][c])    # the output of the step before last has left
                P.svdq_w4a4_nvfp4_linear(codes[r0:r1], scales[b0:b1], U[r0:r1], case.g_a, s["W"], case.g_w,
                                         rows, N, K, RANK, Y[r0:r1])
                ev_k2[par][c].record(s_k)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_k2[par][c])
                hY[r0:r1].copy_(Y[r0:r1], non_blocking=True)
                ev_out[par][c].record(s_out)
        used[par] = True
        count[0] += 1

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    used[0] = used[1] = False                        # no wait on the eager steps' events in the graph
    count[0] = 0
    with torch.cuda.graph(graph, stream=cap):
        fork = torch.cuda.Event()
        fork.record(cap)
        for s in (s_in, s_k, s_out):                 # every stream starts after the fork
            s.wait_event(fork)
        for _ in range(args.e2e_steps):
            step()
        for s in (s_in, s_k, s_out):                 # and the capture stream waits for all three
            join = torch.cuda.Event()
            join.record(s)
            cap.wait_event(join)
    with torch.cuda.stream(cap):
        graph.replay()                               # warm-up replay
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(cap):                     # replay() launches on the current stream
        e0.record(cap)
        graph.replay()
        e1.record(cap)
    torch.cuda.synchronize()
    ms = allreduce_max(e0.elapsed_time(e1), world)
    val = world * args.e2e_steps * svdq_flops(M, K, N) / (ms * 1e-3) / 1e12
    ok = bool(torch.equal(hY.to(dev), case.sets[(args.e2e_steps - 1) % 2]["Y"]))
    return {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": hX.numel() * 2,
            "d2h_bytes_per_step": hY.numel() * 2, "steps": args.e2e_steps, "ms_per_step": ms / args.e2e_steps,
            "note": "attention layer via the public API; pinned host X in, pinned host Y out, every step, "
                    "in %d row chunks over copy-in, kernel and copy-out streams, two device buffer sets in "
                    "alternation, the %d steps captured in one CUDA graph" % (chunks, args.e2e_steps),
            "host_output_matches_device": ok}


# ---------------------------------------------------------------- CPU oracle legs

def _oracle_layer_prepared():
    import synth
    from oracle import nvfp4, svdq
    M, K, N = ATTN
    w = synth.svdq_workload(M, K, N)
    cw, sw, gw = svdq.quantize_weights(w.R)                 # offline, like packing (untimed)
    wq = nvfp4.dequantize(cw, sw, gw)
    a = synth.awq_workload(max(AWQ_MS), AWQ_K, AWQ_N)
    return w, wq, a


def _oracle_svdq_rows(w, wq, rows):
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
    M, K, N = ATTN
    t = time.perf_counter()
    _oracle_svdq_rows(w, wq, M)
    dt = time.perf_counter() - t
    t = time.perf_counter()
    _oracle_awq_rows(a, 64, AWQ_N)
    da = time.perf_counter() - t
    return {"value": svdq_flops(M, K, N) / dt / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
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
    rows = int(max(1, min(ATTN[0], budget / per_row)))
    for _ in range(args.warmup):
        _oracle_svdq_rows(w, wq, rows)
    t = time.perf_counter()
    for _ in range(args.steps):
        _oracle_svdq_rows(w, wq, rows)
    dt = time.perf_counter() - t
    M, K, N = ATTN
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
    """Each kernel launched eagerly `steps` times on one resident copy of a workload (small
    enough for ncu captures): the attention layer and the AWQ layer, the QKV layer at M = 64,
    or the fused QKV layer at M = 4608."""
    import torch
    import bit_diffusion_transformer_act_b200 as P
    dev = torch.device("cuda", torch.cuda.current_device())
    l2 = 126 * 2 ** 20
    import synth
    if args.case == "attention":
        attn = SvdqCase(P, dev, synth.svdq_workload(*ATTN), ATTN[0], l2, nsets=1)
        awq = AwqCase(P, dev, l2, nsets=1)
        jobs = [("k1", lambda: attn.k1(P, 0)), ("k2", lambda: attn.k2(P, 0))] + \
               [("awq%d" % m, (lambda m=m: awq.run(P, 0, m))) for m in AWQ_MS]
    elif args.case == "qkv64":
        c = SvdqCase(P, dev, synth.svdq_workload(64, QKV_K, QKV_N), 64, l2, nsets=1)
        jobs = [("k1", lambda: c.k1(P, 0)), ("k2", lambda: c.k2(P, 0))]
    elif args.case == "qkv4608_fused":
        c = SvdqCase(P, dev, synth.svdq_workload(4608, QKV_K, QKV_N), 4608, l2, nsets=1)
        c.set_qkv(dev, QKV_HEADS, QKV_EPS)
        jobs = [("k2", lambda: c.k2(P, 0)), ("qkv_fused", lambda: c.qkv_fused(P, 0))]
    elif args.case == "int4":
        c = Int4Case(P, dev, synth.svdq_workload(*ATTN), ATTN[0], l2)
        jobs = [("int4_k1", lambda: c.k1(P, 0)), ("int4_k2", lambda: c.k2(P, 0))]
    else:
        up = SvdqCase(P, dev, synth.svdq_workload(*MLP_UP), MLP_UP[0], l2, nsets=1)
        down = SvdqCase(P, dev, synth.svdq_workload(*MLP_DOWN, gelu_input=True), MLP_DOWN[0], l2, nsets=1)
        f = MlpFused(P, dev, up, down)
        jobs = [("up_k2", lambda: up.k2(P, 0)), ("up_fused", lambda: f.up_fused(P, 0))]
    out = {}
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

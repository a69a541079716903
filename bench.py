#!/usr/bin/env python
"""Benchmark of the symmetric INT8 activation-quantized linear layer on B200.

Default workload (one "step" = the whole hot path of one block-wise W8A8 linear layer, the pages'
primary scheme): DeepSeek-R1 dense-MLP up-projection, X bf16 [M=16384, K=7168] (~N(0,1), 0.1% of
entries x50), W [N=18432, K=7168] (~N(0,0.02)) quantized in 128x128 blocks offline; per step:
online per-token-group activation quantization (i8q_quant_act_token_group) + block-wise INT8 GEMM
with per-slab dequantization and bf16 output (i8q_gemm_w8a8_block).  `value` is TOPS of that step.

The same JSON line carries `sub_results`: the other kernels of the metric ("quant-kernel GB/s & %
of HBM peak", decode GEMMs as GB/s), each timed in this run on its own configured shape: the
per-token-group quantizer of the default step, the channel-wise layer (MoE expert down-proj,
M = 4096 and M = 16), block-wise decode (M = 16, up and down), the offline FP8 requant and the
W8A16 decode GEMM (Qwen3-8B shapes, M = 16).  Other workloads are available with --workload.

Timing: W warm-up steps, then K steps back to back between CUDA events on the launching stream,
cycling through enough independent copies of every input and output that the working set of a
cycle exceeds twice the 126 MB L2 (no step reads what the previous one left in L2).  The timed
region holds only the steps' kernels, so a GEMM may overlap its start-up with the kernel before
it (programmatic dependent launch).  A second pass of K steps brackets every kernel with its own
events, which gives each kernel's average launch duration (the roofline figure).  With N > 1
(`--gpus N` spawns one process per GPU itself, or torchrun launches them) every rank runs the same
per-GPU workload on its own tokens (data-parallel, weights replicated, no collective on the data
path): weak scaling, value = all ranks' work / max-over-ranks time.

`--impl reference` times the CPU oracle (the plain C++ oracle the tests compare with, OpenMP over
all host cores) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 INT8 GEMM TOPS & % of B200 INT8 peak; quant-kernel GB/s & % of HBM peak"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 4.5 / 2.25      # nominal dense INT8 : BF16 tensor throughput on B200


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# DRAM bytes (read + written) per launch of the dominant kernel, from one ncu capture of this
# bench's own command (profiles/<file>.md), keyed by (workload, M, N, K).  A kernel change
# invalidates its entry: it must then be re-measured or removed (the line reports null).
MEASURED_TRAFFIC = {
    ("w8a8_block", 16384, 18432, 7168): (1371.3e6, "w8a8_block_up_m16384.md"),
    ("requant", 0, 18432, 7168): (208.5e6, "requant_fp8_block_n18432_k7168.md"),
    ("w8a16", 16, 12288, 4096): (51.29e6, "w8a16_m16_n12288_k4096.md"),
    ("w8a16", 16, 4096, 12288): (51.55e6, "w8a16_m16_n4096_k12288.md"),
}


def measured_traffic(workload: str, config: dict):
    key = (workload, config.get("M", 0), config.get("N"), config.get("K"))
    hit = MEASURED_TRAFFIC.get(key)
    return (hit[0], hit[1]) if hit else (None, None)


# ------------------------------------------------------------------- data-parallel host logic

def shard_seed(base: int, rank: int) -> int:
    """Seed of a rank's activations: every rank draws its own tokens; weights use `base` alone
    (replicated)."""
    return base + 1000 * rank


def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (a job ends when its slowest rank does)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput: the work of every rank's steps over the max-over-ranks time."""
    return units_per_step * steps * world / (ms / 1e3)


# ---------------------------------------------------------------------------------- workloads

class Workload:
    """One linear-layer hot path: buffers (R rotating copies) and the ordered kernel launches of a step."""

    name = ""
    unit = "TOPS"

    def __init__(self, args):
        self.args = args

    # subclasses fill: self.kernels (list of names), self.units_per_step, self.dominant, self.dom_units,
    # self.dom_bound, self.h2d_bytes, self.d2h_bytes, config dict


def _rotations(bytes_per_copy: int) -> int:
    return max(1, min(16, -(-2 * L2_BYTES // max(1, bytes_per_copy)) + 1))


def _scale_rows(run, lo: int, hi: int, budget_s: float) -> int:
    """Rows of an oracle sample that take about `budget_s` seconds: time `lo` rows, then scale."""
    dt = max(run(lo), 1e-4)
    return int(max(lo, min(hi, lo * budget_s / dt)))


def describe(name: str, args) -> dict:
    """Shapes, rotation count and the JSON `config` of a workload, from the arguments alone (no
    device buffers): the GPU arm and the reference arm report the same config."""
    world = getattr(args, "world", 1)
    if name == "w8a8_channel":
        M, N, K = args.M or 4096, 7168, 2048
        R = _rotations(M * K * 3 + 4 * M + N * K + 4 * N + 2 * M * N)
        config = {"workload": f"channel-wise W8A8 linear, DeepSeek-R1 MoE expert down-proj "
                              f"X[{M},{K}] W[{N},{K}] bf16 out; step = per-token act quant + INT8 GEMM",
                  "M": M, "N": N, "K": K, "global_batch": M * world, "seq_len": 1,
                  "parallelism": f"dp{world}", "l2": f"{R} rotating input/output copies (> 2x L2 per cycle)"}
    elif name == "w8a8_block":
        N, K = (18432, 7168) if args.proj == "up" else (7168, 18432)
        M = args.M or 16384
        KB, ld = K // 128, (M + 3) // 4 * 4
        R = _rotations(M * K * 3 + 4 * KB * ld + N * K + 2 * M * N)
        config = {"workload": f"block-wise W8A8 linear, DeepSeek-R1 dense MLP {args.proj}-proj X[{M},{K}] "
                              f"W[{N},{K}] bf16 out; step = per-token-group act quant + INT8 GEMM",
                  "M": M, "N": N, "K": K, "global_batch": M * world, "seq_len": 1,
                  "parallelism": f"dp{world}", "l2": f"{R} rotating input/output copies (> 2x L2 per cycle)"}
    elif name in ("moe_channel", "moe_block"):
        E, N, K = 32, 7168, 2048
        M = args.M or 8192
        R = 2
        scheme = "channel-wise" if name == "moe_channel" else "block-wise"
        config = {"workload": f"grouped (MoE) {scheme} W8A8, DeepSeek-R1 MoE expert down-proj: {E} experts "
                              f"W[{E},{N},{K}], {M} routed token rows X[{M},{K}] (ragged seeded counts) bf16 out; "
                              f"step = act quant + grouped INT8 GEMM",
                  "M": M, "N": N, "K": K, "experts": E, "global_batch": M * world, "seq_len": 1,
                  "parallelism": f"dp{world}", "l2": "2 rotating activation/output copies; 470 MB of weights"}
    elif name == "requant":
        M, N, K, R = 0, 18432, 7168, 2
        config = {"workload": f"offline FP8-E4M3 [{N},{K}] (128x128 fp32 scales) -> BF16 -> INT8 128x128 block requant",
                  "N": N, "K": K, "parallelism": f"dp{world}", "l2": "2 rotating copies of 264 MB"}
    elif name in ("w8a16", "w8a16_bf16"):
        M = args.M or 16
        N, K = (12288, 4096) if args.proj == "up" else (4096, 12288)
        R = _rotations(N * K + 2 * N * (K // 128) + 2 * M * K + 2 * M * N)
        dt = "bf16" if name == "w8a16_bf16" else "fp16"
        kind = "decode" if M <= 64 else "prefill"
        config = {"workload": f"W8A16 group-128 {kind} GEMM, Qwen3-8B linear X {dt}[{M},{K}] W int8[{N},{K}] "
                              f"{dt} out", "M": M, "N": N, "K": K, "global_batch": M * world,
                  "parallelism": f"dp{world}", "l2": f"{R} rotating copies (> 2x L2 per cycle)"}
    elif name == "w8a8_block_fused":
        N, K = (18432, 7168) if args.proj == "up" else (7168, 18432)
        M = args.M or 16
        R = _rotations(M * K * 2 + N * K + 2 * M * N)
        config = {"workload": f"block-wise W8A8 decode linear, DeepSeek-R1 dense MLP {args.proj}-proj X[{M},{K}] "
                              f"W[{N},{K}] bf16 out; step = one GEMM with the per-token-group act quant fused in",
                  "M": M, "N": N, "K": K, "global_batch": M * world, "seq_len": 1,
                  "parallelism": f"dp{world}", "l2": f"{R} rotating input/output copies (> 2x L2 per cycle)"}
    else:
        raise ValueError(name)
    return {"M": M, "N": N, "K": K, "R": R, "config": config}


class ChannelW8A8(Workload):
    name = "w8a8_channel"

    def __init__(self, args, rank=0):
        super().__init__(args)
        import torch
        from activation_quantized_gemm_b200 import i8q, synth
        self.q = i8q
        M, N, K = args.M or 4096, 7168, 2048
        self.M, self.N, self.K = M, N, K
        x = synth.activation_bf16(M, K, seed=shard_seed(1, rank), outlier_p=0.001, outlier_mult=50.0)
        w = synth.weight_bf16(N, K, seed=1)
        self.x_host = torch.from_numpy(x.view(np.int16)).pin_memory()
        per_copy = M * K * 3 + 4 * M + N * K + 4 * N + 2 * M * N
        self.R = _rotations(per_copy)
        dev = "cuda"
        wd = torch.from_numpy(w.view(np.int16)).to(dev)
        self.bufs = []
        for r in range(self.R):
            b = {
                "x": torch.from_numpy(x.view(np.int16)).to(dev),
                "xq": torch.empty((M, K), dtype=torch.int8, device=dev),
                "sx": torch.empty((M,), dtype=torch.float32, device=dev),
                "wq": torch.empty((N, K), dtype=torch.int8, device=dev),
                "sw": torch.empty((N,), dtype=torch.float32, device=dev),
                "y": torch.empty((M, N), dtype=torch.int16, device=dev),
            }
            i8q.i8q_quant_act_token(wd, b["wq"], b["sw"])        # offline: per-output-channel weights
            self.bufs.append(b)
        self.y_host = torch.empty((M, N), dtype=torch.int16).pin_memory()
        self.kernels = ["quant_act_token", "gemm_w8a8_channel"]
        self.units_per_step = 2.0 * M * N * K / 1e12            # tera-ops
        self.dominant = "gemm_w8a8_channel"
        self.dom_units = 2.0 * M * N * K / 1e12
        self.dom_bound = "tensor" if M >= 512 else "hbm"
        self.dom_bytes = M * K + 4 * M + N * K + 4 * N + 2 * M * N
        self.h2d_bytes = M * K * 2
        self.d2h_bytes = M * N * 2
        self.config = describe(self.name, args)["config"]

    def launch(self, i, k, stream):
        b = self.bufs[i % self.R]
        if k == 0:
            self.q.i8q_quant_act_token(b["x"], b["xq"], b["sx"], stream=stream)
        else:
            self.q.i8q_gemm_w8a8_channel(b["xq"], b["sx"], b["wq"], b["sw"], b["y"], stream=stream)

    def e2e_step(self, i, stream):
        b = self.bufs[i % self.R]
        b["x"].copy_(self.x_host, non_blocking=True)
        self.launch(i, 0, stream)
        self.launch(i, 1, stream)
        self.y_host.copy_(b["y"], non_blocking=True)

    def oracle_sample(self, budget_s):
        """The C++ oracle on a row subset of the same workload; returns (units, seconds, description)."""
        from oracle import ref_cpp as O
        from activation_quantized_gemm_b200 import synth
        w = synth.weight_bf16(self.N, self.K, seed=1)
        wq, sw = O.quant_act_token(w)                              # offline, not timed
        x = synth.activation_bf16(min(self.M, 1024), self.K, seed=1, outlier_p=0.001, outlier_mult=50.0)

        def run(rows):
            t0 = time.perf_counter()
            xq, sx = O.quant_act_token(x[:rows])
            O.gemm_w8a8_channel(xq, sx, wq, sw)
            return time.perf_counter() - t0
        rows = _scale_rows(run, 4, x.shape[0], budget_s)
        dt = run(rows)
        return 2.0 * rows * self.N * self.K / 1e12, dt, f"{rows} of {self.M} token rows (quant + GEMM), N={self.N}, K={self.K}"

    def sub_results(self):
        """Per-kernel figures of this workload: the per-token quantizer and the GEMM."""
        M, N, K = self.M, self.N, self.K
        return [("quant_act_token", f"a2 per-token act quant [{M},{K}]", "hbm", 3 * M * K + 4 * M),
                ("gemm_w8a8_channel", f"a5 channel-wise GEMM M={M} N={N} K={K}",
                 self.dom_bound, self.dom_units * 1e12 if self.dom_bound == "tensor" else self.dom_bytes)]


class BlockW8A8(Workload):
    name = "w8a8_block"

    def __init__(self, args, rank=0):
        super().__init__(args)
        import torch
        from activation_quantized_gemm_b200 import i8q, synth
        self.q = i8q
        proj = args.proj
        N, K = (18432, 7168) if proj == "up" else (7168, 18432)
        M = args.M or 16384
        self.M, self.N, self.K = M, N, K
        x = synth.activation_bf16(M, K, seed=shard_seed(2, rank), outlier_p=0.001, outlier_mult=50.0)
        w = synth.weight_bf16(N, K, seed=2)
        self.x_host = torch.from_numpy(x.view(np.int16)).pin_memory()
        KB = K // 128
        ld = (M + 3) // 4 * 4
        per_copy = M * K * 3 + 4 * KB * ld + N * K + 2 * M * N
        self.R = _rotations(per_copy)
        dev = "cuda"
        wd = torch.from_numpy(w.view(np.int16)).to(dev)
        self.bufs = []
        for r in range(self.R):
            b = {
                "x": torch.from_numpy(x.view(np.int16)).to(dev),
                "xq": torch.empty((M, K), dtype=torch.int8, device=dev),
                "sx": torch.empty((KB, ld), dtype=torch.float32, device=dev),
                "wq": torch.empty((N, K), dtype=torch.int8, device=dev),
                "sw": torch.empty(((N + 127) // 128, KB), dtype=torch.float32, device=dev),
                "y": torch.empty((M, N), dtype=torch.int16, device=dev),
            }
            i8q.i8q_quant_weight_block(wd, b["wq"], b["sw"])
            self.bufs.append(b)
        del wd
        self.y_host = torch.empty((M, N), dtype=torch.int16).pin_memory()
        self.kernels = ["quant_act_token_group", "gemm_w8a8_block"]
        self.units_per_step = 2.0 * M * N * K / 1e12
        self.dominant = "gemm_w8a8_block"
        self.dom_units = 2.0 * M * N * K / 1e12
        self.dom_bound = "tensor" if M >= 512 else "hbm"
        self.dom_bytes = M * K + 4 * M * KB + N * K + 4 * ((N + 127) // 128) * KB + 2 * M * N
        self.h2d_bytes = M * K * 2
        self.d2h_bytes = M * N * 2
        self.config = describe(self.name, args)["config"]

    def launch(self, i, k, stream):
        b = self.bufs[i % self.R]
        if k == 0:
            self.q.i8q_quant_act_token_group(b["x"], b["xq"], b["sx"], stream=stream)
        else:
            self.q.i8q_gemm_w8a8_block(b["xq"], b["sx"], b["wq"], b["sw"], b["y"], stream=stream)

    def e2e_step(self, i, stream):
        b = self.bufs[i % self.R]
        b["x"].copy_(self.x_host, non_blocking=True)
        self.launch(i, 0, stream)
        self.launch(i, 1, stream)
        self.y_host.copy_(b["y"], non_blocking=True)

    def oracle_sample(self, budget_s):
        from oracle import ref_cpp as O
        from activation_quantized_gemm_b200 import synth
        w = synth.weight_bf16(self.N, self.K, seed=2)
        wq, sw = O.quant_weight_block(w)                           # offline, not timed
        x = synth.activation_bf16(min(self.M, 256), self.K, seed=2, outlier_p=0.001, outlier_mult=50.0)

        def run(rows):
            t0 = time.perf_counter()
            xq, sx = O.quant_act_token_group(x[:rows])
            O.gemm_w8a8_block(xq, sx, wq, sw)
            return time.perf_counter() - t0
        rows = _scale_rows(run, 1, x.shape[0], budget_s)
        dt = run(rows)
        return 2.0 * rows * self.N * self.K / 1e12, dt, f"{rows} of {self.M} token rows (quant + GEMM), N={self.N}, K={self.K}"

    def sub_results(self):
        M, N, K = self.M, self.N, self.K
        KB = K // 128
        return [("quant_act_token_group", f"a1 per-token-group act quant [{M},{K}]", "hbm",
                 3 * M * K + 4 * M * KB),
                ("gemm_w8a8_block", f"a4 block-wise GEMM {self.args.proj}-proj M={M} N={N} K={K}",
                 self.dom_bound, self.dom_units * 1e12 if self.dom_bound == "tensor" else self.dom_bytes)]


class Requant(Workload):
    name = "requant"
    unit = "GB/s"

    def __init__(self, args, rank=0):
        super().__init__(args)
        import torch
        from activation_quantized_gemm_b200 import i8q, synth
        self.q = i8q
        N, K = 18432, 7168
        self.N, self.K = N, K
        w8, sf = synth.fp8_checkpoint(N, K, seed=3)
        dev = "cuda"
        self.R = 2
        self.bufs = []
        for r in range(self.R):
            self.bufs.append({
                "w8": torch.from_numpy(w8).to(dev), "sf": torch.from_numpy(sf).to(dev),
                "wq": torch.empty((N, K), dtype=torch.int8, device=dev),
                "sw": torch.empty(sf.shape, dtype=torch.float32, device=dev)})
        self.w8_host = torch.from_numpy(w8).pin_memory()
        self.wq_host = torch.empty((N, K), dtype=torch.int8).pin_memory()
        nbytes = N * K * 2 + 8 * sf.size
        self.kernels = ["requant_fp8_to_int8_block"]
        self.units_per_step = nbytes / 1e9
        self.dominant = "requant_fp8_to_int8_block"
        self.dom_units = nbytes / 1e9
        self.dom_bound = "hbm"
        self.dom_bytes = nbytes
        self.h2d_bytes = N * K
        self.d2h_bytes = N * K
        self.config = describe(self.name, args)["config"]

    def launch(self, i, k, stream):
        b = self.bufs[i % self.R]
        self.q.i8q_requant_fp8_to_int8_block(b["w8"], b["sf"], b["wq"], b["sw"], stream=stream)

    def e2e_step(self, i, stream):
        b = self.bufs[i % self.R]
        b["w8"].copy_(self.w8_host, non_blocking=True)
        self.launch(i, 0, stream)
        self.wq_host.copy_(b["wq"], non_blocking=True)

    def oracle_sample(self, budget_s):
        from oracle import ref_cpp as O
        from activation_quantized_gemm_b200 import synth
        w8, sf = synth.fp8_checkpoint(self.N, self.K, seed=3)

        def run(rows):
            rows128 = -(-rows // 128) * 128
            t0 = time.perf_counter()
            O.requant_fp8_to_int8_block(w8[:rows128], sf[:rows128 // 128])
            return time.perf_counter() - t0
        rows = _scale_rows(run, 128, self.N, budget_s)
        rows = -(-rows // 128) * 128
        dt = run(rows)
        return (rows * self.K * 2 + 8 * (rows // 128) * (self.K // 128)) / 1e9, dt, f"{rows} of {self.N} weight rows"

    def sub_results(self):
        return [("requant_fp8_to_int8_block", f"a3 FP8 -> BF16 -> INT8 block requant [{self.N},{self.K}]", "hbm",
                 self.dom_bytes)]


class W8A16(Workload):
    """W8A16 group-wise GEMM (Qwen3-8B linear shapes): fp16 or bf16 activations; decode batches are
    HBM-bound (GB/s), prefill batches (M > 256) tensor-bound against the 16-bit dense peak."""
    name = "w8a16"
    unit = "GB/s"

    def __init__(self, args, rank=0):
        super().__init__(args)
        import torch
        from activation_quantized_gemm_b200 import i8q, synth
        self.q = i8q
        self.bf16 = args.workload == "w8a16_bf16"
        self.name = args.workload
        M = args.M or 16
        N, K = (12288, 4096) if args.proj == "up" else (4096, 12288)
        self.M, self.N, self.K = M, N, K
        if self.bf16:
            x = synth.activation_bf16_plain(M, K, seed=shard_seed(4, rank))
            wq, s = synth.int8_weight_groups(N, K, seed=4, scale_fmt="bf16")
        else:
            x = synth.activation_f16(M, K, seed=shard_seed(4, rank))
            wq, s = synth.int8_weight_groups(N, K, seed=4)
        per_copy = N * K + 2 * N * (K // 128) + 2 * M * K + 2 * M * N
        self.R = _rotations(per_copy)
        dev = "cuda"
        self.bufs = []
        for r in range(self.R):
            self.bufs.append({
                "x": torch.from_numpy(x.view(np.int16)).to(dev), "wq": torch.from_numpy(wq).to(dev),
                "s": torch.from_numpy(s.view(np.int16)).to(dev),
                "y": torch.empty((M, N), dtype=torch.int16, device=dev)})
        self.x_host = torch.from_numpy(x.view(np.int16)).pin_memory()
        self.y_host = torch.empty((M, N), dtype=torch.int16).pin_memory()
        self.kernels = ["gemm_w8a16_group_bf16" if self.bf16 else "gemm_w8a16_group"]
        self.dominant = self.kernels[0]
        self.dom_bytes = per_copy
        if M > 256:                       # prefill: tensor-bound, TFLOP/s of the 16-bit MMAs
            self.unit = "TFLOP/s"
            self.units_per_step = 2.0 * M * N * K / 1e12
            self.dom_units = self.units_per_step
            self.dom_bound = "tensor16"
        else:
            self.units_per_step = per_copy / 1e9
            self.dom_units = per_copy / 1e9
            self.dom_bound = "hbm"
        self.h2d_bytes = 2 * M * K
        self.d2h_bytes = 2 * M * N
        self.config = describe(self.name, args)["config"]

    def launch(self, i, k, stream):
        b = self.bufs[i % self.R]
        if self.bf16:
            self.q.i8q_gemm_w8a16_group_bf16(b["x"], b["wq"], b["s"], b["y"], stream=stream)
        else:
            self.q.i8q_gemm_w8a16_group(b["x"], b["wq"], b["s"], b["y"], stream=stream)

    def e2e_step(self, i, stream):
        b = self.bufs[i % self.R]
        b["x"].copy_(self.x_host, non_blocking=True)
        self.launch(i, 0, stream)
        self.y_host.copy_(b["y"], non_blocking=True)

    def oracle_sample(self, budget_s):
        from oracle import ref_cpp as O
        from activation_quantized_gemm_b200 import synth
        bf16 = getattr(self, "bf16", False)
        Ms = min(self.M, 64)
        if bf16:
            x = synth.activation_bf16_plain(Ms, self.K, seed=4)
            wq, s = synth.int8_weight_groups(self.N, self.K, seed=4, scale_fmt="bf16")
        else:
            x = synth.activation_f16(Ms, self.K, seed=4)
            wq, s = synth.int8_weight_groups(self.N, self.K, seed=4)

        def run(rows):                       # rows of W (output channels)
            t0 = time.perf_counter()
            O.gemm_w8a16_group_fmt(x, wq[:rows], s[:rows], "bf16" if bf16 else "fp16")
            return time.perf_counter() - t0
        rows = _scale_rows(run, 64, self.N, budget_s)
        dt = run(rows)
        frac = rows / self.N * Ms / self.M
        return self.units_per_step * frac, dt, (f"{rows} of {self.N} weight rows x {Ms} of {self.M} tokens, "
                                                f"K={self.K}")

    def sub_results(self):
        dt = "bf16" if self.bf16 else "fp16"
        units = self.dom_units * 1e12 if self.dom_bound == "tensor16" else self.dom_bytes
        return [(self.kernels[0], f"a6 W8A16 GEMM ({dt}) M={self.M} N={self.N} K={self.K}", self.dom_bound, units)]


class FusedBlockW8A8(Workload):
    """Block-wise decode layer with the activation quantization inside the GEMM (one launch per
    step, i8q_gemm_w8a8_block_fused_quant); compare its step with the two-launch block workload."""
    name = "w8a8_block_fused"
    unit = "GB/s"

    def __init__(self, args, rank=0):
        super().__init__(args)
        import torch
        from activation_quantized_gemm_b200 import i8q, synth
        self.q = i8q
        d = describe(self.name, args)
        M, N, K = d["M"], d["N"], d["K"]
        self.M, self.N, self.K = M, N, K
        x = synth.activation_bf16(M, K, seed=shard_seed(2, rank), outlier_p=0.001, outlier_mult=50.0)
        w = synth.weight_bf16(N, K, seed=2)
        dev = "cuda"
        wd = torch.from_numpy(w.view(np.int16)).to(dev)
        self.R = d["R"]
        self.bufs = []
        for r in range(self.R):
            b = {"x": torch.from_numpy(x.view(np.int16)).to(dev),
                 "wq": torch.empty((N, K), dtype=torch.int8, device=dev),
                 "sw": torch.empty(((N + 127) // 128, K // 128), dtype=torch.float32, device=dev),
                 "y": torch.empty((M, N), dtype=torch.int16, device=dev)}
            i8q.i8q_quant_weight_block(wd, b["wq"], b["sw"])
            self.bufs.append(b)
        del wd
        self.x_host = torch.from_numpy(x.view(np.int16)).pin_memory()
        self.y_host = torch.empty((M, N), dtype=torch.int16).pin_memory()
        self.kernels = ["gemm_w8a8_block_fused_quant"]
        self.dom_bytes = 2 * M * K + N * K + 4 * ((N + 127) // 128) * (K // 128) + 2 * M * N
        self.units_per_step = self.dom_bytes / 1e9
        self.dominant = self.kernels[0]
        self.dom_units = self.units_per_step
        self.dom_bound = "hbm"
        self.h2d_bytes = M * K * 2
        self.d2h_bytes = M * N * 2
        self.config = d["config"]

    def launch(self, i, k, stream):
        b = self.bufs[i % self.R]
        self.q.i8q_gemm_w8a8_block_fused_quant(b["x"], b["wq"], b["sw"], b["y"], stream=stream)

    def e2e_step(self, i, stream):
        b = self.bufs[i % self.R]
        b["x"].copy_(self.x_host, non_blocking=True)
        self.launch(i, 0, stream)
        self.y_host.copy_(b["y"], non_blocking=True)

    def oracle_sample(self, budget_s):
        """The oracle's a1 then a4 for all M tokens on a subset of the weight rows; units are the
        step's bytes scaled by the fraction of the output computed."""
        from oracle import ref_cpp as O
        from activation_quantized_gemm_b200 import synth
        w = synth.weight_bf16(self.N, self.K, seed=2)
        wq, sw = O.quant_weight_block(w)                           # offline, not timed
        x = synth.activation_bf16(self.M, self.K, seed=2, outlier_p=0.001, outlier_mult=50.0)

        def run(rows):
            rows = -(-rows // 128) * 128
            t0 = time.perf_counter()
            xq, sx = O.quant_act_token_group(x)
            O.gemm_w8a8_block(xq, sx, wq[:rows], sw[: rows // 128])
            return time.perf_counter() - t0
        rows = _scale_rows(run, 128, self.N, budget_s)
        rows = min(self.N, -(-rows // 128) * 128)
        dt = run(rows)
        step_bytes = 2 * self.M * self.K + self.N * self.K + 2 * self.M * self.N
        return step_bytes * rows / self.N / 1e9, dt, f"{rows} of {self.N} weight rows, all {self.M} tokens (a1 + a4)"

    def sub_results(self):
        return [(self.kernels[0], f"a1 fused into a4, block-wise GEMM {self.args.proj}-proj M={self.M} "
                                  f"N={self.N} K={self.K}", "hbm", self.dom_bytes)]


class GroupedW8A8(Workload):
    """Grouped (MoE) W8A8 layer: 32 experts of the DeepSeek-R1 MoE down-proj shape, token rows
    sorted by expert with seeded ragged counts (some experts may get none); per step the routed
    rows are quantized and every expert's rows multiplied by that expert's weight."""
    name = "moe_channel"

    def __init__(self, args, rank=0):
        super().__init__(args)
        import torch
        from activation_quantized_gemm_b200 import i8q, synth
        self.q = i8q
        self.block = args.workload == "moe_block"
        self.name = args.workload
        d = describe(args.workload, args)
        E, M, N, K = d["config"]["experts"], d["M"], d["N"], d["K"]
        self.E, self.M, self.N, self.K = E, M, N, K
        KB = K // 128
        counts = synth.token_counts(E, M, seed=6)
        off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        x = synth.activation_bf16(M, K, seed=shard_seed(6, rank), outlier_p=0.001, outlier_mult=50.0)
        dev = "cuda"
        self.wq = torch.empty((E, N, K), dtype=torch.int8, device=dev)
        self.sw = (torch.empty((E, (N + 127) // 128, KB), dtype=torch.float32, device=dev) if self.block
                   else torch.empty((E, N), dtype=torch.float32, device=dev))
        for e in range(E):                                       # offline weight quantization
            wd = torch.from_numpy(synth.weight_bf16(N, K, seed=600 + e).view(np.int16)).to(dev)
            if self.block:
                i8q.i8q_quant_weight_block(wd, self.wq[e], self.sw[e])
            else:
                i8q.i8q_quant_act_token(wd, self.wq[e], self.sw[e])
        self.off = torch.from_numpy(off).to(dev)
        ld = (M + 3) // 4 * 4
        self.R = 2
        self.bufs = []
        for r in range(self.R):
            self.bufs.append({
                "x": torch.from_numpy(x.view(np.int16)).to(dev),
                "xq": torch.empty((M, K), dtype=torch.int8, device=dev),
                "sx": (torch.empty((KB, ld), dtype=torch.float32, device=dev) if self.block
                       else torch.empty((M,), dtype=torch.float32, device=dev)),
                "y": torch.empty((M, N), dtype=torch.int16, device=dev)})
        self.x_host = torch.from_numpy(x.view(np.int16)).pin_memory()
        self.y_host = torch.empty((M, N), dtype=torch.int16).pin_memory()
        qk = "quant_act_token_group" if self.block else "quant_act_token"
        gk = "gemm_w8a8_block_grouped" if self.block else "gemm_w8a8_channel_grouped"
        self.kernels = [qk, gk]
        self.units_per_step = 2.0 * M * N * K / 1e12
        self.dominant = gk
        self.dom_units = self.units_per_step
        self.dom_bound = "tensor"
        self.dom_bytes = M * K + E * N * K + 2 * M * N
        self.h2d_bytes = M * K * 2
        self.d2h_bytes = M * N * 2
        self.config = d["config"]

    def launch(self, i, k, stream):
        b = self.bufs[i % self.R]
        if k == 0:
            if self.block:
                self.q.i8q_quant_act_token_group(b["x"], b["xq"], b["sx"], stream=stream)
            else:
                self.q.i8q_quant_act_token(b["x"], b["xq"], b["sx"], stream=stream)
        elif self.block:
            self.q.i8q_gemm_w8a8_block_grouped(b["xq"], b["sx"], self.wq, self.sw, self.off, b["y"], stream=stream)
        else:
            self.q.i8q_gemm_w8a8_channel_grouped(b["xq"], b["sx"], self.wq, self.sw, self.off, b["y"], stream=stream)

    def e2e_step(self, i, stream):
        b = self.bufs[i % self.R]
        b["x"].copy_(self.x_host, non_blocking=True)
        self.launch(i, 0, stream)
        self.launch(i, 1, stream)
        self.y_host.copy_(b["y"], non_blocking=True)

    def oracle_sample(self, budget_s):
        from oracle import ref_cpp as O
        from activation_quantized_gemm_b200 import synth
        E, N, K = self.E, self.N, self.K
        counts = synth.token_counts(E, self.M, seed=6)
        off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
        e0 = int(np.argmax(counts))                              # a sample of one expert's rows
        w = synth.weight_bf16(N, K, seed=600 + e0)
        x = synth.activation_bf16(int(counts[e0]), K, seed=6, outlier_p=0.001, outlier_mult=50.0)
        wq, sw = O.quant_weight_block(w) if self.block else O.quant_act_token(w)

        def run(rows):
            t0 = time.perf_counter()
            if self.block:
                xq, sx = O.quant_act_token_group(x[:rows])
                O.gemm_w8a8_block_grouped(xq, sx, wq[None], sw[None], np.array([0, rows]))
            else:
                xq, sx = O.quant_act_token(x[:rows])
                O.gemm_w8a8_channel_grouped(xq, sx, wq[None], sw[None], np.array([0, rows]))
            return time.perf_counter() - t0
        rows = _scale_rows(run, 1, x.shape[0], budget_s)
        dt = run(rows)
        return 2.0 * rows * N * K / 1e12, dt, f"{rows} token rows of expert {e0} (quant + GEMM), N={N}, K={K}"

    def sub_results(self):
        M, N, K = self.M, self.N, self.K
        qk, gk = self.kernels
        qbytes = 3 * M * K + (4 * M * (K // 128) if self.block else 4 * M)
        return [(qk, f"act quant of the routed rows [{M},{K}]", "hbm", qbytes),
                (gk, f"grouped {'block' if self.block else 'channel'}-wise GEMM, {self.E} experts, "
                     f"M={M} N={N} K={K}", "tensor", self.dom_units * 1e12)]


WORKLOADS = {"w8a8_channel": ChannelW8A8, "w8a8_block": BlockW8A8, "requant": Requant, "w8a16": W8A16,
             "w8a16_bf16": W8A16, "moe_channel": GroupedW8A8, "moe_block": GroupedW8A8,
             "w8a8_block_fused": FusedBlockW8A8}


# ---------------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            p = [t.strip() for t in l.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------- main

def _measure(wl, steps: int, warmup: int, hold_ms: float, stream, barrier, clocks=None):
    """W warm-up steps, K timed steps back to back, then, for each kernel of the step, K launches of
    that kernel alone back to back between one event pair.  Returns (total_ms of the back-to-back
    step region, per-kernel mean launch ms).  (An event pair around every single launch would add
    about 5 us of event overhead to each: an empty kernel measures 6 us that way.)"""
    import torch
    from activation_quantized_gemm_b200 import i8q
    nk = len(wl.kernels)
    for i in range(warmup):
        for k in range(nk):
            wl.launch(i, k, stream)
    i8q.i8q_status_check()
    barrier()
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # Hold the stream with a device-side sleep (outside the timed region) while the host enqueues
    # all K steps, so that host launch overhead never leaves the GPU idle inside the timed region.
    # The timed region holds nothing but the steps' kernels: a GEMM may then overlap its start-up
    # with the tail of the kernel before it (programmatic dependent launch).
    torch.cuda._sleep(int(hold_ms * 1.9e6))
    t_start.record(stream)
    for i in range(steps):
        for k in range(nk):
            wl.launch(i, k, stream)
    t_end.record(stream)
    barrier()
    # Per-kernel durations: each kernel of the step on its own, K launches back to back (the inputs
    # of a later kernel are the outputs the earlier kernels left in the same rotating buffers).
    per_kernel_ms = []
    for k in range(nk):
        k0 = torch.cuda.Event(enable_timing=True)
        k1 = torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(hold_ms * 1.9e6))
        k0.record(stream)
        for i in range(steps):
            wl.launch(i, k, stream)
        k1.record(stream)
        barrier()
        per_kernel_ms.append(k0.elapsed_time(k1) / steps)
    if clocks is not None:
        clocks.stop()
    i8q.i8q_status_check()
    total_ms = t_start.elapsed_time(t_end)
    return total_ms, per_kernel_ms


def _figure(bound: str, units: float, ms: float, peaks) -> dict:
    """Throughput of `units` (ops for a tensor-bound kernel, bytes otherwise) in `ms`, and its
    fraction of the measured peak (INT8 for "tensor", 16-bit for "tensor16", HBM copy otherwise)."""
    if bound == "tensor":
        v = units / 1e12 / (ms / 1e3)
        peak = peaks["bf16_tflops"] * INT8_PER_BF16
        return {"value": round(v, 2), "unit": "TOPS", "frac": round(v / peak, 4)}
    if bound == "tensor16":
        v = units / 1e12 / (ms / 1e3)
        return {"value": round(v, 2), "unit": "TFLOP/s", "frac": round(v / peaks["bf16_tflops"], 4)}
    v = units / 1e9 / (ms / 1e3)
    return {"value": round(v, 1), "unit": "GB/s", "frac": round(v / peaks["hbm_gbs"], 4)}


# The sub-results of the default run: (name, workload, M, proj).  Each is the configured shape of
# one more kernel of the metric; all run on one GPU after the headline step.
SUB_WORKLOADS = [
    ("channel_m4096", "w8a8_channel", 4096, "up"),
    ("channel_m16", "w8a8_channel", 16, "up"),
    ("block_up_m16", "w8a8_block", 16, "up"),
    ("block_down_m16", "w8a8_block", 16, "down"),
    ("block_up_m16_fused", "w8a8_block_fused", 16, "up"),
    ("block_down_m16_fused", "w8a8_block_fused", 16, "down"),
    ("moe_channel_e32", "moe_channel", 8192, "up"),
    ("moe_block_e32", "moe_block", 8192, "up"),
    ("requant", "requant", 0, "up"),
    ("w8a16_m16_n12288", "w8a16", 16, "up"),
    ("w8a16_m16_n4096", "w8a16", 16, "down"),
    ("w8a16_bf16_m16_n12288", "w8a16_bf16", 16, "up"),
    ("w8a16_prefill_m2048_n12288", "w8a16", 2048, "up"),
    ("w8a16_bf16_prefill_m2048_n12288", "w8a16_bf16", 2048, "up"),
]


def _sub_entry(wl, total_ms: float, per_kernel_ms, steps: int, peaks) -> dict:
    """Per-kernel figures of one workload plus its back-to-back step."""
    out = {"config": wl.config["workload"], "kernels": {}}
    step_units = 0.0
    for (kname, label, bound, units) in wl.sub_results():
        ms = per_kernel_ms[wl.kernels.index(kname)]
        fig = _figure(bound, units, ms, peaks)
        out["kernels"][kname] = {"what": label, "us": round(ms * 1e3, 2), "bound": bound, **fig}
        step_units += units if bound == "hbm" else 0.0
    step_ms = total_ms / steps
    out["step_us"] = round(step_ms * 1e3, 2)
    if all(b == "hbm" for (_, _, b, _) in wl.sub_results()):
        fig = _figure("hbm", step_units, step_ms, peaks)
        out["step_GBps"], out["step_frac"] = fig["value"], fig["frac"]
    return out


def run_ours(args):
    import datetime
    import torch
    import torch.distributed as dist
    from activation_quantized_gemm_b200 import build
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    args.world = world
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=datetime.timedelta(seconds=300))
    if rank == 0 or world == 1:
        build.build()
    if world > 1:
        dist.barrier()
    wl = WORKLOADS[args.workload](args, rank)
    stream = torch.cuda.current_stream()
    nk = len(wl.kernels)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    total_ms, per_kernel_ms = _measure(wl, args.steps, args.warmup, args.hold_ms, stream, barrier, clocks)
    total_ms = max_over_ranks(total_ms, "cuda")

    # end to end through the public API: pinned host input -> device, step, result -> host
    for i in range(2):
        wl.e2e_step(i, stream)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(args.hold_ms * 1.9e6))
    e0.record(stream)
    for i in range(args.steps):
        wl.e2e_step(i, stream)
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, "cuda")

    peaks, src = load_peaks()
    subs = None
    if world == 1 and not args.no_sub:
        subs = {args.workload: _sub_entry(wl, total_ms, per_kernel_ms, args.steps, peaks)}
        main_cfg = (args.workload, wl.config.get("M", 0), args.proj)
        del wl.bufs
        torch.cuda.empty_cache()
        for (name, wname, M, proj) in SUB_WORKLOADS:
            if (wname, M, proj) == main_cfg:
                continue
            sargs = argparse.Namespace(**vars(args))
            sargs.M, sargs.proj, sargs.workload = M, proj, wname
            swl = WORKLOADS[wname](sargs, rank)
            t_ms, pk_ms = _measure(swl, args.sub_steps, args.warmup, args.hold_ms, stream, barrier)
            subs[name] = _sub_entry(swl, t_ms, pk_ms, args.sub_steps, peaks)
            del swl
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import ref_cpp
        units, secs, desc = wl.oracle_sample(args.cpu_budget)
        cpu = {"value": units / secs, "unit": wl.unit, "cores": ref_cpp.num_threads(), "kind": "oracle",
               "host_cores": os.cpu_count(),
               "sample": desc + f"; {secs:.2f} s of the plain C++ oracle (g++ -O2, OpenMP over "
                                f"{ref_cpp.num_threads()} threads)"}

    if rank == 0:
        dom_ms = per_kernel_ms[wl.kernels.index(wl.dominant)]
        if wl.dom_bound == "tensor":
            peak = peaks["bf16_tflops"] * INT8_PER_BF16
            achieved = wl.dom_units / (dom_ms / 1e3)
            unit = "TOPS"
            peak_note = f"INT8 dense = {src} burst bf16 {peaks['bf16_tflops']} TFLOP/s x {INT8_PER_BF16} (nominal ratio)"
        elif wl.dom_bound == "tensor16":
            peak = peaks["bf16_tflops"]
            achieved = wl.dom_units / (dom_ms / 1e3)
            unit = "TFLOP/s"
            peak_note = f"{src} burst bf16 dense (fp16 the same rate)"
        else:
            peak = peaks["hbm_gbs"]
            achieved = wl.dom_bytes / 1e9 / (dom_ms / 1e3)
            unit = "GB/s"
            peak_note = f"{src} HBM copy bandwidth"
        traffic, traffic_src = measured_traffic(args.workload, wl.config)
        if args.traffic is not None:
            traffic, traffic_src = args.traffic, "--traffic"
        elif traffic is not None:
            traffic_src = f"ncu dram__bytes_read.sum + dram__bytes_write.sum, profiles/{traffic_src}"
        value = job_throughput(wl.units_per_step, args.steps, world, total_ms)
        e2e_value = job_throughput(wl.units_per_step, args.steps, world, e2e_ms)
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": wl.unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic (seeded, shapes of the DeepSeek-R1 / Qwen3-8B layers; random weights)",
            "config": wl.config,
            "kernels_ms": {k: round(v, 5) for k, v in zip(wl.kernels, per_kernel_ms)},
            "roofline": {"bound": wl.dom_bound, "kernel": wl.dominant, "achieved": round(achieved, 2),
                         "peak": round(peak, 1), "unit": unit, "frac": round(achieved / peak, 4),
                         "traffic": traffic, "traffic_source": traffic_src, "peak_source": peak_note},
            "e2e": {"value": round(e2e_value, 3), "unit": wl.unit, "h2d_bytes_per_step": wl.h2d_bytes,
                    "d2h_bytes_per_step": wl.d2h_bytes},
            "gpu_launches": nk * args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
        }
        if subs is not None:
            line["sub_results"] = subs
            line["sub_results_note"] = (
                "each entry timed in this run after the headline (its own warm-up and "
                f"{args.sub_steps} steps, rotating >2x L2 of inputs); us = mean launch time of that kernel "
                "alone, back to back between one event pair; frac = of the measured HBM copy peak, the "
                "INT8 dense peak (bf16 burst x 2) or the bf16 peak; step_us = back-to-back step of all its "
                "kernels (launches overlap through programmatic dependent launch)")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The CPU oracle as the reference arm: K timed steps, each a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(max(1, args.gpus))))
    if rank != 0:
        return
    args.world = world
    from oracle import ref_cpp

    cls = WORKLOADS[args.workload]
    wl = cls.__new__(cls)
    wl.args = args
    # shapes only (no device buffers); the config is the GPU arm's
    d = describe(args.workload, args)
    wl.M, wl.N, wl.K = d["M"], d["N"], d["K"]
    cfg = d["config"]
    if cls is W8A16:
        wl.bf16 = args.workload == "w8a16_bf16"
        if wl.M > 256:
            wl.unit = "TFLOP/s"
            wl.units_per_step = 2.0 * wl.M * wl.N * wl.K / 1e12
        else:
            wl.units_per_step = (wl.N * wl.K + 2 * wl.N * (wl.K // 128) + 2 * wl.M * wl.K + 2 * wl.M * wl.N) / 1e9
    if cls is GroupedW8A8:
        wl.E, wl.block = cfg["experts"], args.workload == "moe_block"
    budget = max(0.5, min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        wl.oracle_sample(budget)
    tot_u, tot_s, desc = 0.0, 0.0, ""
    for _ in range(args.steps):
        u, s, desc = wl.oracle_sample(budget)
        tot_u += u
        tot_s += s
    v = tot_u / tot_s
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": wl.unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64/fp64",
            "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": round(v, 6), "unit": wl.unit, "cores": ref_cpp.num_threads(),
                             "host_cores": os.cpu_count(), "kind": "oracle",
                             "sample": desc + " per step; the plain C++ oracle (OpenMP)"},
            "e2e": {"value": round(v, 6), "unit": wl.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _spawned_rank(rank: int, args, world: int, port: int):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    run_ours(args)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="w8a8_block")
    ap.add_argument("--M", type=int, default=0, help="token rows (default: the workload's headline M)")
    ap.add_argument("--proj", choices=["up", "down"], default="up")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="skip the per-kernel sub-results")
    ap.add_argument("--sub-steps", type=int, default=20)
    ap.add_argument("--hold-ms", type=float, default=50.0,
                    help="device-side sleep enqueued before each timed region so the host runs ahead")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the dominant kernel from an ncu capture (reported as given)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU, spawned here (torchrun sets WORLD_SIZE itself and skips this)
        import torch.multiprocessing as mp
        mp.spawn(_spawned_rank, args=(args, args.gpus, _free_port()), nprocs=args.gpus, join=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

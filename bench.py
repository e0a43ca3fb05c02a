#!/usr/bin/env python3
"""Benchmark of the quantized-matmul hot path on B200.

One step = one pass over the two headline workloads, each through the C ABI
with its inputs resident in HBM:
  * INT8 GEMM 8192x8192x8200 (row-major A with lda 8200, za = 7; B pre-packed
    once, symmetric, per-column Q31 requant, bias, clamp) -> int8 C
  * A8W4 GEMV 1x14336x4096 (f32 x quantized per row inside the kernel, int4
    group-32 weights pre-packed once) -> f32 y
value = integer ops of both (2 per MAC) / step time, in TOPS, whole job.
Per-part numbers (GEMM TOPS, GEMV HBM GB/s) and each kernel's fraction of the
measured roofline are on the same JSON line.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and cudaDeviceSynchronize on both sides, CUDA events on the launching stream,
max over ranks.  The K timed steps (C-ABI calls) are captured once into a
CUDA graph and replayed, so Python/ctypes launch cost stays out of the kernel
numbers.  Per-call and per-kernel times come from graphs of back-to-back
calls of one part lasting at least 8 ms (up to 200 calls, at least K),
replayed 5 times after idle pauses, median reported: graph start-up is spread
over hundreds of the microsecond calls whatever K is, and each replay is a
burst, not a power-capped loop.  The end-to-end leg is eager (no graph):
each step copies its inputs in from pinned host memory, calls the API and
copies its result out; it is timed serially on one stream and with
consecutive steps pipelined over three streams (copy-in, kernels,
copy-out), and the faster schedule is reported with both figures.  L2 (126 MB) is defeated by rotating input sets larger than it: 2
GEMM sets (A + packed B = 135 MB each) and 8 GEMV weight sets (36.8 MB each,
295 MB in all).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--workload headline|<one workload name below>] [--no-cpu-baseline]
Workloads: int8_gemm_130x70x129, int8_conv_56x56x64_3x3, a8w4_gemv_1x14336x4096,
a8w4_gemv_bf16s_1x14336x4096 (bf16 group scales), a8w4_gemv_actblock_1x14336x4096
(activations quantized per 32-wide K block), a8w4_gemv_asym_1x14336x4096
(asymmetric int4 weights), a8w4_gemm_128x4096x4096,
int8_gemm_8192x8192x8200, a8w4_conv_f32_56x56x64_3x3 and
a8w4_conv_f32_sym_56x56x64_3x3 (float-input conv, unrolled rows quantized
per output pixel, asymmetric or symmetric).
Under torchrun each rank runs the same work on its own GPU (replicas: the
path has no exchange step), and value sums all ranks' work.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "INT8 GEMM TOPS and A8W4 GEMV HBM GB/s, as % of B200 roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 vs 2.25 PFLOPS bf16)
NOMINAL_INT8_TOPS = 4500.0  # B200 dense int8 spec figure, reported beside the measured-derived peak
PART_CALLS = 200     # most calls per per-part timing graph
PART_GRAPH_MS = 8.0  # a per-part graph lasts at least this long (or PART_CALLS calls)
PART_REPLAYS = 5     # replays per per-part graph, each after an idle pause (median reported)


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# Algorithmic work per call (what the method must move / compute)
# ---------------------------------------------------------------------------
def gemm_ops(M, N, K):
    return 2.0 * M * N * K


def gemm_bytes(M, N, K):
    # A, B, C int8 + bias/multiplier/shift int32 per column
    return M * K + K * N + M * N + 3 * 4 * N


def a8w4_bytes(M, N, K, scale_bytes=4):
    # int4 nibbles + group scales (f32, or bf16) + f32 x + f32 bias + f32 y
    return N * K // 2 + N * (K // 32) * scale_bytes + M * K * 4 + N * 4 + M * N * 4


def a8w4_ops(M, N, K):
    return 2.0 * M * N * K


# ---------------------------------------------------------------------------
# Distributed plumbing (replicas; one process per GPU)
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self, want):
        import torch
        self.torch = torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        if want and want != self.world and self.rank == 0:
            print(f"# note: --gpus {want} but WORLD_SIZE={self.world}", file=sys.stderr)

    def barrier(self):
        if self.pg:
            if self.torch.cuda.is_available():
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, v):
        if not self.pg:
            return v
        dev = "cuda" if self.torch.cuda.is_available() else "cpu"
        t = self.torch.tensor([float(v)], dtype=self.torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = str(gpu_index)
        self.proc = None
        self.path = os.path.join("/tmp", f"qg_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.idx, f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(load), "power_w_max": max(r[2] for r in rows), "reasons": reasons}


# ---------------------------------------------------------------------------
# Workload setup on the GPU
# ---------------------------------------------------------------------------
def dev(a, torch):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


class GemmCase:
    """INT8 GEMM (weights pre-packed), `sets` rotating input sets."""

    def __init__(self, qg, torch, w, sets):
        self.M, self.N, self.K = w["M"], w["N"], w["K"]
        self.qg, self.torch = qg, torch
        ratios = np.atleast_1d(w["ratio"])
        params = [qg.qg_requant_params(float(r)) for r in ratios]
        per_channel = ratios.size > 1
        self.inputs = []
        B0 = dev(w["B"], torch)[:, :self.N]
        for s in range(sets):
            # distinct sets (same distributions): rotate A along K and B along K
            A = dev(w["A"], torch)[:, :self.K] if s == 0 else torch.roll(self.inputs[0][0], shifts=s, dims=1)
            B = B0 if s == 0 else torch.roll(B0, shifts=s, dims=0)
            self.inputs.append((A, qg.qgemm_pack_b_s8(B)))
        del B0, B
        if per_channel:
            mult = dev(np.array([p[0] for p in params], np.int32), torch)
            shift = dev(np.array([p[1] for p in params], np.int32), torch)
        else:
            mult, shift = params[0]
        self.bias = None if w["bias"] is None else dev(w["bias"], torch)
        self.rq = qg.make_requant(a_zero_point=w["za"], b_zero_point=w["zb"], bias=self.bias,
                                  multiplier=mult, shift=shift, out_zero_point=w["out_zp"],
                                  clamp_min=w["clamp_min"], clamp_max=w["clamp_max"])
        self.C = torch.empty((self.M, self.N), dtype=torch.int8, device="cuda")
        self.ws = torch.empty(max(qg.qgemm_s8s8_packed_workspace_bytes(self.M, self.K), 1),
                              dtype=torch.uint8, device="cuda")
        # a staging pass runs before the GEMM for row sums (zb != 0) or when A's
        # rows are not 16-byte addressable (copied to a 16-byte pitch)
        self.launches = 1 + (1 if (w["lda"] % 16 or w["zb"]) else 0)
        # the library's choice: CTA pairs for M > 256, or for M > 128 when
        # 128 x 256 one-CTA tiles would take more than one wave of SMs
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        one_cta_tiles = -(-self.M // 128) * -(-self.N // 256)
        pairs = self.M > 128 and (self.M > 256 or one_cta_tiles > sms)
        self.kernel = "i8gemm_tc2_kernel" if pairs else "i8gemm_tc_kernel"
        self.h2d_host = torch.from_numpy(np.ascontiguousarray(w["A"])).pin_memory()
        self.d2h_host = torch.empty((self.M, self.N), dtype=torch.int8).pin_memory()

    def run(self, i, stream=None):
        A, pb = self.inputs[i % len(self.inputs)]
        self.qg.qgemm_s8s8_requant_packed(A, pb, self.N, self.C, self.rq, K=self.K,
                                          workspace=self.ws, stream=stream)

    # The GEMM kernel alone on A copied once to a 16-byte row pitch (both
    # operands by tensor copies; zb == 0: no row sums either).

    def has_kernel_only(self):
        return self.launches > 1

    def prep_kernel_only(self):
        torch = self.torch
        Kp = (self.K + 15) // 16 * 16
        self.kernel_inputs = []
        for A, pb in self.inputs:
            Aal = torch.zeros((self.M, Kp), dtype=torch.int8, device="cuda")
            Aal[:, :self.K].copy_(A)
            self.kernel_inputs.append((Aal[:, :self.K], pb))

    def run_kernel(self, i, stream=None):
        A, pb = self.kernel_inputs[i % len(self.kernel_inputs)]
        self.qg.qgemm_s8s8_requant_packed(A, pb, self.N, self.C, self.rq, K=self.K,
                                          workspace=self.ws, stream=stream)

    def release_kernel_only(self):
        self.kernel_inputs = None

    def prep_e2e(self):
        torch = self.torch
        self.e2e_in = [torch.empty(tuple(self.h2d_host.shape), dtype=torch.int8, device="cuda")
                       for _ in range(2)]
        self.e2e_out = [torch.empty_like(self.C) for _ in range(2)]

    def e2e_compute(self, slot, stream):
        A, pb = self.inputs[0]
        self.qg.qgemm_s8s8_requant_packed(self.e2e_in[slot][:, :self.K], pb, self.N,
                                          self.e2e_out[slot], self.rq, K=self.K,
                                          workspace=self.ws, stream=stream)

    def ops(self):
        return gemm_ops(self.M, self.N, self.K)

    def bytes(self):
        return gemm_bytes(self.M, self.N, self.K)

    def h2d(self):
        return self.h2d_host.numel()

    def d2h(self):
        return self.d2h_host.numel()


class A8W4Case:
    def __init__(self, qg, torch, w, sets, bf16_scales=False, actblock=False, asym=False):
        self.M, self.N, self.K = w["M"], w["N"], w["K"]
        self.qg, self.torch = qg, torch
        self.bf16 = bf16_scales
        self.actblock = actblock  # activations quantized per 32-wide K block
        self.asym = asym          # asymmetric int4 weights: an f32 zero per group
        qw = dev(w["qw"], torch)
        sw = dev(w["sw"], torch)
        self.packed = []
        for s in range(sets):
            # distinct weight sets: rotate the int4 codes along K (still in [-8,7])
            src = qw if s == 0 else torch.roll(qw, shifts=32 * s, dims=1)
            if asym:
                zw = sw * torch.empty_like(sw).uniform_(-8.0, 8.0, generator=torch.Generator(
                    device=sw.device).manual_seed(77 + s))
                self.packed.append(qg.pack_w4_g32_asym(src, sw, zw))
            else:
                self.packed.append(qg.pack_w4_g32(src, sw, bf16_scales=bf16_scales))
        del qw
        self.x = dev(w["x"], torch)
        self.bias = None if w["bias"] is None else dev(w["bias"], torch)
        self.lo, self.hi = w["clamp_min"], w["clamp_max"]
        self.y = torch.empty((self.M, self.N), dtype=torch.float32, device="cuda")
        wsb = qg.qgemm_a8w4_workspace_bytes(self.M, self.N, self.K)
        self.ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda") if wsb else None
        self.launches = 1 if self.M == 1 else 2
        self.kernel = "a8w4_gemv_stream_kernel" if self.M == 1 else "a8w4_tc_kernel"
        self.h2d_host = torch.from_numpy(np.ascontiguousarray(w["x"])).pin_memory()
        self.d2h_host = torch.empty((self.M, self.N), dtype=torch.float32).pin_memory()

    def run(self, i, stream=None):
        if self.asym:
            self.qg.qgemm_a8w4_f32_asym(self.x, self.packed[i % len(self.packed)], self.N,
                                        self.bias, self.lo, self.hi, self.y, workspace=self.ws,
                                        stream=stream)
            return
        if self.actblock:
            self.qg.qgemm_a8w4_f32_actblock(self.x, self.packed[i % len(self.packed)], self.N,
                                            self.bias, self.lo, self.hi, self.y,
                                            workspace=self.ws, stream=stream)
            return
        self.qg.qgemm_a8w4_f32(self.x, self.packed[i % len(self.packed)], self.N, self.bias,
                               self.lo, self.hi, self.y, workspace=self.ws, stream=stream,
                               bf16_scales=self.bf16)

    def prep_e2e(self):
        torch = self.torch
        self.e2e_in = [torch.empty(tuple(self.h2d_host.shape), dtype=torch.float32, device="cuda")
                       for _ in range(2)]
        self.e2e_out = [torch.empty_like(self.y) for _ in range(2)]

    def e2e_compute(self, slot, stream):
        x, y = self.e2e_in[slot], self.e2e_out[slot]
        if self.asym:
            self.qg.qgemm_a8w4_f32_asym(x, self.packed[0], self.N, self.bias, self.lo, self.hi, y,
                                        workspace=self.ws, stream=stream)
        elif self.actblock:
            self.qg.qgemm_a8w4_f32_actblock(x, self.packed[0], self.N, self.bias, self.lo, self.hi,
                                            y, workspace=self.ws, stream=stream)
        else:
            self.qg.qgemm_a8w4_f32(x, self.packed[0], self.N, self.bias, self.lo, self.hi, y,
                                   workspace=self.ws, bf16_scales=self.bf16, stream=stream)

    def ops(self):
        return a8w4_ops(self.M, self.N, self.K)

    def bytes(self):
        zeros = self.N * (self.K // 32) * 4 if self.asym else 0
        return a8w4_bytes(self.M, self.N, self.K, 2 if self.bf16 else 4) + zeros

    def h2d(self):
        return self.h2d_host.numel() * 4

    def d2h(self):
        return self.d2h_host.numel() * 4


class ConvCase:
    def __init__(self, qg, torch, w, sets):
        self.qg, self.torch, self.w = qg, torch, w
        ratios = w["ratio"]
        params = [qg.qg_requant_params(float(r)) for r in ratios]
        self.mult = dev(np.array([p[0] for p in params], np.int32), torch)
        self.shift = dev(np.array([p[1] for p in params], np.int32), torch)
        self.bias = dev(w["bias"], torch)
        self.rq = qg.make_requant(a_zero_point=w["za"], bias=self.bias, multiplier=self.mult,
                                  shift=self.shift, out_zero_point=w["out_zp"],
                                  clamp_min=w["clamp_min"], clamp_max=w["clamp_max"])
        self.x = dev(w["x"], torch)
        # distinct images (the input shifted along W), together larger than L2
        self.inputs = [self.x if k == 0 else torch.roll(self.x, shifts=k, dims=2)
                       for k in range(sets)]
        self.wt = dev(w["w"], torch)
        OH, OW = qg.conv_out_hw(w["H"], w["W"], w["KH"], w["KW"], w["stride"], w["pad"])
        self.y = torch.empty((w["Nb"], OH, OW, w["Cout"]), dtype=torch.int8, device="cuda")
        self.M, self.N, self.K = w["Nb"] * OH * OW, w["Cout"], w["KH"] * w["KW"] * w["Cin"]
        # weights packed once (weights-stationary); each call is one launch
        self.packed = qg.qconv2d_s8_pack_w(self.wt)
        self.launches = 1
        self.kernel = "i8gemm_tc_kernel"
        self.h2d_host = torch.from_numpy(np.ascontiguousarray(w["x"])).pin_memory()
        self.d2h_host = torch.empty(tuple(self.y.shape), dtype=torch.int8).pin_memory()

    def run(self, i, stream=None):
        self.qg.qconv2d_s8_im2col_packed(self.inputs[i % len(self.inputs)], self.packed,
                                         self.wt.shape, self.y, self.rq,
                                         self.w["stride"], self.w["pad"], stream=stream)

    def prep_e2e(self):
        self.e2e_in = [self.torch.empty_like(self.x) for _ in range(2)]
        self.e2e_out = [self.torch.empty_like(self.y) for _ in range(2)]

    def e2e_compute(self, slot, stream):
        self.qg.qconv2d_s8_im2col_packed(self.e2e_in[slot], self.packed, self.wt.shape,
                                         self.e2e_out[slot], self.rq, self.w["stride"],
                                         self.w["pad"], stream=stream)

    def ops(self):
        return gemm_ops(self.M, self.N, self.K)

    def bytes(self):
        w = self.w
        return self.x.numel() + self.wt.numel() + self.y.numel() + 3 * 4 * self.N

    def h2d(self):
        return self.h2d_host.numel()

    def d2h(self):
        return self.d2h_host.numel()


class DynConvCase:
    """Float-input conv: every unrolled row quantized on the fly, int4 weights."""

    def __init__(self, qg, torch, w, sets, symmetric=False):
        self.qg, self.torch, self.w, self.sym = qg, torch, w, symmetric
        self.Cout, self.K = w["Cout"], w["K"]
        self.packed = qg.pack_w4_g32(dev(w["qw"].reshape(self.Cout, self.K), torch),
                                     dev(w["sw"], torch))
        x = dev(w["x"], torch)
        # distinct images (the input shifted along W), together larger than L2
        self.inputs = [x if s == 0 else torch.roll(x, shifts=s, dims=2) for s in range(sets)]
        self.bias = dev(w["bias"], torch)
        self.OH, self.OW = qg.conv_out_hw(w["H"], w["W"], w["KH"], w["KW"], w["stride"], w["pad"])
        self.P = w["Nb"] * self.OH * self.OW
        self.y = torch.empty((w["Nb"], self.OH, self.OW, self.Cout), dtype=torch.float32,
                             device="cuda")
        wsb = qg.qconv2d_f32_dyn_a8w4_workspace_bytes(x.shape, self.Cout, w["KH"], w["KW"],
                                                      w["stride"], w["pad"])
        self.ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        self.launches = 2        # unroll + quantize into bf16 tiles, then the tensor-core GEMM
        self.kernel = "a8w4_tc_kernel"
        self.h2d_host = torch.from_numpy(np.ascontiguousarray(w["x"])).pin_memory()
        self.d2h_host = torch.empty(tuple(self.y.shape), dtype=torch.float32).pin_memory()

    def _call(self, x, stream=None, y=None):
        w = self.w
        self.qg.qconv2d_f32_dyn_a8w4(x, self.packed, self.Cout, w["KH"], w["KW"], w["stride"],
                                     w["pad"], self.bias, w["clamp_min"], w["clamp_max"],
                                     self.y if y is None else y, symmetric=self.sym,
                                     workspace=self.ws, stream=stream)

    def run(self, i, stream=None):
        self._call(self.inputs[i % len(self.inputs)], stream)

    def prep_e2e(self):
        self.e2e_in = [self.torch.empty_like(self.inputs[0]) for _ in range(2)]
        self.e2e_out = [self.torch.empty_like(self.y) for _ in range(2)]

    def e2e_compute(self, slot, stream):
        self._call(self.e2e_in[slot], stream, self.e2e_out[slot])

    def ops(self):
        return a8w4_ops(self.P, self.Cout, self.K)

    def bytes(self):
        # f32 image + int4 nibbles + f32 group scales + f32 bias + f32 output
        return (self.inputs[0].numel() * 4 + self.Cout * self.K // 2
                + self.Cout * (self.K // 32) * 4 + self.Cout * 4 + self.P * self.Cout * 4)

    def h2d(self):
        return self.h2d_host.numel() * 4

    def d2h(self):
        return self.d2h_host.numel() * 4


WORKLOAD_NAMES = ["headline", "int8_gemm_130x70x129", "int8_conv_56x56x64_3x3",
                  "a8w4_gemv_1x14336x4096", "a8w4_gemv_bf16s_1x14336x4096",
                  "a8w4_gemv_actblock_1x14336x4096", "a8w4_gemv_asym_1x14336x4096",
                  "a8w4_gemm_actblock_128x4096x4096", "a8w4_gemm_asym_128x4096x4096",
                  "a8w4_gemm_128x4096x4096", "int8_gemm_8192x8192x8200",
                  "a8w4_conv_f32_56x56x64_3x3", "a8w4_conv_f32_sym_56x56x64_3x3"]


def build_cases(workload, qg, torch):
    import workloads as W
    if workload == "headline":
        return [("int8_gemm_8192x8192x8200", GemmCase(qg, torch, W.int8_gemm_8192x8192x8200(), 2), "tensor"),
                ("a8w4_gemv_1x14336x4096", A8W4Case(qg, torch, W.a8w4_gemv_1x14336x4096(), 8), "hbm")]
    if workload == "int8_gemm_130x70x129":
        return [("int8_gemm_130x70x129", GemmCase(qg, torch, W.int8_gemm_130x70x129(), 1), "latency")]
    if workload == "int8_conv_56x56x64_3x3":
        # 700 input images of 200 KB: 140 MB > L2
        return [("int8_conv_56x56x64_3x3", ConvCase(qg, torch, W.int8_conv_56x56x64_3x3(), 700), "latency")]
    if workload == "a8w4_gemv_1x14336x4096":
        return [("a8w4_gemv_1x14336x4096", A8W4Case(qg, torch, W.a8w4_gemv_1x14336x4096(), 8), "hbm")]
    if workload == "a8w4_gemm_128x4096x4096":
        return [("a8w4_gemm_128x4096x4096", A8W4Case(qg, torch, W.a8w4_gemm_128x4096x4096(), 16), "tensor_bf16")]
    if workload == "a8w4_gemv_asym_1x14336x4096":   # asymmetric int4 weights (44 MB per set)
        return [("a8w4_gemv_asym_1x14336x4096",
                 A8W4Case(qg, torch, W.a8w4_gemv_1x14336x4096(), 7, asym=True), "hbm")]
    if workload == "a8w4_gemm_actblock_128x4096x4096":
        return [("a8w4_gemm_actblock_128x4096x4096",
                 A8W4Case(qg, torch, W.a8w4_gemm_128x4096x4096(), 16, actblock=True), "tensor_bf16")]
    if workload == "a8w4_gemm_asym_128x4096x4096":
        return [("a8w4_gemm_asym_128x4096x4096",
                 A8W4Case(qg, torch, W.a8w4_gemm_128x4096x4096(), 12, asym=True), "tensor_bf16")]
    if workload == "a8w4_gemv_actblock_1x14336x4096":   # activations quantized per K block
        return [("a8w4_gemv_actblock_1x14336x4096",
                 A8W4Case(qg, torch, W.a8w4_gemv_1x14336x4096(), 8, actblock=True), "hbm")]
    if workload == "a8w4_gemv_bf16s_1x14336x4096":   # the GEMV with bf16 group scales (9 sets: 298 MB > L2)
        return [("a8w4_gemv_bf16s_1x14336x4096", A8W4Case(qg, torch, W.a8w4_gemv_1x14336x4096(), 9, True), "hbm")]
    if workload == "int8_gemm_8192x8192x8200":
        return [("int8_gemm_8192x8192x8200", GemmCase(qg, torch, W.int8_gemm_8192x8192x8200(), 2), "tensor")]
    if workload in ("a8w4_conv_f32_56x56x64_3x3", "a8w4_conv_f32_sym_56x56x64_3x3"):
        # 160 input images of 0.8 MB: 128 MB > L2
        return [(workload, DynConvCase(qg, torch, W.a8w4_conv_f32_56x56x64_3x3(), 160,
                                       symmetric="_sym_" in workload), "latency")]
    raise SystemExit(f"unknown workload {workload}")


# ---------------------------------------------------------------------------
# ncu traffic figure (committed summary), valid only for the same kernel source
# ---------------------------------------------------------------------------
# Source file of the kernel behind each workload (plus the shared header).
KERNEL_SOURCES = {
    "int8_gemm_8192x8192x8200": "i8gemm.cu",
    "int8_gemm_130x70x129": "i8gemm.cu",
    "int8_conv_56x56x64_3x3": "i8gemm.cu",
    "a8w4_gemv_1x14336x4096": "a8w4.cu",
    "a8w4_gemm_128x4096x4096": "a8w4_tc.cu",
    "a8w4_gemv_bf16s_1x14336x4096": "a8w4.cu",
    "a8w4_gemv_actblock_1x14336x4096": "a8w4.cu",
    "a8w4_gemm_actblock_128x4096x4096": "a8w4_tc.cu",
    "a8w4_gemm_asym_128x4096x4096": "a8w4_tc.cu",
    "a8w4_gemv_asym_1x14336x4096": "a8w4.cu",
    "a8w4_conv_f32_56x56x64_3x3": "a8w4_tc.cu",
    "a8w4_conv_f32_sym_56x56x64_3x3": "a8w4_tc.cu",
}


def power_capped(clk):
    """True when the 1 kW limiter held the SM clock down while a region was
    timed: sw_power_cap among the reasons AND a median SM clock below 97 % of
    the maximum.  The flag alone also shows while the clock stays at its
    maximum, and then the burst peak is still the fair denominator."""
    if not clk or "sw_power_cap" not in clk.get("reasons", []):
        return False
    mhz, top = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    return not (mhz and top) or mhz < 0.97 * top


def source_digest(kernel):
    """Digest of the source the kernel of `kernel` is built from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gemv_zero_point_b200", "csrc")
    for name in ("qg_internal.cuh", KERNEL_SOURCES.get(kernel, "")):
        path = os.path.join(csrc, name)
        if name and os.path.exists(path):
            with open(path, "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel):
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(kernel)
    for line in open(path):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") == kernel and f.get("src") == digest:
            return float(f["bytes_per_launch"])
    return None


# ---------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# ---------------------------------------------------------------------------
_WORKLOAD_CACHE = {}


def _inputs(name):
    """The seeded inputs of a workload, drawn once per process (drawing the
    8192x8200 GEMM's operands takes longer than the sample it feeds)."""
    if name not in _WORKLOAD_CACHE:
        import workloads
        _WORKLOAD_CACHE[name] = getattr(workloads, name)()
    return _WORKLOAD_CACHE[name]


def oracle_sample(workload, budget_s=12.0, rows_gemm=None, small=False):
    """Time the CPU oracle, as it stands, on a bounded sample of the workload.
    Returns (ops per second, seconds spent, description)."""
    import oracle
    ops, spent, parts = 0.0, 0.0, []
    if workload in ("headline", "int8_gemm_8192x8192x8200"):
        w = _inputs("int8_gemm_8192x8192x8200")
        m0 = np.array([oracle.requant_params(float(r))[0] for r in w["ratio"]])
        sh = np.array([oracle.requant_params(float(r))[1] for r in w["ratio"]])
        cols = 512 if small else w["N"]
        rows = 1 if small else (rows_gemm or 2)
        t = time.perf_counter()
        oracle.qgemm_s8s8_requant(w["A"][:rows, :w["K"]], w["B"][:, :cols], w["za"], w["zb"],
                                  w["bias"][:cols], m0[:cols], sh[:cols], w["out_zp"],
                                  w["clamp_min"], w["clamp_max"])
        dt = time.perf_counter() - t
        ops += gemm_ops(rows, cols, w["K"]); spent += dt
        parts.append(f"int8 GEMM {rows} row(s) x {cols} cols of 8192x8192x8200")
    if workload == "a8w4_gemv_asym_1x14336x4096":
        w = _inputs("a8w4_gemv_1x14336x4096")
        n = 512 if small else w["N"]
        zw = (w["sw"][:n] * np.random.default_rng(77).uniform(-8, 8, w["sw"][:n].shape)).astype(np.float32)
        t = time.perf_counter()
        oracle.qgemm_a8w4_f32_asym(w["x"], w["qw"][:n], w["sw"][:n], zw, w["bias"][:n], -6.0, 6.0)
        dt = time.perf_counter() - t
        ops += a8w4_ops(1, n, w["K"]); spent += dt
        parts.append(f"A8W4 GEMV (asymmetric weights) {n} of 14336 rows")
    if workload in ("headline", "a8w4_gemv_1x14336x4096", "a8w4_gemv_bf16s_1x14336x4096",
                    "a8w4_gemv_actblock_1x14336x4096"):
        w = _inputs("a8w4_gemv_1x14336x4096")
        n = 512 if small else w["N"]
        t = time.perf_counter()
        fn = {"a8w4_gemv_bf16s_1x14336x4096": oracle.qgemm_a8w4_f32_bf16s,
              "a8w4_gemv_actblock_1x14336x4096": oracle.qgemm_a8w4_f32_actblock}.get(
                  workload, oracle.qgemm_a8w4_f32)
        fn(w["x"], w["qw"][:n], w["sw"][:n], w["bias"][:n], -6.0, 6.0)
        dt = time.perf_counter() - t
        ops += a8w4_ops(1, n, w["K"]); spent += dt
        tag = {"a8w4_gemv_bf16s_1x14336x4096": " (bf16 scales)",
               "a8w4_gemv_actblock_1x14336x4096": " (per-block activations)"}.get(workload, "")
        parts.append(f"A8W4 GEMV{tag} {n} of 14336 rows")
    if workload in ("a8w4_gemm_128x4096x4096", "a8w4_gemm_actblock_128x4096x4096",
                    "a8w4_gemm_asym_128x4096x4096"):
        w = _inputs("a8w4_gemm_128x4096x4096")
        rows = 1 if small else 4
        t = time.perf_counter()
        if workload == "a8w4_gemm_asym_128x4096x4096":
            zw = (w["sw"] * np.random.default_rng(77).uniform(-8, 8, w["sw"].shape)).astype(np.float32)
            oracle.qgemm_a8w4_f32_asym(w["x"][:rows], w["qw"], w["sw"], zw, w["bias"], -6.0, 6.0)
        elif workload == "a8w4_gemm_actblock_128x4096x4096":
            oracle.qgemm_a8w4_f32_actblock(w["x"][:rows], w["qw"], w["sw"], w["bias"], -6.0, 6.0)
        else:
            oracle.qgemm_a8w4_f32(w["x"][:rows], w["qw"], w["sw"], w["bias"], -6.0, 6.0)
        dt = time.perf_counter() - t
        ops += a8w4_ops(rows, w["N"], w["K"]); spent += dt
        parts.append(f"{workload.rsplit('_', 1)[0]} {rows} of 128 rows")
    if workload == "int8_gemm_130x70x129":
        w = _inputs("int8_gemm_130x70x129")
        m0, sh = oracle.requant_params(float(w["ratio"][0]))
        t = time.perf_counter()
        oracle.qgemm_s8s8_requant(w["A"], w["B"], w["za"], w["zb"], w["bias"], m0, sh,
                                  w["out_zp"], w["clamp_min"], w["clamp_max"])
        dt = time.perf_counter() - t
        ops += gemm_ops(130, 70, 129); spent += dt
        parts.append("int8 GEMM 130x70x129 (whole)")
    if workload in ("a8w4_conv_f32_56x56x64_3x3", "a8w4_conv_f32_sym_56x56x64_3x3"):
        w = _inputs("a8w4_conv_f32_56x56x64_3x3")
        sym = "_sym_" in workload
        t = time.perf_counter()
        oracle.qconv2d_f32_dyn_a8w4(w["x"], w["qw"], w["sw"], w["stride"], w["pad"], w["bias"],
                                    w["clamp_min"], w["clamp_max"], symmetric=sym)
        dt = time.perf_counter() - t
        ops += a8w4_ops(3136, 64, 576); spent += dt
        parts.append(f"float-input dynamic conv ({'symmetric' if sym else 'asymmetric'} rows) "
                     "1x56x56x64 3x3 (whole)")
    if workload == "int8_conv_56x56x64_3x3":
        w = _inputs("int8_conv_56x56x64_3x3")
        pr = [oracle.requant_params(float(r)) for r in w["ratio"]]
        m0 = np.array([p[0] for p in pr]); sh = np.array([p[1] for p in pr])
        t = time.perf_counter()
        oracle.qconv2d_s8(w["x"], w["w"], w["stride"], w["pad"], w["za"], w["bias"], m0, sh,
                          w["out_zp"], w["clamp_min"], w["clamp_max"])
        dt = time.perf_counter() - t
        ops += gemm_ops(3136, 64, 576); spent += dt
        parts.append("int8 conv 1x56x56x64 3x3 (whole)")
    return ops / spent, spent, "; ".join(parts)


# ---------------------------------------------------------------------------
# The same oracle on all host cores: output rows (and, for the large GEMM,
# column blocks) split over a spawned process pool; the operands sit in
# shared memory so no worker copies them.  Only the GEMM and GEMV parts of
# the workloads are split this way; other workloads report one core only.
# ---------------------------------------------------------------------------
_POOL_ARRAYS = {}


def _pool_init(specs):
    from multiprocessing import shared_memory
    global _POOL_SHM
    _POOL_SHM = []
    for key, (name, shape, dtype) in specs.items():
        shm = shared_memory.SharedMemory(name=name)
        _POOL_SHM.append(shm)
        _POOL_ARRAYS[key] = np.ndarray(shape, dtype=np.dtype(dtype), buffer=shm.buf)


def _pool_task(task):
    import oracle
    a = _POOL_ARRAYS
    kind = task[0]
    if kind == "gemm":
        _, r, c0, c1 = task
        oracle.qgemm_s8s8_requant(a["gA"][r:r + 1], a["gB"][:, c0:c1], int(a["gz"][0]),
                                  int(a["gz"][1]), a["gbias"][c0:c1], a["gm0"][c0:c1],
                                  a["gsh"][c0:c1], int(a["gz"][2]), -128, 127)
    else:
        _, fn, n0, n1 = task
        getattr(oracle, fn)(a["vx"], a["vqw"][n0:n1], a["vsw"][n0:n1], a["vbias"][n0:n1],
                            -6.0, 6.0)
    return 0


def oracle_sample_all_cores(workload):
    """(ops per second, seconds, cores, description) of the oracle split over
    every host core, or None for workloads without a split."""
    import multiprocessing as mp
    from multiprocessing import shared_memory
    gemm = workload in ("headline", "int8_gemm_8192x8192x8200")
    gemv_fn = {"headline": "qgemm_a8w4_f32", "a8w4_gemv_1x14336x4096": "qgemm_a8w4_f32",
               "a8w4_gemv_bf16s_1x14336x4096": "qgemm_a8w4_f32_bf16s",
               "a8w4_gemv_actblock_1x14336x4096": "qgemm_a8w4_f32_actblock"}.get(workload)
    if not gemm and not gemv_fn:
        return None
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cores = max(1, min(cores, 64))   # each GEMM task holds ~70 MB of int64 temporaries
    arrays, tasks, ops, parts = {}, [], 0.0, []
    if gemm:
        import oracle
        w = _inputs("int8_gemm_8192x8192x8200")
        rows = cores
        arrays["gA"] = np.ascontiguousarray(w["A"][:rows, :w["K"]])
        arrays["gB"] = np.ascontiguousarray(w["B"][:, :w["N"]])
        arrays["gbias"] = w["bias"]
        pr = [oracle.requant_params(float(r)) for r in w["ratio"]]
        arrays["gm0"] = np.array([p[0] for p in pr], np.int64)
        arrays["gsh"] = np.array([p[1] for p in pr], np.int64)
        arrays["gz"] = np.array([w["za"], w["zb"], w["out_zp"]], np.int64)
        blk = 1024
        tasks += [("gemm", r, c, min(c + blk, w["N"])) for r in range(rows)
                  for c in range(0, w["N"], blk)]
        ops += gemm_ops(rows, w["N"], w["K"])
        parts.append(f"int8 GEMM {rows} row(s) x 8192 cols of 8192x8192x8200")
    if gemv_fn:
        w = _inputs("a8w4_gemv_1x14336x4096")
        arrays["vx"], arrays["vqw"], arrays["vsw"], arrays["vbias"] = w["x"], w["qw"], w["sw"], w["bias"]
        step = -(-w["N"] // (4 * cores))
        tasks += [("gemv", gemv_fn, n, min(n + step, w["N"])) for n in range(0, w["N"], step)]
        ops += a8w4_ops(1, w["N"], w["K"])
        parts.append(f"A8W4 GEMV ({gemv_fn}) 14336 of 14336 rows")
    shms, specs = [], {}
    try:
        for key, arr in arrays.items():
            arr = np.ascontiguousarray(arr)
            shm = shared_memory.SharedMemory(create=True, size=max(arr.nbytes, 1))
            shms.append(shm)
            np.ndarray(arr.shape, arr.dtype, buffer=shm.buf)[...] = arr
            specs[key] = (shm.name, arr.shape, arr.dtype.str)
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS")}
        os.environ.update({"OMP_NUM_THREADS": "1", "OPENBLAS_NUM_THREADS": "1"})
        try:
            with mp.get_context("spawn").Pool(cores, initializer=_pool_init, initargs=(specs,)) as pool:
                # workers up and the oracle imported before the clock starts; a
                # worker that dies makes get() time out instead of hanging
                warm = ([("gemv", "qgemm_a8w4_f32", 0, 1)] if gemv_fn else [("gemm", 0, 0, 1)]) * cores
                pool.map_async(_pool_task, warm, chunksize=1).get(timeout=300)
                t = time.perf_counter()
                pool.map_async(_pool_task, tasks, chunksize=1).get(timeout=600)
                dt = time.perf_counter() - t
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
    finally:
        for shm in shms:
            shm.close()
            shm.unlink()
    return ops / dt, dt, cores, "; ".join(parts)


def reference_arm(args, dist):
    """--impl reference: the oracle as it stands on the host cores, one bounded
    sample per step, same metric/unit as the GPU arm.  Rank 0 only."""
    if dist.rank != 0:
        return
    total_ops, total_s = 0.0, 0.0
    desc = ""
    for i in range(args.warmup + args.steps):
        rate, spent, desc = oracle_sample(args.workload, small=True)
        if i >= args.warmup:
            total_ops += rate * spent
            total_s += spent
    value = total_ops / total_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": args.workload, "l2": "n/a (CPU)"},
            "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": "TOPS",
                             "sample": "per step: " + desc},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="headline", choices=WORKLOAD_NAMES)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=32)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    dist = Dist(args.gpus)
    if args.impl == "reference":
        reference_arm(args, dist)
        dist.close()
        return

    import torch
    import gemv_zero_point_b200 as qg
    torch.cuda.set_device(dist.local)
    qg.qg_device_status(True)
    cases = build_cases(args.workload, qg, torch)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    # warm-up (eager: also performs the library's one-time per-device set-up)
    for i in range(args.warmup):
        for _, c, _ in cases:
            c.run(i)
    torch.cuda.synchronize()

    # The timed K steps are captured once into a CUDA graph of C-ABI calls and
    # replayed, so host-side launch cost (Python + ctypes) is not in the
    # kernel numbers; every kernel still runs, one launch per call.
    def capture(fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(args.steps):
                for f in fns:
                    f(i + args.warmup)
        return g

    def replay_ms(g):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        return e0.elapsed_time(e1)

    def capture_n(fns, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                for f in fns:
                    f(i + args.warmup)
        return g

    def part_ms(fn):
        """Median per-call time of a call timed alone.  The graph holds enough
        back-to-back calls to last PART_GRAPH_MS (at least --steps calls, at
        most PART_CALLS), so graph start-up is spread over hundreds of short
        calls whatever --steps is; it is replayed PART_REPLAYS times, each
        replay after an idle pause so every replay is a burst (a kernel timed
        alone) rather than a power-capped loop; clocks are sampled meanwhile."""
        probe = capture_n([fn], 10)
        probe.replay()
        torch.cuda.synchronize()
        call_ms = replay_ms(probe) / 10
        del probe
        n = max(args.steps, min(PART_CALLS, int(math.ceil(PART_GRAPH_MS / max(call_ms, 1e-4)))))
        g = capture_n([fn], n)
        g.replay()
        torch.cuda.synchronize()
        clk = Clocks(dist.local)
        clk.start()
        times = []
        for _ in range(PART_REPLAYS):
            time.sleep(0.2)
            times.append(dist.max(replay_ms(g)) / n)
        c = clk.stop()
        del g
        return statistics.median(times), {"calls": n, "replays": len(times),
                                          "min_ms": min(times), "max_ms": max(times), "clocks": c}

    step_graph = capture([c.run for _, c, _ in cases])
    step_graph.replay()          # upload + one more untimed pass
    torch.cuda.synchronize()
    clocks = Clocks(dist.local)
    clocks.start()
    time.sleep(0.3)
    region_ms = replay_ms(step_graph)
    clk = clocks.stop()
    region_ms = dist.max(region_ms)
    del step_graph
    n_calls = len(cases)
    # Each call timed alone, after a short idle so that the power limiter
    # state left by the step above (the GEMM runs at the 1 kW cap) does not
    # carry over into the next call's figure.
    per_call_ms, part_timing = [], []
    for _, c, _ in cases:
        ms, info = part_ms(c.run)
        per_call_ms.append(ms)
        part_timing.append(info)
    # the dominant kernel of each call timed alone (same launch configuration),
    # where a call is more than one launch
    # A one-launch call is its kernel; otherwise the GEMM kernel is also timed
    # alone, on A copied once to a 16-byte pitch.
    kernel_ms, kernel_timing = [], []
    for j, (_, c, _) in enumerate(cases):
        if not hasattr(c, "run_kernel") or not c.has_kernel_only():
            kernel_ms.append(per_call_ms[j])
            kernel_timing.append(None)
            continue
        c.prep_kernel_only()
        for i in range(args.warmup):
            c.run_kernel(i)
        ms, info = part_ms(c.run_kernel)
        kernel_ms.append(ms)
        kernel_timing.append(info)
        c.release_kernel_only()
    status = qg.qg_device_status(True)
    if status != 0:
        raise SystemExit(f"device status after timed region: {qg.lib.qg_status_string(status).decode()}")

    # End to end through the same C ABI with pinned host buffers, every copy
    # timed.  Steps are pipelined over three streams, as a serving loop
    # would run them: the copy-in of step i+1 and the copy-out of step i-1
    # overlap step i's kernels (two device slots for inputs and outputs);
    # each step still copies all of its inputs in and its whole result out.
    for _, c, _ in cases:
        c.prep_e2e()
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        slot = i % 2
        if i >= 2:
            s_in.wait_event(ev_comp[slot])    # the input slot's last reader is done
        with torch.cuda.stream(s_in):
            for _, c, _ in cases:
                c.e2e_in[slot].copy_(c.h2d_host, non_blocking=True)
        ev_in[slot].record(s_in)
        s_comp.wait_event(ev_in[slot])
        if i >= 2:
            s_comp.wait_event(ev_out[slot])   # the output slot has been copied out
        for _, c, _ in cases:
            c.e2e_compute(slot, s_comp)
        ev_comp[slot].record(s_comp)
        s_out.wait_event(ev_comp[slot])
        with torch.cuda.stream(s_out):
            for _, c, _ in cases:
                c.d2h_host.copy_(c.e2e_out[slot], non_blocking=True)
        ev_out[slot].record(s_out)

    def e2e_serial_step(i):
        # one stream, in order: copy in, the API calls, copy out
        with torch.cuda.stream(s_comp):
            for _, c, _ in cases:
                c.e2e_in[0].copy_(c.h2d_host, non_blocking=True)
            for _, c, _ in cases:
                c.e2e_compute(0, s_comp)
            for _, c, _ in cases:
                c.d2h_host.copy_(c.e2e_out[0], non_blocking=True)

    def time_e2e(step_fn, first, last):
        for i in range(2):
            step_fn(i)
        torch.cuda.synchronize()
        dist.barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(first)
        s_comp.wait_event(t0)
        s_out.wait_event(t0)
        for i in range(args.e2e_steps):
            step_fn(i)
        t1.record(last)
        torch.cuda.synchronize()
        return dist.max(t0.elapsed_time(t1)) / args.e2e_steps

    # Both schedules are timed; the faster is the figure (the pipeline pays
    # a cross-stream hand-off per step, which only large copies amortise).
    e2e_pipe_ms = time_e2e(e2e_step, s_in, s_out)
    e2e_serial_ms = time_e2e(e2e_serial_step, s_comp, s_comp)
    e2e_ms = min(e2e_pipe_ms, e2e_serial_ms)

    # The copies alone, both directions at once (no kernels): the floor the
    # pipelined schedule approaches when the link, not the device, bounds it.
    def copy_only_ms():
        def one(i):
            slot = i % 2
            with torch.cuda.stream(s_in):
                for _, c, _ in cases:
                    c.e2e_in[slot].copy_(c.h2d_host, non_blocking=True)
            with torch.cuda.stream(s_out):
                for _, c, _ in cases:
                    c.d2h_host.copy_(c.e2e_out[slot], non_blocking=True)
        for i in range(2):
            one(i)
        torch.cuda.synchronize()
        dist.barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        s_out.wait_event(t0)
        for i in range(args.e2e_steps):
            one(i)
        s_out.wait_stream(s_in)
        t1.record(s_out)
        torch.cuda.synchronize()
        return dist.max(t0.elapsed_time(t1)) / args.e2e_steps

    copy_ms = copy_only_ms()

    step_ops = sum(c.ops() for _, c, _ in cases)
    ms_per_step = region_ms / args.steps
    value = dist.world * step_ops / (ms_per_step * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    # The burst peak describes a GEMM timed alone; once the 1 kW cap holds
    # the clock down (power_capped) the sustained figure is the fair one.
    sustained = region_ms > 1000.0 or power_capped(clk)
    tensor_peak_burst = INT8_OVER_BF16 * peaks["bf16_tflops"]
    tensor_peak_sust = INT8_OVER_BF16 * peaks["bf16_tflops_sustained"]
    tensor_peak_tops = tensor_peak_sust if sustained else tensor_peak_burst
    parts = {}
    rooflines = {}
    for j, (name, c, bound) in enumerate(cases):
        t = per_call_ms[j] * 1e-3
        tk = kernel_ms[j] * 1e-3
        part = {"ms": per_call_ms[j], "TOPS": c.ops() / t / 1e12, "GB/s": c.bytes() / t / 1e9,
                "launches_per_call": c.launches, "kernel_ms": kernel_ms[j],
                "kernel": getattr(c, "kernel", None), "timing": part_timing[j]}
        if kernel_timing[j] is not None:
            part["kernel_timing"] = kernel_timing[j]
        if bound == "tensor":
            kt = c.ops() / tk / 1e12
            part["frac_of_int8_peak"] = part["TOPS"] / tensor_peak_tops
            part["frac_of_int8_peak_burst"] = part["TOPS"] / tensor_peak_burst
            part["frac_of_int8_peak_sustained"] = part["TOPS"] / tensor_peak_sust
            # The kernel alone is timed in bursts after idle pauses: the burst
            # figure is its fair peak, unless the power limiter still showed
            # while it ran.
            kt_info = kernel_timing[j] or part_timing[j]
            k_clk = (kt_info or {}).get("clocks") or {}
            k_sust = power_capped(k_clk)
            k_peak = tensor_peak_sust if k_sust else tensor_peak_burst
            part["frac_of_nominal_int8"] = part["TOPS"] / NOMINAL_INT8_TOPS
            rooflines[name] = {"bound": "tensor", "achieved": kt, "peak": k_peak,
                               "unit": "TOPS", "frac": kt / k_peak,
                               "frac_of_sustained": kt / tensor_peak_sust,
                               "frac_of_nominal_int8": kt / NOMINAL_INT8_TOPS,
                               "traffic": traffic_for(name),
                               "peak_source": f"{peak_src} bf16 {'sustained' if k_sust else 'burst'} x {INT8_OVER_BF16:g} (int8/bf16 nominal)"}
        elif bound == "tensor_bf16":
            # int8 x int4 work done as exact bf16 MMAs: the bf16 tensor rate
            # bounds it (at M = 128 its time at that rate exceeds the time to
            # stream the weights at the copy bandwidth)
            kt = c.ops() / tk / 1e12
            k_clk = (part_timing[j] or {}).get("clocks") or {}
            k_sust = power_capped(k_clk)
            k_peak = peaks["bf16_tflops_sustained"] if k_sust else peaks["bf16_tflops"]
            kb = c.bytes() / tk / 1e9
            part["frac_of_hbm"] = part["GB/s"] / peaks["hbm_gbs"]
            rooflines[name] = {"bound": "tensor", "achieved": kt, "peak": k_peak,
                               "unit": "TFLOP/s", "frac": kt / k_peak,
                               "hbm_frac": kb / peaks["hbm_gbs"],
                               "traffic": traffic_for(name),
                               "peak_source": f"{peak_src} bf16 {'sustained' if k_sust else 'burst'} (the MMAs are bf16)"}
        else:
            kb = c.bytes() / tk / 1e9
            part["frac_of_hbm"] = part["GB/s"] / peaks["hbm_gbs"]
            rooflines[name] = {"bound": "hbm", "achieved": kb, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": kb / peaks["hbm_gbs"],
                               "traffic": traffic_for(name), "peak_source": f"{peak_src} copy bandwidth"}
        parts[name] = part
    dominant = max(range(n_calls), key=lambda j: per_call_ms[j])
    dom_name = cases[dominant][0]

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": " + ".join(n for n, _, _ in cases),
                   "l2": "inputs larger than L2: rotating input sets "
                         + ", ".join(f"{n}: {len(c.inputs) if hasattr(c, 'inputs') else len(c.packed)}"
                                     for n, c, _ in cases),
                   "parallelism": f"replicas x{dist.world}"},
        "parts": parts,
        "roofline": dict(rooflines[dom_name], workload=dom_name,
                         kernel=getattr(cases[dominant][1], "kernel", None)),
        "rooflines": rooflines,
        "gpu_launches": args.steps * sum(c.launches for _, c, _ in cases),
        "e2e": {"value": dist.world * step_ops / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS",
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": sum(c.h2d() for _, c, _ in cases),
                "d2h_bytes_per_step": sum(c.d2h() for _, c, _ in cases),
                "schedule": "pipelined" if e2e_pipe_ms <= e2e_serial_ms else "serial",
                "pipelined_ms_per_step": e2e_pipe_ms, "serial_ms_per_step": e2e_serial_ms,
                "pipelined_note": "copy-in of step i+1 and copy-out of step i-1 overlap step i "
                                  "(three streams, two device slots)",
                "steps": args.e2e_steps,
                "copy_only_ms_per_step": copy_ms,
                "frac_of_copy_floor": copy_ms / e2e_ms if e2e_ms > 0 else None},
        "clocks": clk,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        rate, spent, desc = oracle_sample(args.workload)
        one = {"value": rate / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle",
               "seconds": spent, "sample": desc}
        try:
            allc = oracle_sample_all_cores(args.workload)
        except Exception as e:  # the single-core figure still stands
            print(f"# all-cores oracle timing failed: {e!r}", file=sys.stderr)
            allc = None
        if allc is None:
            line["cpu_baseline"] = dict(one, all_cores=None)
        else:
            r, sec, cores, d = allc
            line["cpu_baseline"] = {"value": r / 1e12, "unit": "TOPS", "cores": cores,
                                    "kind": "oracle", "seconds": sec,
                                    "sample": d + " (rows split over a process pool)",
                                    "single_core": one}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()

"""Benchmark of the block-scaled FP4 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole path over one batch of synthetic input.
The default workload is the largest single-GPU configuration, the NVFP4
prefill up-projection M=8192, N=28672, K=8192: per step the activation's
S_global and alpha, its quantization (BF16 -> E2M1 + E4M3 block scales), then
the block-scaled GEMM D = A_hat W_hat^T in BF16 with the weights quantized
once ahead of the steps.  Other workloads (the square 4096^3 case, decode,
the down-projection, quantizer sweep, MoE, reconstruction) are selectable.

Rank 0 prints one JSON line.  With N > 1 (torchrun) every rank runs an
independent replica (the path does not shard across GPUs: no data-path
collective); NCCL is used only for the barrier and the max-over-ranks time.
`--impl reference` times the CPU oracle (the reference implementation of
the method in this repository) on a bounded sample of the same workload.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_scaled_fp4_05_b200 import fp4, synth  # noqa: E402

METRIC = "FP4 GEMM TFLOPS & quantize GB/s on 1 B200; % of FP4 peak / HBM roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP4_PER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput ratio (9 : 2.25 PFLOP/s)


# ---------------------------------------------------------------------------
# peaks, clocks, traffic
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # raw samples are kept only when a directory for them is named
        d = os.environ.get("FP4_BENCH_CLOCKS_DIR")
        self.path = os.path.join(d, "clocks_rank%d.csv" % gpu_index) if d and os.path.isdir(d) else None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        if self.path:
            with open(self.path, "w") as f:
                f.write(out)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for i, n in enumerate(names):
                if len(r) > 5 + i and r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("gemm.cu", "quantize.cu"):
        with open(os.path.join(ROOT, "block_scaled_fp4_05_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    want = kernel_source_hash()
    with open(p) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            if len(parts) >= 4 and parts[0] == workload and parts[1] == kernel and parts[3] == want:
                return float(parts[2])
    return None


def max_over_ranks(value, dist=None, device=None):
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, seconds_max):
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time (replicas: each rank runs the same workload)."""
    return units_per_rank * world / seconds_max


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
class Workload:
    """Holds device buffers for R rotating input sets and the bound calls of
    one step per set.  `kernels` names the timed kernel groups of a step."""
    name = ""
    unit = "TFLOP/s"

    def step(self, i, ev=None):
        calls = self.calls[i % len(self.calls)]
        for k, group in enumerate(calls):
            if ev is not None:
                ev[k][0].record()
            for c in group:
                c()
            if ev is not None:
                ev[k][1].record()


def _dev_bf16(bits, dev):
    return synth.bits_to_torch(bits).to(dev)


def _qbufs(fmt, rows, K, dev):
    return (torch.empty((rows, K // 2), dtype=torch.uint8, device=dev),
            torch.empty((fp4.fp4_scale_bytes(fmt, rows, K),), dtype=torch.uint8, device=dev))


class E2EPipeline:
    """Steps through the public API with each step's host-to-device copy,
    its compute and its device-to-host copy on three streams, two slots of
    device buffers: step i's input copy and step i-1's result copy run while
    step i's (or i-1's) kernels do, on both directions of the PCIe link.
    Events order, for each slot, the input copy after the compute that last
    read the slot, the compute after its input and after the result copy
    that last read the slot's D, and the result copy after the compute."""

    def __init__(self, wl, dev, new_stream=None, new_event=None, on_stream=None):
        # the CUDA stream/event constructors and stream context (replaceable
        # by recording fakes that check the ordering without a device)
        new_stream = new_stream or (lambda: torch.cuda.Stream(dev))
        new_event = new_event or torch.cuda.Event
        self.on_stream = on_stream or torch.cuda.stream
        self.wl = wl
        self.streams = [new_stream() for _ in range(3)]   # h2d, compute, d2h
        self.ev = {k: [new_event() for _ in range(2)] for k in ("h2d", "comp", "d2h")}
        self.used = [False, False]

    def step(self, i):
        j = i % 2
        sh, sc, sd = self.streams
        with self.on_stream(sh):
            if self.used[j]:
                sh.wait_event(self.ev["comp"][j])
            self.wl.e2e_h2d(j)
            self.ev["h2d"][j].record(sh)
        with self.on_stream(sc):
            sc.wait_event(self.ev["h2d"][j])
            if self.used[j]:
                sc.wait_event(self.ev["d2h"][j])
            self.wl.e2e_compute(j)
            self.ev["comp"][j].record(sc)
        with self.on_stream(sd):
            sd.wait_event(self.ev["comp"][j])
            self.wl.e2e_d2h(j)
            self.ev["d2h"][j].record(sd)
        self.used[j] = True

    def begin(self, ev):
        for s in self.streams:
            s.wait_event(ev)

    def end(self, stream):
        for s in self.streams:
            stream.wait_stream(s)


class SquareWorkload(Workload):
    """Quantize A and B (rowwise, along K) and D = A_hat B_hat^T, M=N=K=n."""

    def __init__(self, fmt, n, dev, sets=4, stream=None):
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.fmt, self.n = fmt, n
        self.name = "%s quantize+GEMM M=N=K=%d" % ("MXFP4" if fmt == fp4.MXFP4 else "NVFP4", n)
        A, B = synth.square(n)
        self.host = (A, B)
        # A and B are quantized by one batched launch (one persistent grid over
        # the tiles of both), then the GEMM
        self.kernels = ["quantize", "gemm"] if fmt == fp4.MXFP4 else \
            ["global_scales", "quantize", "gemm"]
        self.calls = []
        self.bufs = []
        for s in range(sets):
            Ad, Bd = _dev_bf16(A, dev), _dev_bf16(B, dev)
            pA, sA = _qbufs(fmt, n, n, dev)
            pB, sB = _qbufs(fmt, n, n, dev)
            D = torch.empty((n, n), dtype=torch.bfloat16, device=dev)
            groups = []
            if fmt == fp4.NVFP4:
                gA = torch.empty(1, dtype=torch.float32, device=dev)
                gB = torch.empty(1, dtype=torch.float32, device=dev)
                al = torch.empty(1, dtype=torch.float32, device=dev)
                groups.append([fp4.bind_global_scales_pair(Ad, Bd, gA, gB, al, stream)])
            else:
                gA = gB = al = None
            groups.append([fp4.bind_quantize_batch(fmt, [(Ad, pA, sA, gA), (Bd, pB, sB, gB)], stream)])
            groups.append([fp4.bind_gemm(fmt, pA, sA, pB, sB, n, n, n, al, D, None, fp4.GEMM_PREFILL,
                                         stream)])
            self.calls.append(groups)
            self.bufs.append((Ad, Bd, pA, sA, pB, sB, D, gA, gB, al))
        qbytes = n * n * 2 + n * n // 2 + fp4.fp4_scale_bytes(fmt, n, n)
        self.work = {"quantize": 2 * qbytes, "gemm": 2.0 * n ** 3, "global_scales": 2.0 * n * n * 2}
        self.bound = {"quantize": "hbm", "gemm": "tensor", "global_scales": "hbm"}
        self.flops = 2.0 * n ** 3
        self.launches_per_step = 2 if fmt == fp4.MXFP4 else 3
        self.dominant = "gemm"
        self.l2_note = "rotating %d input sets (%.0f MB of BF16 inputs) > %d MB L2" % (
            sets, sets * 4 * n * n / 1e6, L2_BYTES >> 20)

    def value(self, sec_per_step):
        return self.flops / sec_per_step / 1e12

    # ---- end to end through the public API (three phases per step, on two
    # slots of device buffers; E2EPipeline overlaps them across steps) ------
    def e2e_setup(self, dev):
        A, B = self.host
        fmt, n = self.fmt, self.n
        self.hA = synth.bits_to_torch(A).pin_memory()
        self.hB = synth.bits_to_torch(B).pin_memory()
        self.hD = torch.empty((n, n), dtype=torch.bfloat16).pin_memory()
        self.e2e_slots = []
        for _ in range(2):
            sl = {"A": torch.empty((n, n), dtype=torch.bfloat16, device=dev),
                  "B": torch.empty((n, n), dtype=torch.bfloat16, device=dev),
                  "D": torch.empty((n, n), dtype=torch.bfloat16, device=dev)}
            sl["pA"], sl["sA"] = _qbufs(fmt, n, n, dev)
            sl["pB"], sl["sB"] = _qbufs(fmt, n, n, dev)
            sl["g"] = torch.empty(3, dtype=torch.float32, device=dev)   # gA, gB, alpha
            self.e2e_slots.append(sl)
        return 2 * self.hA.numel() * 2, self.hD.numel() * 2

    def e2e_h2d(self, j):
        sl = self.e2e_slots[j]
        sl["A"].copy_(self.hA, non_blocking=True)
        sl["B"].copy_(self.hB, non_blocking=True)

    def e2e_compute(self, j):
        fmt, n, sl = self.fmt, self.n, self.e2e_slots[j]
        if fmt == fp4.NVFP4:
            gA, gB, al = sl["g"][0:1], sl["g"][1:2], sl["g"][2:3]
            fp4.fp4_compute_global_scales_pair(sl["A"], sl["B"], gA, gB, al)
        else:
            gA = gB = al = None
        fp4.fp4_quantize_batch(fmt, [(sl["A"], sl["pA"], sl["sA"], gA), (sl["B"], sl["pB"], sl["sB"], gB)])
        fp4.gemm(fmt, sl["pA"], sl["sA"], sl["pB"], sl["sB"], n, alpha=al, kernel=fp4.GEMM_PREFILL,
                 out=sl["D"])

    def e2e_d2h(self, j):
        self.hD.copy_(self.e2e_slots[j]["D"], non_blocking=True)

    def oracle_sample(self, orc, r):
        """Oracle on an r x r sub-problem of the step: S_global passes (NVFP4)
        and quantization of r rows of A and of B, then the FP64 GEMM of the
        r x r output block; returns (extrapolated seconds per full step,
        seconds spent).  The quantization uses the full tensors' S_global."""
        A, B = self.host
        n = self.n
        fmt = orc.MXFP4 if self.fmt == fp4.MXFP4 else orc.NVFP4
        if not hasattr(self, "_gs"):
            self._gs = ((orc.global_scale(A), orc.global_scale(B)) if fmt == orc.NVFP4
                        else (1.0, 1.0))
        gsA, gsB = self._gs
        a, b = np.ascontiguousarray(A[:r]), np.ascontiguousarray(B[:r])
        t0 = time.perf_counter()
        if fmt == orc.NVFP4:
            orc.global_scale(a)
            orc.global_scale(b)
        pA, sA = orc.quantize(fmt, 0, a, gs=gsA)
        pB, sB = orc.quantize(fmt, 0, b, gs=gsB)
        t1 = time.perf_counter()
        orc.gemm(fmt, pA, sA, pB, sB, alpha=float(np.float32(gsA) * np.float32(gsB)))
        t2 = time.perf_counter()
        return (t1 - t0) * (n / r) + (t2 - t1) * (n / r) ** 2, t2 - t0

    def calibrate(self, orc, budget_s):
        r = 32
        while r < self.n:
            _, spent = self.oracle_sample(orc, r)
            if spent * 3.5 > budget_s:
                break
            r *= 2
        return r

    def sample_note(self, r):
        return ("S_global/quantization of %d rows of A and of B and the FP64 GEMM of the %dx%d "
                "output block (K=%d), extrapolated to the %dx%d step" % (r, r, r, self.n, self.n, self.n))

    def cpu_baseline(self, orc, budget_s=20.0):
        r = self.calibrate(orc, budget_s)
        t_step, spent = self.oracle_sample(orc, r)
        return {"value": self.flops / t_step / 1e12, "unit": "TFLOP/s",
                "cores": orc.num_threads(), "kind": "oracle",
                "sample": self.sample_note(r) + "; %.1f s of CPU work in the measured sample" % spent}


class DecodeWorkload(Workload):
    """NVFP4 decode: W [28672 x 8192] quantized once; per step the M-token
    activation gets S_global, is quantized, and D = A_hat W_hat^T runs on the
    swap-AB stream-K kernel.  dynamic=True: one call, the S_global/alpha
    launch and the decode GEMM that quantizes the activation itself."""
    unit = "GB/s"

    def __init__(self, M, dev, sets=3, N=28672, K=8192, stream=None, dynamic=False):
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.M, self.N, self.K = M, N, K
        self.name = "NVFP4 decode GEMM M=%d N=%d K=%d (W pre-quantized%s)" % (
            M, N, K, ", activation quantized inside the GEMM" if dynamic else "")
        W = synth.decode_weight(N, K)
        A = synth.decode_activation(M, K)
        self.host = (A, W)
        self.kernels = ["act_quantize", "gemm"]
        self.calls, self.bufs = [], []
        Wd = _dev_bf16(W, dev)
        gW = fp4.global_scale(Wd)
        for s in range(sets):
            pW, sW = fp4.quantize(Wd, fp4.NVFP4, fp4.ROWWISE, gW)
            Ad = _dev_bf16(A, dev)
            gA = torch.empty(1, dtype=torch.float32, device=dev)
            al = torch.empty(1, dtype=torch.float32, device=dev)
            pA, sA = _qbufs(fp4.NVFP4, M, K, dev)
            D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.zeros((max(16, fp4.fp4_gemm_workspace_bytes(fp4.NVFP4, M, N, K)),),
                             dtype=torch.uint8, device=dev)
            if dynamic:
                # one call: S_global and alpha (one launch), then the decode GEMM
                # quantizing each K slice of the activation as it needs it
                self.calls.append([[fp4.bind_gemm_decode_dynamic(Ad, pW, sW, gW, D, gA, al, ws, stream)]])
            else:
                # per call: S_global of the activation, its quantization and alpha in
                # one launch, then the decode GEMM (the weights were quantized ahead
                # of time, so it may start streaming them before the quantizer ends)
                self.calls.append([
                    [fp4.bind_quantize_dynamic(Ad, pA, sA, gA, gW, al, stream)],
                    [fp4.bind_gemm(fp4.NVFP4, pA, sA, pW, sW, M, N, K, al, D, ws,
                                   fp4.GEMM_DECODE | fp4.GEMM_B_STATIC, stream)],
                ])
            self.bufs.append((pW, sW, Ad, gA, al, pA, sA, D, ws))
        del Wd
        torch.cuda.empty_cache()
        wbytes = N * K // 2 + fp4.fp4_scale_bytes(fp4.NVFP4, N, K)
        abytes = M * K // 2 + fp4.fp4_scale_bytes(fp4.NVFP4, M, K)
        self.gemm_bytes = wbytes + abytes + M * N * 2
        self.work = {"gemm": self.gemm_bytes, "act_quantize": M * K * 2 + abytes}   # one read of x
        self.bound = {"gemm": "hbm", "act_quantize": "hbm"}
        if dynamic:
            # one group: the S_global launch and the GEMM (timed together)
            self.kernels = ["gemm"]
            self.work = {"gemm": self.gemm_bytes}
        self.flops = 2.0 * M * N * K
        self.launches_per_step = 2   # activation quantizer (or S_global), decode GEMM
        self.dominant = "gemm"
        self.l2_note = "rotating %d quantized weight copies (%.0f MB) > %d MB L2" % (
            sets, sets * wbytes / 1e6, L2_BYTES >> 20)

    def value(self, sec_per_step):
        return self.gemm_bytes / sec_per_step / 1e9


class QuantWorkload(Workload):
    """One quantizer call on a sweep tensor (S_global given, computed once)."""
    unit = "GB/s"

    def __init__(self, fmt, axis, rows, cols, dev, stream=None):
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.fmt, self.axis = fmt, axis
        self.name = "%s %s quantize %dx%d" % ({fp4.NVFP4: "NVFP4", fp4.MXFP4: "MXFP4",
                                               fp4.P1E8: "E8M0/16 under S_global"}[fmt],
                                              "rowwise" if axis == fp4.ROWWISE else "colwise",
                                              rows, cols)
        x = synth.quant_sweep(rows, cols)
        self.host = (x,)
        xd = _dev_bf16(x, dev)
        gs = fp4.global_scale(xd) if fmt != fp4.MXFP4 else None
        out_rows, K = (rows, cols) if axis == fp4.ROWWISE else (cols, rows)
        p, s = _qbufs(fmt, out_rows, K, dev)
        self.calls = [[[fp4.bind_quantize(fmt, axis, xd, p, s, gs, stream)]]]
        self.bufs = [(xd, gs, p, s)]
        self.kernels = ["quantize"]
        self.qbytes = rows * cols * 2 + out_rows * K // 2 + fp4.fp4_scale_bytes(fmt, out_rows, K)
        self.work = {"quantize": self.qbytes}
        self.bound = {"quantize": "hbm"}
        self.flops = 0.0
        self.launches_per_step = 1
        self.dominant = "quantize"
        self.l2_note = "input %.0f MB > %d MB L2" % (rows * cols * 2 / 1e6, L2_BYTES >> 20)

    def value(self, sec_per_step):
        return self.qbytes / sec_per_step / 1e9


class MoeWorkload(Workload):
    """MXFP4 mixture-of-experts up-projection: 8 experts with weights
    14336 x 4096 and uneven token counts (8192 routed tokens in all), per
    step the quantization of every expert's activations (one batched launch)
    and the 8 GEMMs, either as one grouped launch or as 8 separate ones."""
    TOKENS = [1536, 512, 2048, 768, 1024, 256, 1280, 768]

    def __init__(self, dev, grouped=True, stream=None, N=14336, K=4096, sets=2):
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        fmt = fp4.MXFP4
        self.name = "MXFP4 MoE up-projection, 8 experts %dx%d, tokens %s, %s" % (
            N, K, "/".join(str(t) for t in self.TOKENS), "grouped GEMM" if grouped else "8 separate GEMMs")
        experts = []
        for e in range(len(self.TOKENS)):
            W = synth.normal_bf16(N, K, seed=6, tensor_id=100 + e, sigma=0.02)
            Wd = _dev_bf16(W, dev)
            experts.append(fp4.quantize(Wd, fmt, fp4.ROWWISE, None))
            del Wd
        M_all = sum(self.TOKENS)
        A = synth.normal_bf16(M_all, K, seed=6, outlier_factor=50.0)
        self.calls, self.bufs = [], []
        for _ in range(sets):
            Ad = _dev_bf16(A, dev)
            q_items, g_items, views = [], [], []
            r0 = 0
            for e, m in enumerate(self.TOKENS):
                pA, sA = _qbufs(fmt, m, K, dev)
                D = torch.empty((m, N), dtype=torch.bfloat16, device=dev)
                q_items.append((Ad[r0:r0 + m], pA, sA, None))
                g_items.append((pA, sA, experts[e][0], experts[e][1], K, None, D))
                views.append((pA, sA, D))
                r0 += m
            quant = [fp4.bind_quantize_batch(fmt, q_items, stream)]
            if grouped:
                gemm = [fp4.bind_gemm_grouped(fmt, g_items, stream)]
            else:
                gemm = [fp4.bind_gemm(fmt, it[0], it[1], it[2], it[3], it[6].shape[0], N, K, None, it[6], None,
                                      fp4.GEMM_PREFILL, stream) for it in g_items]
            self.calls.append([quant, gemm])
            self.bufs.append((Ad, views))
        self.experts = experts
        torch.cuda.empty_cache()
        self.kernels = ["quantize", "gemm"]
        qbytes = M_all * K * 2 + M_all * K // 2 + sum(fp4.fp4_scale_bytes(fmt, m, K) for m in self.TOKENS)
        self.flops = 2.0 * M_all * N * K
        self.work = {"quantize": qbytes, "gemm": self.flops}
        self.bound = {"quantize": "hbm", "gemm": "tensor"}
        self.launches_per_step = 2 if grouped else 1 + len(self.TOKENS)
        self.dominant = "gemm"
        self.l2_note = "expert weights %.0f MB > %d MB L2" % (
            len(self.TOKENS) * (N * K // 2 + fp4.fp4_scale_bytes(fmt, N, K)) / 1e6, L2_BYTES >> 20)

    def value(self, sec_per_step):
        return self.flops / sec_per_step / 1e12


class DequantWorkload(Workload):
    """Reconstruction of the NVFP4 decode weight W 28672x8192 to BF16 (the
    input a W4A16 path gives a 16-bit GEMM)."""
    unit = "GB/s"

    def __init__(self, dev, stream=None, N=28672, K=8192, sets=2):
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.name = "NVFP4 dequantize %dx%d to BF16" % (N, K)
        W = synth.decode_weight()
        Wd = _dev_bf16(W, dev)
        gW = fp4.global_scale(Wd)
        pW, sW = fp4.quantize(Wd, fp4.NVFP4, fp4.ROWWISE, gW)
        del Wd
        self.calls, self.bufs = [], []
        for _ in range(sets):
            out = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
            self.calls.append([[fp4.BoundCall("fp4_dequantize", fp4.NVFP4, fp4._dptr(pW, "packed"),
                                              fp4._dptr(sW, "scales"), fp4._dptr(gW, "gs"), N, K,
                                              fp4._dptr(out, "out"), K, fp4._stream(stream))]])
            self.bufs.append(out)
        self.keep = (pW, sW, gW)
        torch.cuda.empty_cache()
        self.kernels = ["dequantize"]
        self.qbytes = N * K // 2 + fp4.fp4_scale_bytes(fp4.NVFP4, N, K) + N * K * 2
        self.work = {"dequantize": self.qbytes}
        self.bound = {"dequantize": "hbm"}
        self.flops = 0.0
        self.launches_per_step = 1
        self.dominant = "dequantize"
        self.l2_note = "%d output copies of %.0f MB > %d MB L2" % (sets, N * K * 2 / 1e6, L2_BYTES >> 20)

    def value(self, sec_per_step):
        return self.qbytes / sec_per_step / 1e9


class PrefillWorkload(Workload):
    """NVFP4 prefill: per step the activation's S_global (and alpha) and its
    quantization, then D = A_hat W_hat^T on the persistent tensor-core kernel;
    the weights are quantized once, ahead of the steps, and stay resident.
    With dev=None only the host inputs exist (the reference arm)."""
    TILE = 128   # side of the output tiles the CPU sample computes

    def __init__(self, M, N, K, dev, stream=None):
        self.M, self.N, self.K = M, N, K
        self.name = "NVFP4 prefill GEMM M=%d N=%d K=%d" % (M, N, K)
        self.host = synth.prefill(M, N, K)
        self.flops = 2.0 * M * N * K
        self.l2_note = "operands %.0f MB > %d MB L2" % ((M + N) * K * 0.5625 / 1e6, L2_BYTES >> 20)
        if dev is None:
            return
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        A, W = self.host
        Ad, Wd = _dev_bf16(A, dev), _dev_bf16(W, dev)
        gW = fp4.global_scale(Wd)
        pW, sW = fp4.quantize(Wd, fp4.NVFP4, fp4.ROWWISE, gW)
        del Wd
        gA = torch.empty(1, dtype=torch.float32, device=dev)
        al = torch.empty(1, dtype=torch.float32, device=dev)
        pA, sA = _qbufs(fp4.NVFP4, M, K, dev)
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        # per step: the activation's S_global and alpha (one launch), its
        # quantization (one launch), the GEMM
        self.calls = [[
            [fp4.bind_quantize_dynamic(Ad, pA, sA, gA, gW, al, stream)],
            [fp4.bind_gemm(fp4.NVFP4, pA, sA, pW, sW, M, N, K, al, D, None, fp4.GEMM_PREFILL, stream)],
        ]]
        self.bufs = [(Ad, gA, al, pA, sA, pW, sW, D, gW)]
        self.weights = (pW, sW, gW)
        torch.cuda.empty_cache()
        self.kernels = ["act_quantize", "gemm"]
        abytes = M * K // 2 + fp4.fp4_scale_bytes(fp4.NVFP4, M, K)
        # two passes over the activation (amax, then quantization) + codes and scales
        self.work = {"gemm": self.flops, "act_quantize": 2 * M * K * 2 + abytes}
        self.bound = {"gemm": "tensor", "act_quantize": "hbm"}
        self.launches_per_step = 3
        self.dominant = "gemm"

    def value(self, sec_per_step):
        return self.flops / sec_per_step / 1e12

    # ---- end to end through the public API (three phases per step, on two
    # slots of device buffers; E2EPipeline overlaps them across steps) ------
    # The step's activation arrives from pinned host memory; the resident
    # quantized weights are the layer's parameters; D goes back to the host.
    def e2e_setup(self, dev):
        A, _ = self.host
        M, N, K = self.M, self.N, self.K
        self.hA = synth.bits_to_torch(A).pin_memory()
        self.hD = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        self.e2e_slots = []
        for _ in range(2):
            sl = {"A": torch.empty((M, K), dtype=torch.bfloat16, device=dev),
                  "D": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                  "g": torch.empty(2, dtype=torch.float32, device=dev)}   # gA, alpha
            sl["pA"], sl["sA"] = _qbufs(fp4.NVFP4, M, K, dev)
            self.e2e_slots.append(sl)
        return self.hA.numel() * 2, self.hD.numel() * 2

    def e2e_h2d(self, j):
        self.e2e_slots[j]["A"].copy_(self.hA, non_blocking=True)

    def e2e_compute(self, j):
        K, sl = self.K, self.e2e_slots[j]
        pW, sW, gW = self.weights
        fp4.fp4_quantize_dynamic(sl["A"], sl["pA"], sl["sA"], sl["g"][0:1], gW, sl["g"][1:2])
        fp4.gemm(fp4.NVFP4, sl["pA"], sl["sA"], pW, sW, K, alpha=sl["g"][1:2], kernel=fp4.GEMM_PREFILL,
                 out=sl["D"])

    def e2e_d2h(self, j):
        self.hD.copy_(self.e2e_slots[j]["D"], non_blocking=True)

    def e2e_expected(self):
        """The device path's D for the same activation (the timed graph's
        output), which the host copy of the last end-to-end step must equal."""
        return self.bufs[0][7]

    # ---- the oracle on a bounded sample of the step ------------------------
    def oracle_sample(self, orc, tiles, seed=0):
        """The oracle on a sample of one step: S_global of the whole
        activation, the quantization of the 128-row blocks of A that the
        sampled tiles need, and the FP64 GEMM of `tiles` sampled 128x128
        output tiles (K = full depth).  The weights' blocks are quantized
        before the clock starts (they are resident, outside the step).
        Returns (seconds per full step, extrapolated by the number of row
        blocks and of output tiles; seconds spent)."""
        A, W = self.host
        T = self.TILE
        nbm, nbn = self.M // T, self.N // T
        rng = np.random.default_rng(seed)
        tm = rng.integers(0, nbm, size=tiles)
        tn = rng.integers(0, nbn, size=tiles)
        if not hasattr(self, "_gW"):
            self._gW = orc.global_scale(W)
            self._qw = {}
        for b in np.unique(tn):
            if b not in self._qw:
                self._qw[b] = orc.quantize(orc.NVFP4, 0, np.ascontiguousarray(W[b * T:(b + 1) * T]),
                                           gs=self._gW)
        t0 = time.perf_counter()
        gA = orc.global_scale(A)
        t1 = time.perf_counter()
        qa = {b: orc.quantize(orc.NVFP4, 0, np.ascontiguousarray(A[b * T:(b + 1) * T]), gs=gA)
              for b in np.unique(tm)}
        t2 = time.perf_counter()
        alpha = float(np.float32(gA) * np.float32(self._gW))
        for i in range(tiles):
            a, b = qa[tm[i]], self._qw[tn[i]]
            orc.gemm(orc.NVFP4, a[0], a[1], b[0], b[1], alpha=alpha)
        t3 = time.perf_counter()
        t_step = ((t1 - t0) + (t2 - t1) * nbm / len(qa) + (t3 - t2) * (nbm * nbn) / tiles)
        return t_step, t3 - t0

    def calibrate(self, orc, budget_s, max_tiles=4096):
        """Tile count whose sample takes about budget_s seconds (4..max_tiles):
        the fixed part (S_global of the whole activation) and the cost of one
        more tile come from two short probes."""
        _, fixed = self.oracle_sample(orc, 2, seed=1)
        _, spent = self.oracle_sample(orc, 18, seed=2)
        per_tile = max((spent - fixed) / 16, 1e-3)
        return int(max(4, min(max_tiles, (budget_s - fixed) / per_tile)))

    def sample_note(self, tiles):
        return ("S_global of the whole %dx%d activation, quantization of the sampled 128-row "
                "blocks of A and the FP64 GEMM of %d sampled 128x128 output tiles (K=%d); "
                "extrapolated to the %dx%d step by row blocks and tiles" % (
                    self.M, self.K, tiles, self.K, self.M, self.N))

    def cpu_baseline(self, orc, budget_s=30.0):
        # the probes overestimate the cost per tile (they include row blocks
        # of A the full sample shares): about 10-20 s are spent
        tiles = self.calibrate(orc, budget_s)
        t_step, spent = self.oracle_sample(orc, tiles)
        return {"value": self.flops / t_step / 1e12, "unit": "TFLOP/s",
                "cores": orc.num_threads(), "kind": "oracle",
                "sample": self.sample_note(tiles) + "; %.1f s of CPU work in the measured sample" % spent}


class TorchCall:
    """A comparison-point call into a library (torch) inside a step; it runs
    on the current stream, so on_stream only records nothing new."""

    def __init__(self, fn, name):
        self.fn, self.name = fn, name

    def __call__(self):
        self.fn()

    def on_stream(self, stream):
        return self


class W4A16Workload(Workload):
    """The W4A16 comparison path: per step the NVFP4 weights are
    reconstructed to BF16 (this library's fp4_dequantize) and a 16-bit GEMM
    (torch.matmul, i.e. cuBLAS) multiplies the BF16 activation by them.  A
    comparison point for the native W4A4 path on the same shapes, not part
    of the product."""

    def __init__(self, M, N, K, dev, stream=None, act=None):
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.M, self.N, self.K = M, N, K
        self.name = "W4A16 comparison: NVFP4 weights -> BF16, then BF16 GEMM, M=%d N=%d K=%d" % (M, N, K)
        if M <= 16:
            W = synth.decode_weight(N, K)
            A = synth.decode_activation(M, K)
        else:
            A, W = synth.prefill(M, N, K)
        Wd = _dev_bf16(W, dev)
        gW = fp4.global_scale(Wd)
        pW, sW = fp4.quantize(Wd, fp4.NVFP4, fp4.ROWWISE, gW)
        del Wd
        Ad = _dev_bf16(A, dev)
        W16 = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        deq = fp4.BoundCall("fp4_dequantize", fp4.NVFP4, fp4._dptr(pW, "packed"), fp4._dptr(sW, "scales"),
                            fp4._dptr(gW, "gs"), N, K, fp4._dptr(W16, "out"), K, fp4._stream(stream))
        mm = TorchCall(lambda: torch.matmul(Ad, W16.t(), out=D), "bf16_gemm")
        self.calls = [[[deq], [mm]]]
        self.bufs = [(pW, sW, gW, Ad, W16, D)]
        torch.cuda.empty_cache()
        self.kernels = ["dequantize", "bf16_gemm"]
        self.flops = 2.0 * M * N * K
        self.work = {"dequantize": N * K // 2 + fp4.fp4_scale_bytes(fp4.NVFP4, N, K) + N * K * 2,
                     "bf16_gemm": self.flops}
        self.bound = {"dequantize": "hbm", "bf16_gemm": "tensor"}
        self.tensor_ratio = {"bf16_gemm": 1.0}   # a BF16 contraction: the BF16 peak
        self.launches_per_step = 1              # this library's kernels (the GEMM is cuBLAS)
        self.dominant = "bf16_gemm"
        self.l2_note = "BF16 weights %.0f MB > %d MB L2" % (N * K * 2 / 1e6, L2_BYTES >> 20)

    def value(self, sec_per_step):
        return self.flops / sec_per_step / 1e12


def make_workload(name, dev, stream):
    if name == "square_mx":
        return SquareWorkload(fp4.MXFP4, 4096, dev, stream=stream)
    if name == "square_nv":
        return SquareWorkload(fp4.NVFP4, 4096, dev, stream=stream)
    if name.startswith("decode_m"):
        return DecodeWorkload(int(name[len("decode_m"):]), dev, stream=stream)
    if name.startswith("decode_dyn_m"):
        return DecodeWorkload(int(name[len("decode_dyn_m"):]), dev, stream=stream, dynamic=True)
    if name == "prefill_up":
        return PrefillWorkload(8192, 28672, 8192, dev, stream=stream)
    if name == "prefill_down":
        return PrefillWorkload(8192, 8192, 28672, dev, stream=stream)
    if name in ("moe_grouped_mx", "moe_separate_mx"):
        return MoeWorkload(dev, grouped=name == "moe_grouped_mx", stream=stream)
    if name == "dequant_w_nv":
        return DequantWorkload(dev, stream=stream)
    if name == "w4a16_prefill_up":
        return W4A16Workload(8192, 28672, 8192, dev, stream=stream)
    if name == "w4a16_decode_m16":
        return W4A16Workload(16, 28672, 8192, dev, stream=stream)
    if name.startswith("quant_"):
        _, shape, f, ax = name.split("_")
        rows, cols = (16384, 16384) if shape == "16384" else (8192, 28672)
        fmt = {"nv": fp4.NVFP4, "mx": fp4.MXFP4, "p1e8": fp4.P1E8}[f]
        return QuantWorkload(fmt, fp4.ROWWISE if ax == "row" else fp4.COLWISE, rows, cols, dev, stream=stream)
    raise SystemExit("unknown workload %r" % name)


WORKLOADS = ["square_mx", "square_nv", "decode_m1", "decode_m4", "decode_m16", "decode_dyn_m1",
             "decode_dyn_m4", "decode_dyn_m16", "prefill_up",
             "prefill_down", "moe_grouped_mx", "moe_separate_mx", "dequant_w_nv", "w4a16_prefill_up", "w4a16_decode_m16"] + ["quant_%s_%s_%s" % (s, f, a) for s in ("16384", "8192x28672")
                                for f in ("nv", "mx", "p1e8") for a in ("row", "col")]


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample
# ---------------------------------------------------------------------------
def host_workload(name):
    """The workload's host inputs only (no device), for the reference arm."""
    if name == "prefill_up":
        return PrefillWorkload(8192, 28672, 8192, None)
    if name == "prefill_down":
        return PrefillWorkload(8192, 8192, 28672, None)
    if name in ("square_mx", "square_nv"):
        fmt = fp4.MXFP4 if name == "square_mx" else fp4.NVFP4

        class HostOnly(SquareWorkload):
            def __init__(self):
                n, sets = 4096, 4
                self.fmt, self.n = fmt, n
                self.host = synth.square(n)
                self.flops = 2.0 * n ** 3
                self.name = "%s quantize+GEMM M=N=K=%d" % ("MXFP4" if fmt == fp4.MXFP4 else "NVFP4", n)
                # the same config description as this workload's line on the GPU arm
                self.l2_note = "rotating %d input sets (%.0f MB of BF16 inputs) > %d MB L2" % (
                    sets, sets * 4 * n * n / 1e6, L2_BYTES >> 20)
        return HostOnly()
    raise SystemExit("the reference arm covers the prefill and square workloads")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as orc
    wl = host_workload(args.workload)
    # each step is a bounded sample: the whole run stays within a few minutes
    budget = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    r = wl.calibrate(orc, budget)
    for _ in range(args.warmup):
        wl.oracle_sample(orc, r)
    secs = [wl.oracle_sample(orc, r)[0] for _ in range(args.steps)]
    sec = statistics.median(secs)
    v = wl.flops / sec / 1e12
    sample = "per step: " + wl.sample_note(r)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "l2": wl.l2_note, "replicas": 1,
                   "inputs": "seeded synthetic BF16 (Philox), outlier channels"},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": orc.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="prefill_up", choices=WORKLOADS)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()

    if args.impl == "reference":
        if args.steps is None:
            args.steps = 3
        if args.warmup is None:
            args.warmup = 1
        run_reference(args)
        return

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    wl = make_workload(args.workload, dev, stream)
    per_step_guess = {"square_mx": 60e-6, "square_nv": 70e-6, "prefill_up": 0.9e-3,
                      "prefill_down": 1.0e-3}.get(args.workload, 200e-6)
    steps = args.steps if args.steps is not None else max(50, int(2.0 / per_step_guess))
    warmup = args.warmup if args.warmup is not None else max(3, min(200, steps // 20))

    # eager warm-up (also sets every kernel's attributes before capture)
    for i in range(max(3, len(wl.calls))):
        wl.step(i)
    torch.cuda.synchronize()
    if fp4.fp4_get_device_status(stream) != 0:
        raise SystemExit("device status: a kernel timed out during warm-up")

    # The timed region replays CUDA graphs of the step (no host launch gaps):
    # one graph of G consecutive steps (G a multiple of the rotating input
    # sets), replayed steps // G times, plus a graph of the remainder.  In the
    # last rotation of the G steps every kernel group is bracketed by timing
    # events captured into the graph; the per-kernel times are those of the
    # last replay.  (Events between every kernel would add gaps to the step.)
    nsets = len(wl.calls)
    G = min(steps, max(nsets, (32 // nsets) * nsets))
    reps, rem = divmod(steps, G)
    n_ev = min(G, nsets)
    ev = [[[torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)] for _ in wl.kernels]
          for _ in range(n_ev)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            e = G - 1 - i
            wl.step(i, ev[e] if e < n_ev else None)
    graph_rem = None
    if rem:
        graph_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_rem, stream=stream):
            for i in range(rem):
                wl.step(i)
    for _ in range(max(1, warmup // G)):
        graph.replay()
    torch.cuda.synchronize()
    warmup = max(3, nsets) + G * max(1, warmup // G)   # warm-up steps actually run

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t_start.record(stream)
    for _ in range(reps):
        graph.replay()
    if graph_rem is not None:
        graph_rem.replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    status = fp4.fp4_get_device_status(stream)
    if status != 0:
        raise SystemExit("device status: a kernel timed out in the timed region")
    j = n_ev

    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)
    sec_per_step = elapsed_ms / 1e3 / steps
    value = job_throughput(wl.value(sec_per_step), world, 1.0)

    in_step_ms = {k: statistics.mean(e[ki][0].elapsed_time(e[ki][1]) for e in ev[:j])
                  for ki, k in enumerate(wl.kernels)}
    # Each kernel group alone: a graph of G back-to-back launches over the
    # rotating input sets (all on the main stream), timed with events around
    # its replay.  Events inside the step above
    # separate the kernels (no overlap of one kernel's set-up with the
    # previous one, an event's own gap); this is the kernel's own rate.
    kern_ms = {}
    for ki, k in enumerate(wl.kernels):
        group_calls = [[c.on_stream(stream) for c in wl.calls[i][ki]] for i in range(nsets)]
        g_k = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_k, stream=stream):
            for i in range(G):
                for c in group_calls[i % nsets]:
                    c()
        g_k.replay()
        stream.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g_k.replay()
        b.record(stream)
        stream.synchronize()
        kern_ms[k] = max_over_ranks(a.elapsed_time(b) / G, dist, dev)
        del g_k
    if fp4.fp4_get_device_status(stream) != 0:
        raise SystemExit("device status: a kernel timed out in the per-kernel timing")
    peaks = load_peaks()
    # the per-kernel durations time each kernel alone: the burst GEMM figure
    # is the tensor denominator (conservative when the clocks were capped)
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    rooflines = {}
    for k in wl.kernels:
        dur = kern_ms[k] / 1e3
        if wl.bound[k] == "tensor":
            ach = wl.work[k] / dur / 1e12
            peak = peaks["bf16_tflops"] * getattr(wl, "tensor_ratio", {}).get(k, FP4_PER_BF16)
            rooflines[k] = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                            "frac": ach / peak, "ms": kern_ms[k], "in_step_ms": in_step_ms[k]}
        else:
            ach = wl.work[k] / dur / 1e9
            rooflines[k] = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": ach / peaks["hbm_gbs"], "ms": kern_ms[k], "in_step_ms": in_step_ms[k]}
    dom = dict(rooflines[wl.dominant])
    dom.pop("ms")
    dom.pop("in_step_ms")
    dom["timing"] = "kernel alone, %d back-to-back launches in a graph, CUDA events" % G
    dom["traffic"] = recorded_traffic(args.workload, wl.dominant)
    dom["kernel"] = wl.dominant
    ratio = getattr(wl, "tensor_ratio", {}).get(wl.dominant, FP4_PER_BF16)
    dom["peak_source"] = ("%s: %s" % (peaks["source"],
                                      ("bf16 burst x %.0f (nominal FP4:BF16)" % ratio if ratio != 1.0
                                       else "bf16 burst") if dom["bound"] == "tensor" else "HBM copy"))
    # the same kernel inside the long timed step (events captured into the
    # step graph, which separate it from its neighbours): against the
    # sustained tensor peak, the denominator for a kernel timed in a long step
    ins = in_step_ms[wl.dominant] / 1e3
    if dom["bound"] == "tensor":
        ach_in = wl.work[wl.dominant] / ins / 1e12
        peak_in = peaks["bf16_tflops_sustained"] * ratio
        src_in = "%s: bf16 sustained x %.0f" % (peaks["source"], ratio)
    else:
        ach_in = wl.work[wl.dominant] / ins / 1e9
        peak_in = peaks["hbm_gbs"]
        src_in = "%s: HBM copy" % peaks["source"]
    dom["in_step"] = {"achieved": ach_in, "peak": peak_in, "frac": ach_in / peak_in, "ms": in_step_ms[wl.dominant],
                      "timing": "events captured into the step graph during the timed region",
                      "peak_source": src_in}

    e2e = None
    if not args.no_e2e and hasattr(wl, "e2e_setup"):
        hb, db = wl.e2e_setup(dev)
        pipe = E2EPipeline(wl, dev)
        for i in range(3):
            pipe.step(i)
        torch.cuda.synchronize()
        n_e2e = 20
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        pipe.begin(a)
        for i in range(n_e2e):
            pipe.step(i)
        pipe.end(stream)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, dist, dev)
        e2e = {"value": job_throughput(wl.value(e_ms / 1e3), world, 1.0), "unit": wl.unit,
               "h2d_bytes_per_step": hb,
               "d2h_bytes_per_step": db, "ms_per_step": e_ms,
               "pipeline": "3 streams, 2 buffer slots: step i's input copy and step i-1's result copy "
                           "overlap the kernels"}
        if hasattr(wl, "e2e_expected"):
            same = bool(torch.equal(wl.hD, wl.e2e_expected().cpu()))
            e2e["result_matches_device_path"] = same
            if not same:
                raise SystemExit("end-to-end result differs from the device path's")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and hasattr(wl, "cpu_baseline"):
        import oracle as orc
        cpu = wl.cpu_baseline(orc)

    del graph, graph_rem
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": wl.unit, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": sec_per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e2m1 x e2m1 -> f32 accumulate, bf16 out",
        "data": "synthetic",
        "config": {"workload": wl.name, "l2": wl.l2_note, "replicas": world,
                   "inputs": "seeded synthetic BF16 (Philox), outlier channels"},
        "roofline": dom,
        "kernels": rooflines,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": wl.launches_per_step * steps,
        "clocks": clk,
    }
    if args.workload.startswith("square"):
        line["gemm_tflops"] = rooflines["gemm"]["achieved"]
        line["quantize_gbs"] = statistics.mean(rooflines[k]["achieved"] for k in wl.kernels
                                               if k.startswith("quantize"))
    print(json.dumps(line))


if __name__ == "__main__":
    main()

"""Benchmark of the NVFP4 calibration path on B200.

One step = one pass of the whole path over one workload's inputs, which are
resident in HBM when the timed region starts.  Default workload: the MoE
experts (128 experts of 768x2048, 262,144 routed calibration tokens), the
largest single-GPU configuration by blocks searched, whose step is

    global scale(W, per expert) -> zero H -> grouped Gram(X) ->
    Local-Hessian search -> quantise+pack -> dequantise

Other workloads (--workload): dense (W 4096x4096, X 2048x4096: global scale,
Gram, max rule, MSE and Local-Hessian search, pack, dequantise, W4A4
fake-quant of X), tiny, mlp_pair (up and down projections with the 16
calibration chunks of 65,536 tokens each kept resident), w4a4 (activation
fake-quant of 32768x8192 with packed outputs), and the rows beyond the core
path (four_over_six, w4a4_gemm, act_calib, lh_gptq).  H is zeroed at the start
of every step (its own row, a memset), so every step's search sees the
configuration's Gram.

Metric: NVFP4 blocks per second through the step (weight blocks; activation
blocks for w4a4).  The L2 cache is flushed before every timed step, outside
the step's CUDA events: a 256 MiB write, then a read of the same buffer, so
that the write's dirty lines are written back before the step rather than by
its first kernels.  The value comes from K steps timed with CUDA events at the
step boundaries only (the launches follow one another as in use); per-row
times come from K further steps with an event between rows.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no cross-GPU exchange); timing is the max over ranks.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 blocks/s (local-Hessian scale search); quant/Gram GB/s vs roofline"
UNIT = "blocks/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0
SM_COUNT = 148
FP32_LANES_PER_SM = 128
WORKLOAD_NAMES = ["moe", "dense", "tiny", "mlp_pair", "w4a4", "four_over_six", "w4a4_gemm",
                  "act_calib", "lh_gptq"]
DEFAULT_WORKLOAD = "moe"
ISSUE_SLOTS_PER_SM = 4  # one warp instruction per clock per SM sub-partition
FP64_FMA_PER_SM = 64  # B200: 64 fp64 FMA per clock per SM (about 40 TFLOP/s at boost clock)
GPTQ_DAMP = 0.01

# Local-Hessian search work per block, counted on the definition E = delta
# H_b delta^T: per candidate 256 FMA for H_b delta and 16 FMA for the dot
# product, 2 flop each (the E2M1 encodes are not counted as flops).
LH_FLOP_PER_EVAL = 2 * (256 + 16)  # delta H_b delta^T for one candidate
# bytes per activation element of the fused fake-quant with packed outputs:
# amax pass 2, fused pass 2 read + 2 write + 0.5 packed + 1/16 block codes
FAKE_QUANT_BYTES_PER_ELEM = 2 + 2 + 2 + 0.5 + 1 / 16


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ workloads
class Layer:
    """One weight tensor (optionally batched) with its calibration input."""

    def __init__(self, name, W, X=None, offsets=None, chunks=None):
        self.name = name
        self.W = W if W.dim() == 3 else W.unsqueeze(0)
        self.X = X
        self.offsets = offsets
        self.chunks = chunks  # list of resident calibration chunks
        B, R, C = self.W.shape
        dev = self.W.device
        self.B, self.R, self.C = B, R, C
        self.s_g = torch.empty(B, dtype=torch.float32, device=dev)
        self.H = torch.zeros(B, C // 16, 16, 16, dtype=torch.float32, device=dev)
        self.c_max = torch.empty(B, R, C // 16, dtype=torch.uint8, device=dev)
        self.c_mse = torch.empty_like(self.c_max)
        self.c_46 = torch.empty_like(self.c_max)
        self.c_lh = torch.empty_like(self.c_max)
        self.packed = torch.empty(B, R, C // 2, dtype=torch.uint8, device=dev)
        self.deq = torch.empty(B, R, C, dtype=torch.bfloat16, device=dev)

    def blocks(self):
        return self.B * self.R * self.C // 16

    def tokens(self):
        if self.chunks is not None:
            return sum(c.shape[0] for c in self.chunks)
        return 0 if self.X is None else self.X.shape[0]


class Runner:
    """Rows of one workload: (name, callable, algorithmic bytes, launches)."""

    def __init__(self, workload, device):
        from scale_calibration_nvfp4_b200 import nvfp4, workloads
        self.nv = nvfp4
        self.workload = workload
        self.gptq = False
        wl = workloads
        if workload in ("tiny", "dense"):
            W, X = wl.layer_inputs(workload, device)
            self.layers = [Layer(workload, W, X)]
            self.desc = wl.BY_NAME[workload].description
            self.rules = ["max", "mse", "lh"]
            self.fq_input = X
        elif workload == "lh_gptq":
            # the dense projection under Local-Hessian scales and GPTQ rounding:
            # the block-diagonal and the full Gram of its calibration tokens,
            # the scale search, GPTQ (dampening 0.01), dequantise
            W, X = wl.layer_inputs("dense", device)
            L = Layer("dense", W, X)
            L.Hf = torch.zeros(L.C, L.C, dtype=torch.float32, device=W.device)
            self.layers = [L]
            self.desc = ("Local-Hessian + GPTQ on the dense projection (W 4096x4096, X 2048x4096): "
                         "global scale, block-diagonal and full Gram, scale search, GPTQ "
                         "rounding (damp %.2f), dequantise" % GPTQ_DAMP)
            self.rules = ["lh"]
            self.gptq = True
            self.fq_input = None
        elif workload == "four_over_six":
            # the MoE experts' weights (the largest weight tensor of the
            # workloads, 403 MB) under the Four Over Six rule
            W, _, _ = wl.moe_inputs(device)
            self.layers = [Layer("experts", W, None)]
            self.desc = ("Four Over Six on the MoE experts' weights (128 x 768x2048, per-expert "
                         "tensor scales): global scale, the rule, pack, dequantise")
            self.rules = ["four_over_six"]
            self.fq_input = None
        elif workload == "moe":
            W, X, offsets = wl.moe_inputs(device)
            self.layers = [Layer("experts", W, X, offsets=offsets.to(device))]
            self.desc = wl.BY_NAME["moe"].description
            self.rules = ["lh"]
            self.fq_input = None
        elif workload == "mlp_pair":
            up, down = wl.mlp_weights(device)
            p = wl.BY_NAME["mlp_pair"].params
            ch_up = [wl.mlp_chunk("up", k, device) for k in range(p["chunks"])]
            ch_dn = [wl.mlp_chunk("down", k, device) for k in range(p["chunks"])]
            self.layers = [Layer("up", up, chunks=ch_up), Layer("down", down, chunks=ch_dn)]
            self.desc = wl.BY_NAME["mlp_pair"].description
            self.rules = ["lh"]
            self.fq_input = None
        elif workload == "w4a4_gemm":
            # the W4A4 activations times an 8192x8192 NVFP4 weight: per step the
            # dynamic fake-quant of X (packed outputs) and the product
            X = wl.w4a4_inputs(device)
            self.layers = []
            self.desc = ("W4A4 layer: X 32768x8192 dynamic NVFP4 (fake-quant with packed "
                         "outputs) times W 8192x8192 NVFP4 (seed 9, N(0,0.02), quantised once)")
            self.rules = []
            self.fq_input = X
            g = torch.Generator(device=X.device).manual_seed(9)
            W = (torch.randn(8192, 8192, generator=g, device=X.device) * 0.02).to(torch.bfloat16)
            self.gemm_w = W
            if X.is_cuda:
                self.gw_sg = nvfp4.global_scale(W)
                self.gw_codes = nvfp4.scale_search_max(W, self.gw_sg)
                self.gw_packed = nvfp4.quantize_pack(W, self.gw_sg, self.gw_codes)
                self.gemm_out = torch.empty(X.shape[0], 8192, dtype=torch.bfloat16, device=X.device)
        elif workload == "act_calib":
            # static activation range: the W4A4 activations as the calibration
            # set; per step the |x| histogram, the 99.99th-percentile tensor
            # scale and the static fake-quant with packed outputs
            X = wl.w4a4_inputs(device)
            self.layers = []
            self.desc = ("static activation range on X 32768x8192 (the W4A4 activations): |x| "
                         "histogram, 99.99th-percentile tensor scale, static fake-quant")
            self.rules = []
            self.fq_input = X
            self.hist = torch.zeros(32768, dtype=torch.int64, device=X.device)
            self.calib_sg = torch.empty(1, dtype=torch.float32, device=X.device)
        elif workload == "w4a4":
            X = wl.w4a4_inputs(device)
            self.layers = []
            self.desc = wl.BY_NAME["w4a4"].description
            self.rules = []
            self.fq_input = X
        else:
            raise ValueError(workload)
        if self.fq_input is not None:
            X = self.fq_input
            self.fq_out = torch.empty_like(X)
            self.fq_packed = torch.empty(X.shape[0], X.shape[1] // 2, dtype=torch.uint8,
                                         device=X.device)
            self.fq_codes = torch.empty(X.shape[0], X.shape[1] // 16, dtype=torch.uint8,
                                        device=X.device)
            self.fq_sg = torch.empty(1, dtype=torch.float32, device=X.device)
        self.rows = self._rows()

    def _rows(self):
        nv = self.nv
        rows = []
        for L in self.layers:
            n_w = L.B * L.R * L.C
            nb = n_w // 16
            h = L.H.numel() * 4
            pre = L.name + "." if len(self.layers) > 1 else ""
            rows.append((pre + "global_scale",
                         lambda L=L: nv.global_scale(L.W, batch=L.B, out=L.s_g), 2 * n_w, 3))
            if L.X is not None or L.chunks is not None:
                # a fresh Gram every step (a torch memset, not one of ours)
                rows.append((pre + "zero_H", lambda L=L: L.H.zero_(), h, 0))
            if self.gptq:
                rows.append((pre + "zero_H_full", lambda L=L: L.Hf.zero_(), 4 * L.C * L.C, 0))
            if L.chunks is not None:
                def gram(L=L):
                    for ch in L.chunks:
                        nv.hessian_accumulate(ch, L.H[0])
                rows.append((pre + "gram", gram,
                             2 * L.tokens() * L.C + 2 * h * len(L.chunks), 2 * len(L.chunks)))
            elif L.offsets is not None:
                rows.append((pre + "gram",
                             lambda L=L: nv.hessian_accumulate_grouped(L.X, L.offsets, L.H),
                             2 * L.X.numel() + 2 * h, 3))
            elif L.X is not None:
                rows.append((pre + "gram", lambda L=L: nv.hessian_accumulate(L.X, L.H[0]),
                             2 * L.X.numel() + 2 * h, 2))
            if self.gptq:
                rows.append((pre + "gram_full", lambda L=L: nv.hessian_full_accumulate(L.X, L.Hf),
                             2 * L.X.numel() + 8 * L.C * L.C, 1))
            if "max" in self.rules:
                rows.append((pre + "search_max",
                             lambda L=L: nv.scale_search_max(L.W, L.s_g, out=L.c_max),
                             2 * n_w + nb, 1))
            if "four_over_six" in self.rules:
                rows.append((pre + "search_four_over_six",
                             lambda L=L: nv.scale_search_four_over_six(L.W, L.s_g, out=L.c_46),
                             2 * n_w + nb, 1))
            if "mse" in self.rules:
                rows.append((pre + "search_mse",
                             lambda L=L: nv.scale_search_mse(L.W, L.s_g, out=L.c_mse),
                             2 * n_w + nb, 1))
            if "lh" in self.rules:
                rows.append((pre + "search_lh",
                             lambda L=L: nv.scale_search_local_hessian(L.W, L.s_g, L.H,
                                                                       out=L.c_lh),
                             2 * n_w + nb + h, 2))  # factor_kernel + search_kernel
            # pack (GPTQ rounding or plain) and dequantise with the codes of the
            # workload's final rule
            fin = L.c_lh if "lh" in self.rules else L.c_46
            if self.gptq:
                npan = (L.C + 127) // 128
                rows.append((pre + "gptq",
                             lambda L=L, c=fin: nv.gptq(L.W[0], L.s_g, c[0], L.Hf, GPTQ_DAMP,
                                                        out=L.packed[0]),
                             2 * n_w + nb + 4 * L.C * L.C + n_w // 2, gptq_launches(npan)))
            else:
                rows.append((pre + "quantize_pack",
                             lambda L=L, c=fin: nv.quantize_pack(L.W, L.s_g, c, out=L.packed),
                             2 * n_w + nb + n_w // 2, 1))
            rows.append((pre + "dequantize",
                         lambda L=L, c=fin: nv.dequantize(L.packed, c, L.s_g, out=L.deq),
                         n_w // 2 + nb + 2 * n_w, 1))
        if self.fq_input is not None:
            n_x = self.fq_input.numel()
            if self.workload == "act_calib":
                X = self.fq_input
                rows.append(("abs_histogram",
                             lambda: (self.hist.zero_(), nv.abs_histogram(X, self.hist)),
                             2 * n_x, 1))  # (the zeroing is a torch fill)
                rows.append(("static_scale",
                             lambda: nv.static_scale_from_histogram(self.hist, 0.9999,
                                                                    out=self.calib_sg),
                             32768 * 8, 1))
                rows.append(("fake_quant_static", lambda: self._fq_static(),
                             (FAKE_QUANT_BYTES_PER_ELEM - 2) * n_x, 1))
            elif self.workload == "w4a4_gemm":
                X = self.fq_input
                M, K, N = X.shape[0], X.shape[1], self.gemm_w.shape[0]
                rows.append(("fake_quant", lambda: self._fq(True),
                             FAKE_QUANT_BYTES_PER_ELEM * n_x, 4))
                if X.is_cuda:
                    rows.append(("gemm", lambda: nv.gemm(self.fq_packed, self.fq_codes, self.fq_sg,
                                                          self.gw_packed, self.gw_codes,
                                                          self.gw_sg,
                                                          out=self.gemm_out),
                                 M * K // 2 + N * K // 2 + M * N * 2, 4))  # 2 scale layouts, alpha, GEMM
            elif self.workload == "w4a4":
                rows.append(("fake_quant", lambda: self._fq(True),
                             FAKE_QUANT_BYTES_PER_ELEM * n_x, 4))
            else:
                rows.append(("fake_quant", lambda: self._fq(False), 6 * n_x, 4))
        return rows

    def _fq_static(self):
        nv = self.nv
        X = self.fq_input
        nv._call("nvfp4_fake_quant_static", nv._p(X), X.shape[0], X.shape[1], nv._p(self.calib_sg),
                 nv._p(self.fq_out), nv._p(self.fq_packed), nv._p(self.fq_codes), nv._stream())

    def _fq(self, packed):
        nv = self.nv
        X = self.fq_input
        nv._call("nvfp4_fake_quant", nv._p(X), X.shape[0], X.shape[1], nv._p(self.fq_out),
                 nv._p(self.fq_packed) if packed else None,
                 nv._p(self.fq_codes) if packed else None, nv._p(self.fq_sg), nv._stream())

    def blocks(self):
        if self.layers:
            return sum(L.blocks() for L in self.layers)
        return self.fq_input.numel() // 16

    def launches(self):
        return sum(r[3] for r in self.rows)

    def inputs(self):
        t = []
        for L in self.layers:
            t.append(L.W)
            if L.X is not None:
                t.append(L.X)
            if L.chunks is not None:
                t.extend(L.chunks)
        if self.fq_input is not None and not any(x is self.fq_input for x in t):
            t.append(self.fq_input)
        return t

    def results(self):
        """Every output the step writes: tensor scales, Grams, the codes of
        every rule, packed and dequantised weights, fake-quant outputs."""
        out = []
        for L in self.layers:
            out.append(L.s_g)
            if L.X is not None or L.chunks is not None:
                out.append(L.H)
            if self.gptq:
                out.append(L.Hf)
            for rule, t in (("max", L.c_max), ("mse", L.c_mse), ("lh", L.c_lh),
                            ("four_over_six", L.c_46)):
                if rule in self.rules:
                    out.append(t)
            out += [L.packed, L.deq]
        if self.fq_input is not None:
            out.append(self.fq_out)
            if self.workload != "act_calib":  # there the static scale is calib_sg
                out.append(self.fq_sg)
            if self.workload != "dense" and self.workload != "tiny":
                out += [self.fq_packed, self.fq_codes]  # packed outputs requested there
        if self.workload == "act_calib":
            out += [self.hist, self.calib_sg]
        if self.workload == "w4a4_gemm":
            out += [self.gemm_out]
        return out


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ helpers
def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


# source files each reported kernel is built from
KERNEL_SOURCES = {
    "search_lh": ("search.cu", "common.cuh", "chained.cuh"),
    "fake_quant": ("quant.cu", "common.cuh", "chained.cuh"),
    "gram": ("gram.cu", "common.cuh", "chained.cuh"),
    "four_over_six": ("quant.cu", "common.cuh", "chained.cuh"),
}


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "scale_calibration_nvfp4_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_counters(kernel, workload):
    """The ncu counters committed for a kernel on a workload (DRAM bytes and
    warp instructions per call), if they were taken on the current sources
    of that kernel; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    ent = t.get(kernel, {}).get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current sources of that kernel."""
    ent = recorded_counters(kernel, workload)
    return None if ent is None else ent.get("dram_bytes_per_launch")


def dist_env():
    if "RANK" in os.environ and "WORLD_SIZE" in os.environ:
        return int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"]), \
            int(os.environ.get("LOCAL_RANK", os.environ["RANK"]))
    return 0, 1, 0


def max_over_ranks(pg, value, device="cuda"):
    """Max of a per-rank value over all ranks (the job's time is the slowest
    rank's)."""
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.item()


def job_value(world, blocks_per_rank, ms_per_step):
    """Whole-job throughput: every rank processes its own replica of the
    workload (weak scaling), timed by the slowest rank."""
    return world * blocks_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------ GPU arm
def run_gpu(args):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        pg = dist
    from scale_calibration_nvfp4_b200 import build, nvfp4
    if rank == 0:
        build.build()
    if pg:
        pg.barrier()
    nvfp4.lib()

    run = Runner(args.workload, "cuda")
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    rows = run.rows

    def step(events=None):
        for i, r in enumerate(rows):
            if events is not None:
                events[i].record(stream)
            r[1]()
        if events is not None:
            events[-1].record(stream)

    def flush_l2():
        # a 256 MiB write, then a read of it: the write's dirty lines are
        # written back here, not by the step's first kernels
        flush.zero_()
        flush.sum()

    # timed pass: events at the step boundaries only, so that the step's
    # launches follow one another as they would in use
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    # per-row pass (after the timed one, not part of the value): an event
    # between rows
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(rows) + 1)]
          for _ in range(args.steps)]
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    # the warm-up steps come after the sampler's start-up pause, so that the
    # timed steps follow them without the GPU idling in between
    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    nvfp4.search_evaluations(reset=True)  # synchronises
    for k in range(args.steps):
        flush_l2()
        ev_step[k][0].record(stream)
        step()
        ev_step[k][1].record(stream)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    # rows sent to the fp64 re-score, and (block, candidate) evaluations the
    # searches made, per step (the second read resets both)
    rescores = [v / args.steps for v in nvfp4.search_rescores()]
    evals = [v / args.steps for v in nvfp4.search_evaluations(reset=True)]
    for k in range(args.steps):
        flush_l2()
        step(ev[k])
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None

    per_row = {r[0]: [] for r in rows}
    step_ms = []
    for k in range(args.steps):
        for i, r in enumerate(rows):
            per_row[r[0]].append(ev[k][i].elapsed_time(ev[k][i + 1]))
        step_ms.append(ev_step[k][0].elapsed_time(ev_step[k][1]))
    log("timed steps (ms):", " ".join("%.4f" % v for v in step_ms))
    ms_per_step = max_over_ranks(pg, sum(step_ms)) / args.steps
    blocks = run.blocks()
    value = job_value(world, blocks, ms_per_step)

    e2e = None if args.no_e2e else run_e2e(run, args, pg, world)

    if rank == 0:
        pk, pk_kind = peaks()
        hbm = float(pk.get("hbm_gbs", FALLBACK_HBM_GBS))
        kernels = {}
        for r in rows:
            ms = statistics.mean(per_row[r[0]])
            gbs = r[2] / (ms / 1e3) / 1e9
            kernels[r[0]] = {"ms": round(ms, 5), "GB/s": round(gbs, 1),
                             "frac_of_%s_hbm" % pk_kind: round(gbs / hbm, 3)}
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64" if run.gptq else "bf16",
            "data": "synthetic (seeded; no dataset or trained weights)",
            "config": {"workload": args.workload, "desc": run.desc, "blocks_per_step": blocks,
                       "rows": [r[0] for r in rows],
                       "parallelism": "replicas (one per GPU)" if world > 1 else "single GPU",
                       "cache": "L2 flushed before every timed step: a 256 MiB write, then a read of it "
                                "(its dirty lines written back outside the step)",
                       "timing": "value from K steps with CUDA events at the step boundaries; "
                                 "per-row times from K further steps with an event between rows"},
            "roofline": make_roofline(run, kernels, pk, pk_kind, args.workload, evals[1],
                                      clk["sm_mhz"] if clk else None),
            "search_evaluated_per_block": {"mse": round(evals[0] / blocks, 2),
                                           "local_hessian": round(evals[1] / blocks, 2)},
            "search_rescored_per_block": {
                "mse_best_two": round(rescores[0] / blocks, 5),
                "mse_all_126": round(rescores[1] / blocks, 6),
                "local_hessian_best_two": round(rescores[2] / blocks, 5),
                "local_hessian_all_126": round(rescores[3] / blocks, 6)},
            "search_lh_blocks_per_s": search_blocks_per_s(run, kernels),
            "hbm_rows_GB/s": {k: v["GB/s"] for k, v in kernels.items()
                              if k.split(".")[-1] in HBM_ROWS},
            "kernels": kernels,
            "gpu_launches": args.steps * run.launches(),
            "clocks": clk,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline and world == 1:
            out["cpu_baseline"] = cpu_baseline(run, budget_s=args.cpu_seconds)
        print(json.dumps(out), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


# rows that stream HBM (their GB/s is the figure of merit)
HBM_ROWS = ("global_scale", "gram", "search_max", "quantize_pack", "dequantize", "fake_quant",
            "fake_quant_static", "abs_histogram")


def search_blocks_per_s(run, kernels):
    """Blocks per second of the Local-Hessian search call alone (None when
    the workload has no Local-Hessian search)."""
    ms = sum(v["ms"] for k, v in kernels.items() if k.endswith("search_lh"))
    return round(run.blocks() / (ms / 1e3), 1) if ms > 0 else None


def gptq_launches(npan):
    """Kernels one GPTQ call launches for npan 128-column panels: lambda and
    the reversed copy; per panel the diagonal block, and (but the last) the
    panel solve and the next panel's update, the update beyond it (but the
    last two); per column block the row kernel and (but the last) the
    running-sum product."""
    return (2 + npan + 2 * max(npan - 1, 0) + max(npan - 2, 0) + npan + max(npan - 1, 0))


def make_roofline(run, kernels, pk, pk_kind, workload, lh_evals, sm_mhz_live=None):
    if "gptq" in kernels:
        # fp64 arithmetic of the definition: the column loop's update of the
        # later columns (R C^2 / 2 FMA) and the Cholesky factor (C^3 / 6 FMA)
        L = run.layers[0]
        R, C = L.R, L.C
        ms = kernels["gptq"]["ms"]
        sm_mhz = float(pk.get("sm_max_mhz", 1965.0))
        fp64_peak = SM_COUNT * FP64_FMA_PER_SM * 2 * sm_mhz * 1e6 / 1e12
        flop = R * C * C + C ** 3 / 3
        achieved = flop / (ms / 1e3) / 1e12
        return {"kernel": "gptq (Cholesky + column loop + lazy-batch fp64 MMA updates)",
                "bound": "alu", "achieved": round(achieved, 2), "peak": round(fp64_peak, 2),
                "unit": "TFLOP/s", "frac": round(achieved / fp64_peak, 4), "traffic": None,
                "peak_kind": "derived: 148 SMs x 64 fp64 FMA x 2 flop x %.0f MHz (%s clocks)"
                             % (sm_mhz, pk_kind),
                "flop_basis": "R C^2 (column loop) + C^3/3 (Cholesky), R=%d C=%d" % (R, C)}
    lh_rows = [k for k in kernels if k.endswith("search_lh")]
    if lh_rows:
        return search_roofline(run, kernels, lh_rows, pk, pk_kind, workload, lh_evals,
                               sm_mhz_live)
    if "fake_quant_static" in kernels:
        ms = kernels["abs_histogram"]["ms"] + kernels["fake_quant_static"]["ms"]
        n = run.fq_input.numel()
        achieved = FAKE_QUANT_BYTES_PER_ELEM * n / (ms / 1e3) / 1e9
        hbm = float(pk.get("hbm_gbs", FALLBACK_HBM_GBS))
        return {"kernel": "abs_histogram + fake_quant_static", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": None,
                "peak_kind": "%s HBM copy bandwidth" % pk_kind,
                "bytes_per_element": FAKE_QUANT_BYTES_PER_ELEM}
    if "gemm" in kernels:
        X = run.fq_input
        M, K, N = X.shape[0], X.shape[1], run.gw_packed.shape[0]
        ms = kernels["gemm"]["ms"]
        achieved = 2.0 * M * N * K / (ms / 1e3) / 1e12
        bf16 = float(pk.get("bf16_tflops", 1595.8))
        peak = 4.0 * bf16
        return {"kernel": "NVFP4 GEMM (scale layout + block-scaled tcgen05 MMA)", "bound": "tensor",
                "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": None,
                "peak_kind": "%s bf16 GEMM burst x 4 (nominal dense FP4/BF16 ratio 9/2.25)" % pk_kind,
                "flop_basis": "2 M N K, M=%d N=%d K=%d" % (M, N, K)}
    if "search_four_over_six" in kernels:
        # a streaming pass over W (2 B per value read, a code byte per 16
        # written); the exact encode of its two candidates is what bounds it
        ms = kernels["search_four_over_six"]["ms"]
        n = run.blocks() * 16
        achieved = (2 * n + n // 16) / (ms / 1e3) / 1e9
        hbm = float(pk.get("hbm_gbs", FALLBACK_HBM_GBS))
        return {"kernel": "four_over_six_kernel", "bound": "hbm", "achieved": round(achieved, 1),
                "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "traffic": recorded_traffic("four_over_six", workload),
                "peak_kind": "%s HBM copy bandwidth" % pk_kind,
                "bytes_per_element": 2 + 1 / 16,
                "note": "issue-bound on the fp32 block MSE of both candidates"}
    ms = kernels["fake_quant"]["ms"]
    n = run.fq_input.numel()
    achieved = FAKE_QUANT_BYTES_PER_ELEM * n / (ms / 1e3) / 1e9
    hbm = float(pk.get("hbm_gbs", FALLBACK_HBM_GBS))
    return {"kernel": "fake_quant (amax pass + fused pass)", "bound": "hbm",
            "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4),
            "traffic": recorded_traffic("fake_quant", workload),
            "peak_kind": "%s HBM copy bandwidth" % pk_kind,
            "bytes_per_element": FAKE_QUANT_BYTES_PER_ELEM}


def search_roofline(run, kernels, lh_rows, pk, pk_kind, workload, lh_evals, sm_mhz_live=None):
    """Roofline of the Local-Hessian search call (factor_kernel +
    search_kernel).  The kernel is bound by instruction issue (the candidate
    walk, the exact encode and the pruning bounds around a 16x16 tensor-core
    product per candidate), so the roofline is issue slots: one warp
    instruction per clock on each of the 4 sub-partitions of the 148 SMs, at
    the SM clock sampled during the timed region.  `achieved` is the warp
    instructions one call executes (ncu smsp__inst_executed.sum of both
    kernels, committed with the hash of their sources; the walk is
    deterministic for given inputs) over the call's live CUDA-event time.
    Without a counter taken on the current sources, the definition-equivalent
    arithmetic rate stands in, labelled as such."""
    lh_ms = sum(kernels[k]["ms"] for k in lh_rows)
    sm_mhz = float(sm_mhz_live or pk.get("sm_max_mhz", 1965.0))
    blocks = run.blocks()
    fp32_peak = SM_COUNT * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12
    definition = {
        "note": "not a utilisation: the definition's 544 flop (delta H_b delta^T) per "
                "(block, candidate) over the FP32 CUDA-core peak; the product itself runs "
                "on the tensor cores and the pruned walk skips candidates that provably lose",
        "TFLOP/s_on_evaluations_made": round(LH_FLOP_PER_EVAL * lh_evals / (lh_ms / 1e3) / 1e12, 2),
        "TFLOP/s_all_126_equivalent": round(LH_FLOP_PER_EVAL * 126 * blocks / (lh_ms / 1e3) / 1e12,
                                            2),
        "fp32_peak_TFLOP/s": round(fp32_peak, 2),
    }
    rec = recorded_counters("search_lh", workload) or {}
    inst = rec.get("warp_inst_per_launch")
    out = {"kernel": "factor_kernel + search_kernel<Local-Hessian> (one call)",
           "bound": "alu", "traffic": rec.get("dram_bytes_per_launch"),
           "evaluated_per_block": round(lh_evals / blocks, 2),
           "definition_equivalent": definition}
    if inst:
        peak = SM_COUNT * ISSUE_SLOTS_PER_SM * sm_mhz * 1e6 / 1e12
        achieved = inst / (lh_ms / 1e3) / 1e12
        out.update({"achieved": round(achieved, 4), "peak": round(peak, 4),
                    "unit": "Twarp-instructions/s", "frac": round(achieved / peak, 4),
                    "peak_kind": "derived: 148 SMs x 4 issue slots x %.0f MHz (SM clock %s)"
                                 % (sm_mhz, "sampled under load" if sm_mhz_live else
                                    "max, %s" % pk_kind),
                    "basis": "warp instructions per call from ncu (smsp__inst_executed.sum, "
                             "current sources) over the live call time",
                    "warp_inst_per_call": inst, "pipes": rec.get("pipes")})
    else:
        out.update({"achieved": definition["TFLOP/s_on_evaluations_made"],
                    "peak": definition["fp32_peak_TFLOP/s"], "unit": "TFLOP/s",
                    "frac": round(definition["TFLOP/s_on_evaluations_made"] / fp32_peak, 4),
                    "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 2 flop x %.0f MHz" % sm_mhz,
                    "basis": "definition-equivalent (no instruction count recorded on the "
                             "current sources): not a utilisation"})
    return out


def run_e2e(run, args, pg, world):
    """Same metric through the public API with host buffers: every step copies
    the inputs from pinned host memory to the device, runs the path and reads
    the results (codes and packed weights, or packed activations) back.

    The steps are pipelined the way a calibration loop streams its layers:
    uploads on one stream, the path on another, downloads on a third, and
    two sets of device buffers used in turn where the device has room for a
    second (one set otherwise).  Step k + 1's uploads go to the other set and
    run while step k's path runs and its results come back (the two copy
    directions use separate copy engines); a set is refilled once the path
    two steps back has read it, and its results are overwritten once they
    have left.  Every step still moves all of its inputs and results."""
    runs = [run]
    free, _ = torch.cuda.mem_get_info()
    if free > 1.5 * torch.cuda.memory_allocated():
        runs.append(Runner(run.workload, "cuda"))
    hosts = [h for h in (t.cpu().pin_memory() for t in run.inputs())]
    outs = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in run.results()]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_c = torch.cuda.current_stream()
    state = [{"computed": None, "drained": None} for _ in runs]
    last = {"drained": None}

    def step(k):
        b = k % len(runs)
        R, st = runs[b], state[b]
        up, done, down = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        with torch.cuda.stream(s_in):
            if st["computed"] is not None:
                s_in.wait_event(st["computed"])      # this set's inputs have been read
            for d, h in zip(R.inputs(), hosts):
                d.copy_(h, non_blocking=True)
            up.record(s_in)
        s_c.wait_event(up)
        if st["drained"] is not None:
            s_c.wait_event(st["drained"])           # this set's results have left
        for r in R.rows:
            r[1]()
        done.record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            for d, h in zip(R.results(), outs):
                h.copy_(d, non_blocking=True)
            down.record(s_out)
        st["computed"], st["drained"] = done, down
        last["drained"] = down

    for k in range(max(len(runs), args.warmup)):
        step(k)
    s_c.wait_event(last["drained"])
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_c)
    s_in.wait_event(e0)
    for k in range(args.steps):
        step(k)
    s_c.wait_event(last["drained"])                # the last results are on the host
    e1.record(s_c)
    torch.cuda.synchronize()
    ms_step = max_over_ranks(pg, e0.elapsed_time(e1)) / args.steps
    h2d = sum(h.numel() * h.element_size() for h in hosts)
    d2h = sum(h.numel() * h.element_size() for h in outs)
    return {"value": round(job_value(world, run.blocks(), ms_step), 1), "unit": UNIT,
            "ms_per_step": round(ms_step, 5), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "device_buffer_sets": len(runs),
            "overlap": "uploads of step k+1 (into the other buffer set) with the path and the "
                       "downloads of step k; separate streams and copy engines"}


# ------------------------------------------------------------------ CPU arm
def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def cpu_baseline(run, budget_s=15.0):
    """The oracle, as it stands, on a bounded sample of the same workload: the
    step's rows on the first weight rows, the Gram on the same fraction of the
    calibration tokens (fake-quant on the same fraction of activation rows);
    blocks/s over the sample."""
    import oracle
    oracle.lib()
    if run.workload == "w4a4_gemm":
        # the weight is quantised once (setup, not timed); the step is the
        # activations' fake-quant and the product, on leading rows of X
        wb = _bits(run.gemm_w)
        wsg = oracle.global_scale(wb)
        wc = oracle.scale_search_max(wb, wsg)
        wp = oracle.quantize_pack(wb, wsg, wc)
        X = run.fq_input

        def step(n):
            t0 = time.perf_counter()
            _, ap, ac, asg = oracle.fake_quant(_bits(X[:n]))
            oracle.gemm_nvfp4(ap, ac, asg, wp, wc, wsg)
            return time.perf_counter() - t0
        t1, t2 = step(4), step(16)
        per_row = max((t2 - t1) / 12, 1e-6)
        n = int(max(1, min(X.shape[0], (budget_s - max(t1 - 4 * per_row, 0.0)) / per_row)))
        t = step(n)
        blocks = n * X.shape[1] // 16
        return {"value": round(blocks / t, 2), "unit": UNIT, "cores": oracle.max_threads(),
                "kind": "oracle", "seconds": round(t, 3),
                "sample": "fake-quant of %d of %d token rows and their product with the "
                          "8192x8192 NVFP4 weight (%d activation blocks)"
                          % (n, X.shape[0], blocks)}
    if run.workload == "act_calib":
        X = run.fq_input

        def step(n):
            xu = _bits(X[:n])
            t0 = time.perf_counter()
            h = oracle.abs_histogram(xu)
            sg = oracle.static_scale(oracle.quantile_magnitude(h, 0.9999))
            oracle.fake_quant_static(xu, sg)
            return time.perf_counter() - t0
        t1, t2 = step(64), step(256)
        per_row = max((t2 - t1) / 192, 1e-7)
        n = int(max(1, min(X.shape[0], (budget_s - max(t1 - 64 * per_row, 0.0)) / per_row)))
        t = step(n)
        blocks = n * X.shape[1] // 16
        return {"value": round(blocks / t, 2), "unit": UNIT, "cores": oracle.max_threads(),
                "kind": "oracle", "seconds": round(t, 3),
                "sample": "histogram, 99.99th-percentile scale and static fake-quant of %d of "
                          "%d token rows (%d blocks)" % (n, X.shape[0], blocks)}
    if not run.layers:  # activation-only workload: fake-quant on leading rows
        X = run.fq_input
        t0 = time.perf_counter()
        oracle.fake_quant(_bits(X[:64]))
        per_row = (time.perf_counter() - t0) / 64
        n = int(max(1, min(X.shape[0], budget_s / max(per_row, 1e-6))))
        xu = _bits(X[:n])
        t0 = time.perf_counter()
        oracle.fake_quant(xu)
        t = time.perf_counter() - t0
        blocks = n * X.shape[1] // 16
        return {"value": round(blocks / t, 2), "unit": UNIT, "cores": oracle.max_threads(),
                "kind": "oracle", "seconds": round(t, 3),
                "sample": "fake-quant of %d of %d token rows (%d blocks)"
                          % (n, X.shape[0], blocks)}
    L = run.layers[0]
    if L.B > 1:
        return _cpu_baseline_experts(run, L, budget_s)
    W = L.W[0]
    R, C = W.shape
    wu_all = _bits(W)
    if L.chunks is not None:
        X = L.chunks[0]
    elif L.offsets is not None:
        X = L.X[int(L.offsets[0]):int(L.offsets[1])]
    else:
        X = L.X
    n_tok_total = 0 if X is None else (L.tokens() if L.offsets is None else X.shape[0])

    def path(rows):
        frac = rows / R
        x_rows = 0 if X is None else min(X.shape[0], max(16, int(n_tok_total * frac)))
        xu = None if X is None else _bits(X[:x_rows])
        fq = None
        if run.fq_input is not None:
            fq = _bits(run.fq_input[:max(1, int(run.fq_input.shape[0] * frac))])
        t0 = time.perf_counter()
        sg = oracle.global_scale(wu_all)
        H = None if xu is None else oracle.gram(xu)
        Hf = oracle.gram_full(xu) if run.gptq else None
        wu = np.ascontiguousarray(wu_all[:rows])
        if "max" in run.rules:
            oracle.scale_search_max(wu, sg)
        if "four_over_six" in run.rules:
            codes = oracle.scale_search_four_over_six(wu, sg)
        if "mse" in run.rules:
            oracle.scale_search_mse(wu, sg)
        if "lh" in run.rules:
            codes, _ = oracle.scale_search_lh(wu, sg, H)
        if run.gptq:
            U = oracle.gptq_factor(Hf, GPTQ_DAMP)
            packed, _ = oracle.gptq_rows(wu, sg, codes, U, np.arange(rows))
        else:
            packed = oracle.quantize_pack(wu, sg, codes)
        oracle.dequantize(packed, codes, sg)
        if fq is not None:
            oracle.fake_quant(fq)
        return time.perf_counter() - t0, x_rows

    # time = fixed part (tensor scale, thread start-up) + per-row part, fitted
    # from two probes, then the sample sized to the budget
    p1, p2 = min(R, 32), min(R, 128)
    t1, _ = path(p1)
    t2, _ = path(p2)
    per_row = max((t2 - t1) / max(p2 - p1, 1), 1e-7)
    fixed = max(t1 - p1 * per_row, 0.0)
    rows = int(max(1, min(R, (budget_s - fixed) / per_row)))
    t, x_rows = path(rows)
    blocks = rows * C // 16
    return {"value": round(blocks / t, 2), "unit": UNIT, "cores": oracle.max_threads(),
            "kind": "oracle", "seconds": round(t, 3),
            "sample": "the step's rows on %d of %d weight rows (%d blocks) of %s with %d "
                      "calibration tokens (the same fraction); blocks/s over the sample"
                      % (rows, R, blocks, L.name, x_rows)}


def _cpu_baseline_experts(run, L, budget_s):
    """Batched experts: the step's rows (tensor scale, Gram of the expert's
    routed tokens, the search, pack, dequantise) on whole experts 0, 1, ...
    as many as the budget takes (expert 0 has the most tokens, so the probe
    on it over-estimates the later ones); blocks/s over the sample."""
    import oracle
    off = None if L.offsets is None else [int(v) for v in L.offsets.cpu()]

    def inputs(e):
        return _bits(L.W[e]), None if off is None else _bits(L.X[off[e]:off[e + 1]])

    def experts(data):
        t0 = time.perf_counter()
        for wu, xu in data:
            sg = oracle.global_scale(wu)
            if "lh" in run.rules:
                codes, _ = oracle.scale_search_lh(wu, sg, oracle.gram(xu))
            elif "four_over_six" in run.rules:
                codes = oracle.scale_search_four_over_six(wu, sg)
            else:
                codes = oracle.scale_search_max(wu, sg)
            packed = oracle.quantize_pack(wu, sg, codes)
            oracle.dequantize(packed, codes, sg)
        return time.perf_counter() - t0

    t1 = experts([inputs(0)])
    n = int(max(1, min(L.B, budget_s / max(t1, 1e-6))))
    data = [inputs(e) for e in range(n)]
    t = experts(data)
    blocks = n * L.R * L.C // 16
    calib = "" if off is None else " with their %d routed calibration tokens" % (off[n] - off[0])
    return {"value": round(blocks / t, 2), "unit": UNIT, "cores": oracle.max_threads(),
            "kind": "oracle", "seconds": round(t, 3),
            "sample": "the step's rows on experts 0..%d of %d (%d blocks)%s; blocks/s over the "
                      "sample" % (n - 1, L.B, blocks, calib)}


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return
    small = args.workload in ("tiny", "dense", "w4a4", "w4a4_gemm", "act_calib", "lh_gptq")
    dev = "cpu" if small or not torch.cuda.is_available() else "cuda"
    run = Runner(args.workload, dev)
    budget = args.cpu_seconds / max(1, args.steps)
    for _ in range(args.warmup):
        cpu_baseline(run, budget_s=min(budget, 2.0))
    steps = [cpu_baseline(run, budget_s=budget) for _ in range(args.steps)]
    v = statistics.mean(s["value"] for s in steps)
    ms = statistics.mean(s["seconds"] for s in steps) * 1e3
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": UNIT,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
           "config": {"workload": args.workload, "desc": run.desc},
           "cpu_baseline": {"value": round(v, 2), "unit": UNIT, "cores": steps[-1]["cores"],
                            "kind": "oracle", "sample": steps[-1]["sample"]},
           "e2e": {"value": round(v, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOAD_NAMES)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warmup raised to 3")
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()

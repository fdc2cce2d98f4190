"""Benchmark of the NVFP4 calibration path on B200.

One step = one pass of the whole path over one layer of the chosen workload
(default: dense projection, W 4096x4096, X 2048x4096):

    global scale(W) -> Gram(X) -> max rule -> MSE search -> Local-Hessian
    search -> quantise+pack (Local-Hessian codes) -> dequantise ->
    W4A4 fake-quant(X)

Metric: NVFP4 weight blocks per second through the whole path (the
Local-Hessian search dominates).  Inputs are resident in HBM; the L2 cache is
flushed (a 256 MiB write) before every timed step, outside the step's CUDA
events.  Per-row kernel times are CUDA events on the launching stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dense|tiny|moe|mlp_pair]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no cross-GPU exchange); timing is the max over ranks.
"""
import argparse
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

ROWS = ["global_scale", "gram", "search_max", "search_mse", "search_lh", "quantize_pack",
        "dequantize", "fake_quant"]
# kernels of this library launched by each row (memsets are not kernels)
LAUNCHES = {"global_scale": 2, "gram": 2, "search_max": 1, "search_mse": 1, "search_lh": 1,
            "quantize_pack": 1, "dequantize": 1, "fake_quant": 3}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ inputs
def make_inputs(workload, device):
    from scale_calibration_nvfp4_b200 import workloads
    if workload in ("tiny", "dense"):
        W, X = workloads.layer_inputs(workload, device)
        return dict(W=W.unsqueeze(0), X=X, offsets=None, desc=workloads.BY_NAME[workload].description)
    if workload == "moe":
        W, X, offsets = workloads.moe_inputs(device)
        return dict(W=W, X=X, offsets=offsets.to(device), desc=workloads.BY_NAME["moe"].description)
    if workload == "mlp_pair":
        up, _ = workloads.mlp_weights(device)
        X = workloads.mlp_chunk("up", 0, device)
        return dict(W=up.unsqueeze(0), X=X, offsets=None,
                    desc="up projection 12288x4096 with one 65,536-token Student-t chunk")
    raise ValueError(workload)


class Path:
    """Preallocated outputs and the per-row calls of one step."""

    def __init__(self, inp):
        from scale_calibration_nvfp4_b200 import nvfp4
        self.nv = nvfp4
        self.W, self.X, self.offsets = inp["W"], inp["X"], inp["offsets"]
        B, R, C = self.W.shape
        dev = self.W.device
        self.B, self.R, self.C = B, R, C
        self.s_g = torch.empty(B, dtype=torch.float32, device=dev)
        self.H = torch.zeros(B, C // 16, 16, 16, dtype=torch.float32, device=dev)
        self.c_max = torch.empty(B, R, C // 16, dtype=torch.uint8, device=dev)
        self.c_mse = torch.empty_like(self.c_max)
        self.c_lh = torch.empty_like(self.c_max)
        self.packed = torch.empty(B, R, C // 2, dtype=torch.uint8, device=dev)
        self.deq = torch.empty(B, R, C, dtype=torch.bfloat16, device=dev)
        self.fq = torch.empty_like(self.X)

    def row(self, name):
        nv = self.nv
        if name == "global_scale":
            nv.global_scale(self.W, batch=self.B, out=self.s_g)
        elif name == "gram":
            if self.offsets is None:
                nv.hessian_accumulate(self.X, self.H[0])
            else:
                nv.hessian_accumulate_grouped(self.X, self.offsets, self.H)
        elif name == "search_max":
            nv.scale_search_max(self.W, self.s_g, out=self.c_max)
        elif name == "search_mse":
            nv.scale_search_mse(self.W, self.s_g, out=self.c_mse)
        elif name == "search_lh":
            nv.scale_search_local_hessian(self.W, self.s_g, self.H, out=self.c_lh)
        elif name == "quantize_pack":
            nv.quantize_pack(self.W, self.s_g, self.c_lh, out=self.packed)
        elif name == "dequantize":
            nv.dequantize(self.packed, self.c_lh, self.s_g, out=self.deq)
        elif name == "fake_quant":
            nv.fake_quant(self.X, want_packed=False, out=self.fq)

    def blocks(self):
        return self.B * self.R * self.C // 16

    def algorithmic_bytes(self):
        """Bytes each row must move at least (read + write), per step."""
        n_w = self.B * self.R * self.C
        n_x = self.X.numel()
        nb = n_w // 16
        h = self.H.numel() * 4
        return {
            "global_scale": 2 * n_w,
            "gram": 2 * n_x + 2 * h,
            "search_max": 2 * n_w + nb,
            "search_mse": 2 * n_w + nb,
            "search_lh": 2 * n_w + nb + h,
            "quantize_pack": 2 * n_w + nb + n_w // 2,
            "dequantize": n_w // 2 + nb + 2 * n_w,
            "fake_quant": 6 * n_x,
        }


# Local-Hessian search work per block, counted on the definition E = delta
# H_b delta^T: per candidate 256 FMA for H_b delta and 16 FMA for the dot
# product, 2 flop each (the E2M1 encodes are not counted as flops).
LH_FLOP_PER_BLOCK = 126 * 2 * (256 + 16)


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


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "scale_calibration_nvfp4_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    ent = t.get(kernel, {}).get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


def dist_env():
    if "RANK" in os.environ and "WORLD_SIZE" in os.environ:
        return int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"]), \
            int(os.environ.get("LOCAL_RANK", os.environ["RANK"]))
    return 0, 1, 0


# ------------------------------------------------------------------ GPU arm
def run_gpu(args):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        pg = dist
    from scale_calibration_nvfp4_b200 import build, nvfp4
    if rank == 0:
        build.build()
    if pg:
        pg.barrier()
    nvfp4.lib()

    inp = make_inputs(args.workload, "cuda")
    path = Path(inp)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")

    def step(events=None):
        for i, name in enumerate(ROWS):
            if events is not None:
                events[i].record(stream)
            path.row(name)
        if events is not None:
            events[-1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ROWS) + 1)]
          for _ in range(args.steps)]
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.zero_()
        step(ev[k])
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clk = clocks.stop() if clocks else None

    per_row = {n: [] for n in ROWS}
    step_ms = []
    for k in range(args.steps):
        for i, n in enumerate(ROWS):
            per_row[n].append(ev[k][i].elapsed_time(ev[k][i + 1]))
        step_ms.append(ev[k][0].elapsed_time(ev[k][-1]))
    ms_total = sum(step_ms)
    if pg:
        t = torch.tensor([ms_total], dtype=torch.float64, device="cuda")
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        ms_total = t.item()
    ms_per_step = ms_total / args.steps
    blocks = path.blocks()
    value = world * blocks / (ms_per_step / 1e3)

    # end to end through the C ABI with host buffers
    e2e = run_e2e(path, inp, args, pg, world) if not args.no_e2e else None

    if rank == 0:
        pk, pk_kind = peaks()
        rows_ms = {n: statistics.mean(v) for n, v in per_row.items()}
        alg = path.algorithmic_bytes()
        kernels = {}
        for n in ROWS:
            kernels[n] = {"ms": round(rows_ms[n], 5),
                          "GB/s": round(alg[n] / (rows_ms[n] / 1e3) / 1e9, 1)}
        lh_ms = rows_ms["search_lh"]
        sm_mhz_peak = float(pk.get("sm_max_mhz", 1965.0))
        fp32_peak = SM_COUNT * FP32_LANES_PER_SM * 2 * sm_mhz_peak * 1e6 / 1e12
        achieved = LH_FLOP_PER_BLOCK * blocks / (lh_ms / 1e3) / 1e12
        roofline = {
            "kernel": "search_kernel<Local-Hessian>",
            "bound": "alu", "achieved": round(achieved, 2), "peak": round(fp32_peak, 2),
            "unit": "TFLOP/s", "frac": round(achieved / fp32_peak, 4),
            "traffic": recorded_traffic("search_lh", args.workload),
            "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 2 flop x %.0f MHz (%s clocks)"
                         % (sm_mhz_peak, pk_kind),
            "flop_per_block": LH_FLOP_PER_BLOCK,
            "flop_basis": "definition delta H delta^T: 126 x (256 + 16) FMA per block",
        }
        hbm = float(pk.get("hbm_gbs", FALLBACK_HBM_GBS))
        streaming = {n: {"GB/s": kernels[n]["GB/s"], "frac_of_%s_hbm" % pk_kind:
                         round(kernels[n]["GB/s"] / hbm, 3)}
                     for n in ("gram", "quantize_pack", "dequantize", "fake_quant",
                               "global_scale", "search_max")}
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; no dataset or trained weights)",
            "config": {"workload": args.workload, "desc": inp["desc"],
                       "blocks_per_step": blocks, "rows": ROWS,
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "cache": "L2 flushed (256 MiB write) before every timed step"},
            "roofline": roofline,
            "hbm_kernels": streaming,
            "kernels": kernels,
            "gpu_launches": args.steps * sum(LAUNCHES.values()),
            "clocks": clk,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline and world == 1:
            out["cpu_baseline"] = cpu_baseline(args.workload, inp, budget_s=args.cpu_seconds)
        print(json.dumps(out), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def run_e2e(path, inp, args, pg, world):
    """Same metric through the public API with host buffers: every step copies
    W and X from pinned host memory to the device, runs the path and reads
    the Local-Hessian codes and packed weights back."""
    W_h = path.W.cpu().pin_memory()
    X_h = path.X.cpu().pin_memory()
    codes_h = torch.empty(path.c_lh.shape, dtype=torch.uint8).pin_memory()
    packed_h = torch.empty(path.packed.shape, dtype=torch.uint8).pin_memory()
    stream = torch.cuda.current_stream()

    def step():
        path.W.copy_(W_h, non_blocking=True)
        path.X.copy_(X_h, non_blocking=True)
        for name in ROWS:
            path.row(name)
        codes_h.copy_(path.c_lh, non_blocking=True)
        packed_h.copy_(path.packed, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if pg:
        t = torch.tensor([ms], dtype=torch.float64, device="cuda")
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        ms = t.item()
    ms_step = ms / args.steps
    h2d = W_h.numel() * 2 + X_h.numel() * 2
    d2h = codes_h.numel() + packed_h.numel()
    return {"value": round(world * path.blocks() / (ms_step / 1e3), 1), "unit": UNIT,
            "ms_per_step": round(ms_step, 5), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h}


# ------------------------------------------------------------------ CPU arm
def cpu_baseline(workload, inp, budget_s=15.0):
    """The oracle, as it stands, on a bounded sample of the same workload: the
    whole path on the first rows of the (first) weight, the Gram on a
    proportional share of the tokens; blocks/s extrapolated from the sample."""
    import oracle
    oracle.lib()

    def bits(t):
        return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    W = inp["W"][0]
    X = inp["X"]
    R, C = W.shape
    wu_all = bits(W)
    # calibrate the sample size with a short probe, then run ~budget_s
    probe_rows = max(1, min(R, 8))
    t_probe = _oracle_path(wu_all, bits(X[: max(16, X.shape[0] * probe_rows // R)]), probe_rows)
    rows = int(max(1, min(R, probe_rows * budget_s / max(t_probe, 1e-3))))
    x_rows = max(16, X.shape[0] * rows // R)
    t = _oracle_path(wu_all, bits(X[:x_rows]), rows)
    blocks = rows * C // 16
    return {"value": round(blocks / t, 2), "unit": UNIT, "cores": oracle.max_threads(),
            "kind": "oracle", "seconds": round(t, 3),
            "sample": "whole path on %d of %d weight rows (%d blocks) with %d of %d "
                      "calibration tokens; blocks/s over the sample" % (rows, R, blocks, x_rows,
                                                                       X.shape[0])}


def _oracle_path(wu_all, xu, rows):
    import oracle
    t0 = time.perf_counter()
    sg = oracle.global_scale(wu_all)
    H = oracle.gram(xu)
    wu = np.ascontiguousarray(wu_all[:rows])
    oracle.scale_search_max(wu, sg)
    oracle.scale_search_mse(wu, sg)
    codes, _ = oracle.scale_search_lh(wu, sg, H)
    packed = oracle.quantize_pack(wu, sg, codes)
    oracle.dequantize(packed, codes, sg)
    oracle.fake_quant(xu, want_packed=False)
    return time.perf_counter() - t0


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return
    inp = make_inputs(args.workload, "cpu")
    steps = []
    cb = None
    for k in range(args.warmup + args.steps):
        cb = cpu_baseline(args.workload, inp, budget_s=args.cpu_seconds / max(1, args.steps))
        if k >= args.warmup:
            steps.append(cb)
    v = statistics.mean(s["value"] for s in steps)
    ms = statistics.mean(s["seconds"] for s in steps) * 1e3
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": UNIT,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
           "config": {"workload": args.workload, "desc": inp["desc"]},
           "cpu_baseline": {"value": round(v, 2), "unit": UNIT, "cores": cb["cores"],
                            "kind": "oracle", "sample": cb["sample"]},
           "e2e": {"value": round(v, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dense", choices=["dense", "tiny", "moe", "mlp_pair"])
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

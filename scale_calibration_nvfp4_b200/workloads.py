"""Seeded synthetic inputs for the NVFP4 calibration workloads.

This module draws random numbers and nothing else: it holds none of the
quantisation arithmetic, and both the CUDA path and the CPU oracle consume
its outputs.  Every tensor is drawn in fp32 and cast to bf16 (round to
nearest even).  Draw order inside one workload is fixed: weights, weight
outlier positions, activations, activation outlier channels.  Outlier
entries are an exact count picked with ``randperm`` and multiplied in
place; outlier channels are whole activation columns.

The five named workloads follow the sizes of the calibration recipe in the
Local-Hessian write-up ("4 比特量化到底让模型笨了多少？", section on trying it
yourself: 512 samples of sequence length 2048).  No dataset or trained
weights are involved.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_with_outliers(rows: int, cols: int, std: float, n_outliers: int, factor: float,
                           seed: int, device="cpu", gen: Optional[torch.Generator] = None):
    """bf16 [rows, cols] ~ N(0, std) with ``n_outliers`` entries multiplied by ``factor``."""
    g = gen if gen is not None else _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
    if n_outliers > 0:
        idx = torch.randperm(rows * cols, generator=g, device=device)[:n_outliers]
        x.view(-1)[idx] *= factor
    return x.to(torch.bfloat16)


def activations_with_outlier_channels(tokens: int, cols: int, n_channels: int, factor: float,
                                      seed: int, device="cpu",
                                      gen: Optional[torch.Generator] = None, std: float = 1.0):
    """bf16 [tokens, cols] ~ N(0, std) with ``n_channels`` whole columns times ``factor``."""
    g = gen if gen is not None else _gen(seed, device)
    x = torch.randn(tokens, cols, generator=g, device=device, dtype=torch.float32) * std
    if n_channels > 0:
        ch = torch.randperm(cols, generator=g, device=device)[:n_channels]
        x[:, ch] *= factor
    return x.to(torch.bfloat16)


def student_t4(tokens: int, cols: int, seed: int, device="cpu",
               gen: Optional[torch.Generator] = None):
    """bf16 [tokens, cols] Student-t with 4 degrees of freedom, unit scale:
    t = Z / sqrt(chi2_4 / 4) with chi2_4 = -2 ln(U1 U2)."""
    g = gen if gen is not None else _gen(seed, device)
    z = torch.randn(tokens, cols, generator=g, device=device, dtype=torch.float32)
    u1 = torch.rand(tokens, cols, generator=g, device=device, dtype=torch.float32)
    u2 = torch.rand(tokens, cols, generator=g, device=device, dtype=torch.float32)
    # rand is in [0, 1); map to (0, 1] so the logarithm stays finite
    chi2 = -2.0 * (torch.log1p(-u1) + torch.log1p(-u2))
    return (z / torch.sqrt(chi2 * 0.25)).to(torch.bfloat16)


def zipf_counts(total: int, groups: int, alpha: float, seed: int):
    """Routed token counts per expert: multinomial(total, p_e ~ (e+1)^-alpha), on the CPU."""
    g = _gen(seed, "cpu")
    p = torch.arange(1, groups + 1, dtype=torch.float64).pow(-alpha)
    p = p / p.sum()
    draws = torch.multinomial(p, total, replacement=True, generator=g)
    return torch.bincount(draws, minlength=groups).to(torch.int64)


@dataclass
class Workload:
    name: str
    description: str
    seed: int
    params: dict = field(default_factory=dict)


WORKLOADS: List[Workload] = [
    Workload("tiny", "W 256x512 N(0,0.02), 1% entries x20; X 512x512 N(0,1), 4 channels x30",
             0, dict(R=256, C=512, w_std=0.02, w_out_frac=0.01, w_out=20.0,
                     N=512, x_ch=4, x_out=30.0)),
    Workload("dense", "W 4096x4096 N(0,0.02), 0.5% entries x15; X 2048x4096 N(0,1), "
             "8 channels (0.2%) x50", 1,
             dict(R=4096, C=4096, w_std=0.02, w_out_frac=0.005, w_out=15.0,
                  N=2048, x_ch=8, x_out=50.0)),
    Workload("mlp_pair", "up W 12288x4096 and down W 4096x12288 N(0,0.015); "
             "1,048,576 calibration tokens in 16 chunks of 65,536, Student-t(4)", 2,
             dict(up=(12288, 4096), down=(4096, 12288), w_std=0.015, chunks=16,
                  chunk_tokens=65536)),
    Workload("moe", "128 experts W_e 768x2048 N(0,0.02); 262,144 routed tokens, counts "
             "multinomial with p_e ~ (e+1)^-1.1; X N(0,1) with 4 channels x30", 3,
             dict(G=128, R=768, C=2048, w_std=0.02, tokens=262144, alpha=1.1,
                  x_ch=4, x_out=30.0)),
    Workload("w4a4", "X 32768x8192 N(0,1) with 82 channels (1%) x40", 4,
             dict(N=32768, C=8192, x_ch=82, x_out=40.0)),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def layer_inputs(name: str, device="cpu"):
    """(W, X) of the single-layer workloads ``tiny`` and ``dense``."""
    wl = BY_NAME[name]
    p = wl.params
    g = _gen(wl.seed, device)
    n_out = int(round(p["w_out_frac"] * p["R"] * p["C"]))
    W = gaussian_with_outliers(p["R"], p["C"], p["w_std"], n_out, p["w_out"], wl.seed,
                               device, gen=g)
    X = activations_with_outlier_channels(p["N"], p["C"], p["x_ch"], p["x_out"], wl.seed,
                                          device, gen=g)
    return W, X


def mlp_weights(device="cpu"):
    wl = BY_NAME["mlp_pair"]
    p = wl.params
    g = _gen(wl.seed, device)
    up = gaussian_with_outliers(*p["up"], p["w_std"], 0, 1.0, wl.seed, device, gen=g)
    down = gaussian_with_outliers(*p["down"], p["w_std"], 0, 1.0, wl.seed, device, gen=g)
    return up, down


def mlp_chunk(which: str, k: int, device="cpu", tokens: Optional[int] = None):
    """Calibration chunk k (0..15) for the ``up`` (4096 channels) or ``down``
    (12288 channels) projection; each chunk has its own seed so that any chunk
    can be regenerated alone."""
    wl = BY_NAME["mlp_pair"]
    p = wl.params
    cols = p["up"][1] if which == "up" else p["down"][1]
    seed = wl.seed * 1000 + (0 if which == "up" else 500) + k
    return student_t4(tokens or p["chunk_tokens"], cols, seed, device)


def moe_inputs(device="cpu"):
    """(W [G, R, C], X [sum n_g, C] sorted by expert, offsets [G+1] int64 CPU)."""
    wl = BY_NAME["moe"]
    p = wl.params
    counts = zipf_counts(p["tokens"], p["G"], p["alpha"], wl.seed)
    offsets = torch.zeros(p["G"] + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(counts, 0)
    g = _gen(wl.seed, device)
    W = gaussian_with_outliers(p["G"] * p["R"], p["C"], p["w_std"], 0, 1.0, wl.seed, device,
                               gen=g).view(p["G"], p["R"], p["C"])
    X = activations_with_outlier_channels(p["tokens"], p["C"], p["x_ch"], p["x_out"], wl.seed,
                                          device, gen=g)
    return W, X, offsets


def w4a4_inputs(device="cpu"):
    wl = BY_NAME["w4a4"]
    p = wl.params
    g = _gen(wl.seed, device)
    return activations_with_outlier_channels(p["N"], p["C"], p["x_ch"], p["x_out"], wl.seed,
                                             device, gen=g)

"""Seeded synthetic inputs for the QLoRA NF4 layer workloads.

This module only draws random tensors and describes workload shapes; it holds
none of the method's arithmetic. Both the CUDA path and the CPU oracle are
fed from it (the same bytes, copied between devices), so neither side needs a
generator of its own.

Workloads (sizes of the pages' examples and of common Llama shapes):

* ``tiny``      one 256 -> 512 layer, 32 tokens, rank 8, alpha 16;
* ``l4096``     one 4096 x 4096 layer, 4096 tokens, rank 64, alpha 128, with 0.1 %
                outliers scaled by 10 in W;
* ``llama7b``   the seven projections of a Llama-7B block (q, k, v, o 4096x4096;
                gate, up 11008x4096; down 4096x11008), std 0.02 jittered +-20 %;
* ``decode7b``  the same block with 1, 4 or 16 tokens, rank 16 on q, k, v, o only;
* ``l70b``      a 70B-like block (q, o 8192x8192; k, v 1024x8192; gate, up
                28672x8192; down 8192x28672), std 0.015, rank 64, alpha 128, 4096 tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

LLAMA7B_PROJ = [  # (name, d_out, d_in) in the nn.Linear [d_out, d_in] layout
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
]
L70B_PROJ = [
    ("q", 8192, 8192), ("k", 1024, 8192), ("v", 1024, 8192), ("o", 8192, 8192),
    ("gate", 28672, 8192), ("up", 28672, 8192), ("down", 8192, 28672),
]


@dataclass
class Layer:
    name: str
    d_out: int
    d_in: int
    w_std: float
    r: int = 0            # 0: no adapter
    alpha: float = 0.0
    a_std: float = 0.02
    b_std: float = 0.02
    outlier_frac: float = 0.0
    outlier_scale: float = 10.0

    @property
    def s(self) -> float:
        return self.alpha / self.r if self.r else 0.0


@dataclass
class Workload:
    name: str
    layers: list = field(default_factory=list)
    M: int = 0            # tokens
    w_dtype: str = "f32"  # dtype W is handed to the quantiser in
    seed: int = 0
    std_jitter: float = 0.0


def workload(name: str, M: int | None = None, n_layers: int = 1) -> Workload:
    if name == "tiny":
        return Workload("tiny", [Layer("l0", 512, 256, 0.02, r=8, alpha=16)], M=32, seed=1000)
    if name == "l4096":
        return Workload("l4096", [Layer("l0", 4096, 4096, 0.02, r=64, alpha=128, a_std=0.02, b_std=0.01,
                                        outlier_frac=0.001)], M=4096, seed=2000)
    if name == "llama7b":
        layers = []
        for li in range(n_layers):
            for (p, o, i) in LLAMA7B_PROJ:
                layers.append(Layer(f"L{li}.{p}", o, i, 0.02))
        return Workload("llama7b", layers, M=0, w_dtype="bf16", seed=3000, std_jitter=0.2)
    if name == "decode7b":
        layers = []
        for (p, o, i) in LLAMA7B_PROJ:
            r = 16 if p in ("q", "k", "v", "o") else 0
            layers.append(Layer(p, o, i, 0.02, r=r, alpha=32 if r else 0.0))
        return Workload("decode7b", layers, M=1 if M is None else M, w_dtype="bf16", seed=4000)
    if name == "l70b":
        layers = [Layer(p, o, i, 0.015, r=64, alpha=128) for (p, o, i) in L70B_PROJ]
        return Workload("l70b", layers, M=4096, seed=5000)
    raise KeyError(name)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int, device="cpu", dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from a seeded generator, then cast to dtype."""
    g = _gen(device, seed)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype) if dtype != torch.float32 else t


def weight(layer: Layer, seed: int, device="cpu", dtype=torch.float32, std_jitter: float = 0.0) -> torch.Tensor:
    """A frozen weight [d_out, d_in]: N(0, std^2), std jittered per matrix by
    a factor in [1-j, 1+j]; optionally a fraction of entries scaled (outliers)."""
    std = layer.w_std
    if std_jitter:
        u = torch.rand(1, generator=_gen("cpu", seed + 7919)).item()
        std = std * (1.0 - std_jitter + 2.0 * std_jitter * u)
    w = normal((layer.d_out, layer.d_in), std, seed, device=device)
    if layer.outlier_frac > 0:
        g = _gen(device, seed + 104729)
        mask = torch.rand(layer.d_out, layer.d_in, generator=g, device=device) < layer.outlier_frac
        w = torch.where(mask, w * layer.outlier_scale, w)
    return w.to(dtype) if dtype != torch.float32 else w


def seed_of(wl: Workload, layer_index: int, tensor: str) -> int:
    """Per-tensor seed: workload base seed + layer index and tensor slot."""
    slot = {"W": 0, "X": 1, "A": 2, "B": 3, "dY": 4}[tensor]
    return wl.seed + 10 * layer_index + slot


def layer_inputs(wl: Workload, li: int, device="cpu", M: int | None = None, w_device=None):
    """All tensors of layer li: W (fp32 or bf16), X, dY (bf16 [M, .]), A [d_in, r], B [r, d_out] (bf16)."""
    L = wl.layers[li]
    M = wl.M if M is None else M
    wdt = torch.bfloat16 if wl.w_dtype == "bf16" else torch.float32
    out = {"W": weight(L, seed_of(wl, li, "W"), device=w_device or device, dtype=wdt, std_jitter=wl.std_jitter)}
    if M:
        out["X"] = normal((M, L.d_in), 1.0, seed_of(wl, li, "X"), device=device, dtype=torch.bfloat16)
        out["dY"] = normal((M, L.d_out), 1.0, seed_of(wl, li, "dY"), device=device, dtype=torch.bfloat16)
    if L.r:
        out["A"] = normal((L.d_in, L.r), L.a_std, seed_of(wl, li, "A"), device=device, dtype=torch.bfloat16)
        out["B"] = normal((L.r, L.d_out), L.b_std, seed_of(wl, li, "B"), device=device, dtype=torch.bfloat16)
    return out

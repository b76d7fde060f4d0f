"""Seeded synthetic inputs for the rotated W4A4 linear layer.

This module holds no arithmetic of the method: it only draws random bf16
tensors of the shapes and value distributions the layer is exercised on, so
that the CUDA path and the CPU oracle see identical bytes.  Everything is
drawn on the CPU from one ``torch.Generator`` per workload, in a fixed order:
activations, weights, bias, then outlier positions; values are drawn in fp32,
scaled, and cast to bf16 with round-to-nearest-even.

The shapes stand in for the pages' workloads: a small layer of the kind the
"convrot-mlx" README's core example builds (64 x 1024 -> 1024), transformer
linears shaped like a FLUX-style DiT block at 512 x 512 (1536 tokens, hidden
3072, MLP 12288), a fused QKV projection, a square compute-bound layer, and a
skinny decode-size sweep.  No model weights or datasets are used.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Linear:
    """One linear layer: y[M][N] = x[M][K] W[N][K]^T + b[N], rotated in groups."""
    M: int
    K: int
    N: int
    group: int
    bias: bool = True                # bias N(0, 0.02^2) when True, zeros otherwise
    act_outlier_frac: float = 0.0    # fraction of activation channels scaled
    act_outlier_scale: float = 1.0
    w_outlier_frac: float = 0.0      # fraction of weight entries scaled
    w_outlier_scale: float = 1.0


@dataclass(frozen=True)
class Workload:
    name: str
    layers: tuple                    # one Linear, or two chained (MLP pair)
    description: str
    seed: int = 0
    chained: bool = False            # second layer's input is the first's output

    @property
    def ops(self) -> int:
        """Integer multiply-adds x 2 over all layers (2 M N K each)."""
        return sum(2 * l.M * l.N * l.K for l in self.layers)

    @property
    def tokens(self) -> int:
        return self.layers[0].M


WORKLOADS = {
    "small_g256": Workload(
        "small_g256", (Linear(64, 1024, 1024, 256),),
        "64 x 1024 -> 1024, group 256, x N(0,1), W N(0,0.02^2), bias N(0,0.02^2)"),
    "outlier_g64": Workload(
        "outlier_g64",
        (Linear(1024, 3072, 3072, 64, bias=False, act_outlier_frac=0.01, act_outlier_scale=50.0,
                w_outlier_frac=0.001, w_outlier_scale=10.0),),
        "1024 x 3072 -> 3072, group 64, 1% of activation channels x50, 0.1% of weights x10, "
        "bias zero"),
    "dit_mlp_g256": Workload(
        "dit_mlp_g256", (Linear(1536, 3072, 12288, 256), Linear(1536, 12288, 3072, 256)),
        "DiT MLP pair, 1536 tokens: 3072 -> 12288 then 12288 -> 3072, group 256, no "
        "nonlinearity between", chained=True),
    "qkv_g256": Workload(
        "qkv_g256", (Linear(4608, 3072, 9216, 256),),
        "fused QKV 4608 x 3072 -> 9216, group 256"),
    "square_g256": Workload(
        "square_g256", (Linear(8192, 8192, 8192, 256),),
        "square 8192 x 8192 -> 8192, group 256"),
}
for _m in (1, 16, 128, 512):
    WORKLOADS[f"skinny_m{_m}_g64"] = Workload(
        f"skinny_m{_m}_g64", (Linear(_m, 4096, 14336, 64, bias=False),),
        f"skinny {_m} x 4096 -> 14336, group 64, bias zero")

# The workload a single benchmark step runs by default: the square 8192^3
# layer, the largest single-GPU configuration and the one whose GEMM target
# (>= 60% of the dense int8 peak at M >= 4096) the layer is measured against.
DEFAULT_BENCH = "square_g256"


def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16).contiguous()


@dataclass
class LayerTensors:
    x: torch.Tensor | None           # bf16 [M][K] (None for a chained layer)
    w: torch.Tensor                  # bf16 [N][K]
    b: torch.Tensor | None           # bf16 [N] or None
    spec: Linear = field(default=None)


def make_layer(spec: Linear, g: torch.Generator, with_x: bool = True) -> LayerTensors:
    x = torch.randn(spec.M, spec.K, generator=g, dtype=torch.float32) if with_x else None
    w = torch.randn(spec.N, spec.K, generator=g, dtype=torch.float32) * 0.02
    b = (torch.randn(spec.N, generator=g, dtype=torch.float32) * 0.02) if spec.bias else None
    if with_x and spec.act_outlier_frac > 0:
        n_ch = int(round(spec.act_outlier_frac * spec.K))
        ch = torch.randperm(spec.K, generator=g)[:n_ch]
        x[:, ch] *= spec.act_outlier_scale
    if spec.w_outlier_frac > 0:
        n_w = int(round(spec.w_outlier_frac * spec.N * spec.K))
        idx = torch.randperm(spec.N * spec.K, generator=g)[:n_w]
        w.view(-1)[idx] *= spec.w_outlier_scale
    return LayerTensors(None if x is None else _bf16(x), _bf16(w),
                        None if b is None else _bf16(b), spec)


def make_workload(name: str, seed: int | None = None) -> list[LayerTensors]:
    wl = WORKLOADS[name]
    g = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    out = []
    for i, spec in enumerate(wl.layers):
        out.append(make_layer(spec, g, with_x=not (wl.chained and i > 0)))
    return out


def make_random_layer(M: int, K: int, N: int, group: int, seed: int, bias: bool = True,
                      x_scale: float = 1.0) -> LayerTensors:
    """An ad-hoc layer with the same distributions (used for parity sweeps)."""
    g = torch.Generator().manual_seed(seed)
    lt = make_layer(Linear(M, K, N, group, bias=bias), g)
    if x_scale != 1.0:
        lt.x = _bf16(lt.x.float() * x_scale)
    return lt


def bf16_bits(t: torch.Tensor):
    """The raw uint16 patterns of a CPU bf16 tensor, as numpy."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)

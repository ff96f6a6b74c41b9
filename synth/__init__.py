"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws Q, K, V and the
upstream gradient dO from one CPU ``torch.Generator`` (seed 0 unless stated),
in float32 and in the order Q, K, V, dO, then rounds to the workload's dtype
(bf16 round-to-nearest-even). Both the oracle and the CUDA path read the same
tensors; the oracle gets the rounded values widened back to float32.

The named workloads stand in for the pages' benchmarks (character text of
length 12288, 64x64x3 image rasters of 12288 values, raw audio of 65536
samples) with their sequence lengths and strides; no dataset is read.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "strided" | "fixed" | "dense"
    mode: str          # "split" | "merged"
    B: int
    H: int
    T: int
    d: int
    l: int
    c: int
    dtype: str         # "f32" | "bf16" | "f16"
    std: float         # standard deviation of Q, K, V
    backward: bool = True
    note: str = field(default="", compare=False)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("strided-split-T256", "strided", "split", 1, 2, 256, 32, 16, 1, "f32", 1.0,
                 note="fp32 N(0,1); forward plus a tiny backward"),
        Workload("fixed-split-T4096", "fixed", "split", 4, 8, 4096, 64, 64, 8, "bf16",
                 64 ** -0.25, note="bf16 N(0,1)/d^(1/4)"),
        Workload("fixed-merged-T12288", "fixed", "merged", 2, 8, 12288, 64, 128, 8, "bf16", 0.5,
                 note="text-like; bf16 std 0.5"),
        Workload("strided-split-T12288", "strided", "split", 4, 16, 12288, 64, 192, 1, "bf16",
                 0.5, note="image-like, 64x64x3 raster, l = one pixel row; bf16 std 0.5"),
        Workload("strided-merged-T65536", "strided", "merged", 1, 8, 65536, 64, 256, 1, "bf16",
                 0.5, note="audio-like; bf16 std 0.5"),
    ]
}

# Order in which the workloads are listed in reports.
ORDER = list(WORKLOADS)


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[name]


def draw(B, H, T, d, dtype="bf16", std=1.0, seed=0, dout_std=1.0):
    """Q, K, V, dO as CPU tensors of the given dtype, [B,H,T,d] contiguous.

    Draw order: Q, K, V, dO, each float32 N(0,1) scaled by its std, then one
    rounding to the target dtype."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, T, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32) * std
    k = torch.randn(shape, generator=g, dtype=torch.float32) * std
    v = torch.randn(shape, generator=g, dtype=torch.float32) * std
    do = torch.randn(shape, generator=g, dtype=torch.float32) * dout_std
    td = torch_dtype(dtype)
    return tuple(x.to(td).contiguous() for x in (q, k, v, do))


def draw_workload(w: Workload, seed=0):
    return draw(w.B, w.H, w.T, w.d, w.dtype, w.std, seed)


def as_f32(x: torch.Tensor):
    """float32 numpy copy (exact for bf16 inputs), for the oracle."""
    return x.detach().to("cpu", torch.float32).contiguous().numpy()

"""Seeded synthetic inputs for the FP4 linear layer.

This module holds no arithmetic of the method: it only draws the activation
matrix A (M x K, tokens x in-features) and the weight matrix W (K x N) with
the shapes and value distributions of the LLaMA-shaped workloads, and casts
them to the workload dtype.  Both the CUDA path and the CPU oracle are fed the
same bytes from here.

Recipe (per layer, generator seeded with 1000 * config_index + layer_index):
  1. A base draw: standard normal, or Student-t(df) formed as
     Z / sqrt(V / df) with V the sum of df squared standard normals.
  2. Outliers: whole channels (columns of A) scaled by a factor, or a number
     of entries chosen uniformly without replacement (among a set of
     channels, or among all entries) scaled by a factor.
  3. W ~ N(0, w_std^2).
  4. Cast fp32 -> bf16 by round-to-nearest-even for bf16 workloads.
The draws use torch generators on the requested device; CPU and CUDA streams
differ, so a test always draws once and hands the same tensors to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch


@dataclass(frozen=True)
class Layer:
    name: str
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    dtype: str               # "f32" or "bf16"
    M: int
    layers: Tuple[Layer, ...]
    dist: Tuple              # ("normal",) or ("student_t", df)
    outliers: Optional[Tuple]  # see _apply_outliers
    w_std: float
    alphas: Tuple[float, ...]
    description: str = ""

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def flops(self) -> int:
        return sum(2 * self.M * l.K * l.N for l in self.layers)


WORKLOADS = {
    "tiny": Workload(
        "tiny", 0, "f32", 256, (Layer("linear", 512, 512),), ("normal",),
        ("channel_entries", 8, 0.005, 50.0), 0.02, (0.99,),
        "single linear, A 256x512 fp32 N(0,1), 0.5% of the entries of 8 channels x50"),
    "llama1.3b": Workload(
        "llama1.3b", 1, "bf16", 4096,
        (Layer("attn_proj", 2048, 2048), Layer("mlp_up", 2048, 5504),
         Layer("mlp_down", 5504, 2048)),
        ("student_t", 4), ("channels", 4, 30.0), 0.02, (0.99,),
        "LLaMA-1.3B-shaped linears, M=4096 tokens, Student-t(4), 4 channels x30"),
    "llama7b": Workload(
        "llama7b", 2, "bf16", 8192,
        (Layer("attn_proj", 4096, 4096), Layer("qkv", 4096, 12288),
         Layer("mlp_gate", 4096, 11008), Layer("mlp_up", 4096, 11008),
         Layer("mlp_down", 11008, 4096)),
        ("student_t", 4), ("random_entries", 0.001, 50.0), 0.02, (0.99,),
        "LLaMA-7B-shaped linears, M=8192, Student-t(4), 0.1% random entries x50"),
    "llama13b": Workload(
        "llama13b", 3, "bf16", 8192,
        (Layer("attn_proj", 5120, 5120), Layer("qkv", 5120, 15360),
         Layer("mlp_gate", 5120, 13824), Layer("mlp_up", 5120, 13824),
         Layer("mlp_down", 13824, 5120)),
        ("normal",), ("channels", 16, 40.0), 0.015, (0.999,),
        "LLaMA-13B-shaped linears, M=8192, N(0,1), 16 channels x40"),
    "block16k": Workload(
        "block16k", 4, "bf16", 16384,
        (Layer("qkv", 4096, 12288), Layer("o", 4096, 4096),
         Layer("gate_up", 4096, 22016), Layer("down", 11008, 4096)),
        ("student_t", 3), None, 0.02, (0.99, 0.999),
        "7B decoder block linear stream at M=16384, Student-t(3)"),
}


def seed_for(workload: Workload, layer_index: int) -> int:
    return 1000 * workload.index + layer_index


def _base(shape, dist, g, device):
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if dist[0] == "normal":
        return z
    if dist[0] == "student_t":
        df = int(dist[1])
        v = torch.zeros(shape, device=device, dtype=torch.float32)
        for _ in range(df):
            e = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            v.addcmul_(e, e)
        return z / torch.sqrt(v / df)
    raise ValueError(dist)


def _apply_outliers(A, spec, g):
    if spec is None:
        return A
    M, K = A.shape
    kind = spec[0]
    if kind == "channels":
        n, factor = int(spec[1]), float(spec[2])
        ch = torch.randperm(K, generator=g, device=A.device)[:n]
        A[:, ch] *= factor
    elif kind == "channel_entries":
        n, frac, factor = int(spec[1]), float(spec[2]), float(spec[3])
        ch = torch.randperm(K, generator=g, device=A.device)[:n]
        count = int(round(frac * M * K))
        pick = torch.randperm(M * n, generator=g, device=A.device)[:count]
        rows = pick // n
        cols = ch[pick % n]
        A[rows, cols] *= factor
    elif kind == "random_entries":
        frac, factor = float(spec[1]), float(spec[2])
        count = int(round(frac * M * K))
        pick = torch.randperm(M * K, generator=g, device=A.device)[:count]
        A.view(-1)[pick] *= factor
    else:
        raise ValueError(kind)
    return A


def make_layer_inputs(workload, layer_index: int = 0, device="cpu", M: Optional[int] = None):
    """Draw (A, W) for one layer of a workload, in the workload dtype.

    ``M`` overrides the token count (used for reduced-size test cases).
    """
    if isinstance(workload, str):
        workload = WORKLOADS[workload]
    layer = workload.layers[layer_index]
    M = workload.M if M is None else int(M)
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(workload, layer_index))
    A = _base((M, layer.K), workload.dist, g, device)
    A = _apply_outliers(A, workload.outliers, g)
    W = torch.randn((layer.K, layer.N), generator=g, device=device,
                    dtype=torch.float32) * workload.w_std
    return A.to(workload.torch_dtype).contiguous(), W.to(workload.torch_dtype).contiguous()


def make_matrix(shape, dist=("normal",), seed=0, device="cpu", dtype=torch.float32,
                outliers=None, scale=1.0):
    """A generic seeded matrix for shape sweeps and edge-case tests."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    A = _base(tuple(shape), dist, g, device) * scale
    A = _apply_outliers(A, outliers, g)
    return A.to(dtype).contiguous()

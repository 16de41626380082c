"""Seeded synthetic inputs for the SmoothQuant W8A8 linear layer.

This module only draws random tensors with the shapes and value distributions
of the benchmark workloads; it contains none of the method's arithmetic (no
absmax, smoothing, quantisation or GEMM).  The same bytes are handed to the
CUDA library and to the CPU oracle.

Distributions (one seeded generator per tensor, seed derived from the workload
name, the tensor name and a base seed):
  * activations: N(0, 1); a fixed set of "outlier" input channels, chosen by a
    seeded permutation, is multiplied by a constant factor (x40 / x60 / x80);
    bf16 tensors are rounded to bf16 after the scaling;
  * the MLP down-projection input is SiLU(g) * u with g, u ~ N(0, 1) in fp32,
    then the outlier scaling, then bf16;
  * the same input before the gated activation, [gate | up] (2K values a
    row): g, u ~ N(0, 1) in fp32 with u's outlier channels scaled, then bf16;
  * weights: N(0, sigma) with sigma 0.02 (8B shapes, small case) or 0.015
    (70B shapes).
The outlier count is round(0.001 * K): 4 at K=4096, 8 at 8192, 14 at 14336 and
29 at 28672.  The small case uses the fixed channels {3, 77, 150, 201}.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List, Optional, Sequence, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Linear:
    """One linear layer of a workload: Y[M, N] = X[M, K] W[N, K]^T."""

    name: str
    N: int
    K: int
    act: str = "normal"  # "normal" or "silu_mul" (down-projection input)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    description: str
    linears: Tuple[Linear, ...]
    Ms: Tuple[int, ...]
    alpha: float
    calib_tokens: int
    w_sigma: float
    outlier_scale: float
    dtype: str  # "f32" or "bf16" for inputs
    out_dtype: str  # "f32" or "bf16"
    fixed_outliers: Optional[Tuple[int, ...]] = None
    fused_decode: bool = False


WORKLOADS: Dict[str, Workload] = {
    "small": Workload(
        "small",
        "single SmoothQuant W8A8 linear, fp32: Xcal 64x256 with channels {3,77,150,201} x40, "
        "W 256x256 N(0,0.02), alpha 0.5, X 16x256, fp32 out",
        (Linear("linear", 256, 256),),
        (16,),
        0.5,
        64,
        0.02,
        40.0,
        "f32",
        "f32",
        fixed_outliers=(3, 77, 150, 201),
    ),
    "llama3_8b_attn": Workload(
        "llama3_8b_attn",
        "Llama-3-8B attention projections: K=4096, fused QKV N=6144 and O N=4096, bf16, "
        "0.1% outlier channels x60, calibration 128x512 tokens, alpha 0.5, M 16/128/1024/4096",
        (Linear("qkv", 6144, 4096), Linear("o_proj", 4096, 4096)),
        (16, 128, 1024, 4096),
        0.5,
        128 * 512,
        0.02,
        60.0,
        "bf16",
        "bf16",
    ),
    "llama3_8b_mlp": Workload(
        "llama3_8b_mlp",
        "Llama-3-8B MLP: gate/up K=4096 N=28672, down K=14336 N=4096 (input SiLU(g)*u), "
        "outliers x60, alpha 0.8, calibration 128x512 tokens, M 1024/4096/8192",
        (Linear("gate_up", 28672, 4096), Linear("down", 4096, 14336, act="silu_mul")),
        (1024, 4096, 8192),
        0.8,
        128 * 512,
        0.02,
        60.0,
        "bf16",
        "bf16",
    ),
    "llama3_8b_decode": Workload(
        "llama3_8b_decode",
        "decode-shaped weight streaming: M 1/8/32 against the Llama-3-8B linears, int8 weights "
        "prepared off the clock, per-token quant fused into the GEMM, alpha 0.5",
        (
            Linear("qkv", 6144, 4096),
            Linear("o_proj", 4096, 4096),
            Linear("gate_up", 28672, 4096),
            Linear("down", 4096, 14336, act="silu_mul"),
        ),
        (1, 8, 32),
        0.5,
        128 * 512,
        0.02,
        60.0,
        "bf16",
        "bf16",
        fused_decode=True,
    ),
    "llama3_70b": Workload(
        "llama3_70b",
        "Llama-3-70B linears: K=8192 N=10240/8192/57344, K=28672 N=8192, W N(0,0.015), "
        "outliers x80, alpha 0.85, calibration 64x1024 tokens, M 2048/8192",
        (
            Linear("qkv", 10240, 8192),
            Linear("o_proj", 8192, 8192),
            Linear("gate_up", 57344, 8192),
            Linear("down", 8192, 28672, act="silu_mul"),
        ),
        (2048, 8192),
        0.85,
        64 * 1024,
        0.015,
        80.0,
        "bf16",
        "bf16",
    ),
}


def seed_for(workload: str, tensor: str, base_seed: int = 0) -> int:
    """Stable 63-bit seed from (workload, tensor, base seed)."""
    h = zlib.crc32(f"{workload}/{tensor}/{base_seed}".encode())
    return (h * 2654435761 + base_seed * 97 + 12345) & 0x7FFFFFFFFFFFFFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_channels(wl: Workload, K: int, base_seed: int = 0) -> List[int]:
    """The fixed outlier channel set of a workload at width K."""
    if wl.fixed_outliers is not None:
        return list(wl.fixed_outliers)
    count = int(round(0.001 * K))
    g = _gen("cpu", seed_for(wl.name, f"outliers/K{K}", base_seed))
    perm = torch.randperm(K, generator=g)
    return sorted(int(i) for i in perm[:count])


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def activations(
    wl: Workload,
    lin: Linear,
    rows: int,
    tensor: str,
    device="cpu",
    base_seed: int = 0,
    dtype: Optional[str] = None,
) -> torch.Tensor:
    """[rows, K] activations with the workload's outlier channels."""
    K = lin.K
    g = _gen(device, seed_for(wl.name, f"{tensor}/{lin.name}/{rows}", base_seed))
    if lin.act == "silu_mul":
        gate = torch.randn(rows, K, generator=g, device=device, dtype=torch.float32)
        up = torch.randn(rows, K, generator=g, device=device, dtype=torch.float32)
        x = torch.nn.functional.silu(gate) * up
        del gate, up
    else:
        x = torch.randn(rows, K, generator=g, device=device, dtype=torch.float32)
    idx = torch.tensor(outlier_channels(wl, K, base_seed), device=device, dtype=torch.long)
    x[:, idx] *= wl.outlier_scale
    return x.to(_torch_dtype(dtype or wl.dtype))


def gate_up(
    wl: Workload,
    lin: Linear,
    rows: int,
    tensor: str,
    device="cpu",
    base_seed: int = 0,
    dtype: Optional[str] = None,
) -> torch.Tensor:
    """[rows, 2K] = [gate | up], the feed-forward projections before the gated
    activation of the down projection (K = lin.K): N(0, 1) each, the up half
    scaled at the workload's outlier channels."""
    K = lin.K
    g = _gen(device, seed_for(wl.name, f"{tensor}/{lin.name}/gate_up/{rows}", base_seed))
    gu = torch.randn(rows, 2 * K, generator=g, device=device, dtype=torch.float32)
    idx = torch.tensor(outlier_channels(wl, K, base_seed), device=device, dtype=torch.long)
    gu[:, K + idx] *= wl.outlier_scale
    return gu.to(_torch_dtype(dtype or wl.dtype))


def calibration(wl: Workload, lin: Linear, device="cpu", base_seed: int = 0, tokens: Optional[int] = None):
    """Calibration activations [T, K] for one linear's input."""
    T = wl.calib_tokens if tokens is None else tokens
    return activations(wl, lin, T, "calib", device=device, base_seed=base_seed)


def inputs(wl: Workload, lin: Linear, M: int, device="cpu", base_seed: int = 0):
    """Inference activations [M, K], drawn independently of the calibration set."""
    return activations(wl, lin, M, "x", device=device, base_seed=base_seed)


def weight(wl: Workload, lin: Linear, device="cpu", base_seed: int = 0,
           rows: Optional[int] = None) -> torch.Tensor:
    """Weight [N, K] (out x in), N(0, sigma); `rows` draws a smaller [rows, K]
    sample with the same distribution (its own seed)."""
    tag = f"w/{lin.name}" if rows is None else f"w/{lin.name}/rows{rows}"
    g = _gen(device, seed_for(wl.name, tag, base_seed))
    n = lin.N if rows is None else rows
    w = torch.randn(n, lin.K, generator=g, device=device, dtype=torch.float32) * wl.w_sigma
    return w.to(_torch_dtype(wl.dtype))


def random_tensor(shape: Sequence[int], seed: int, dtype=torch.float32, device="cpu", scale: float = 1.0):
    """Generic seeded N(0, scale) tensor for edge-case tests."""
    g = _gen(device, seed)
    return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * scale).to(dtype)


def random_int8(shape: Sequence[int], seed: int, device="cpu", lo: int = -127, hi: int = 127):
    g = _gen(device, seed)
    return torch.randint(lo, hi + 1, tuple(shape), generator=g, device=device, dtype=torch.int8)

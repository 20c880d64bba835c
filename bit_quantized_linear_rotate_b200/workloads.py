"""Seeded synthetic inputs for the five workloads.

This module only draws random numbers; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it. Every tensor is drawn on the CPU with ``torch.Generator`` in a fixed
order (activations, outlier columns, weight bytes, weight scales, zeros), so
the bytes are identical wherever they are generated.

The shapes stand in for the pages' workloads: Z-Image activation shapes
[32 | 8192, 3840 | 10240] (comfy-kitchen PR #155, "Performance and memory"),
and the Qwen-Image-Edit modulation linear K=3072 -> N=6*3072
(``comfy_kitchen/tensor/awq_w4a16.py``, module docstring). No real
activations or checkpoints are used.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LinearWorkload:
    name: str
    M: int
    K: int
    N: int
    G: int
    seed: int
    outlier_cols: int          # number of activation columns multiplied by 20
    rq_group: int | None = None  # extra standalone rotate_quant group size


@dataclass(frozen=True)
class GemvW4A8Workload:
    name: str
    Ms: tuple
    K: int
    N: int
    seed: int


@dataclass(frozen=True)
class GemvAwqWorkload:
    name: str
    Ms: tuple
    K: int
    N: int
    G: int
    seed: int


# W4A4 linear, M=32, K=N=3840, G=64, 8 outlier channels x20, seed 0
LINEAR_M32 = LinearWorkload("w4a4_linear_M32_K3840_N3840_G64", 32, 3840, 3840, 64, 0, 8)
# W4A4 linear, M=8192, K=N=3840, G=64, seed 1
LINEAR_M8192 = LinearWorkload("w4a4_linear_M8192_K3840_N3840_G64", 8192, 3840, 3840, 64, 1, 8)
# W4A4 linear, MLP-down shape, 1% of 10240 columns x20, plus rotate_quant at G=16
LINEAR_MLP_DOWN = LinearWorkload("w4a4_linear_M8192_K10240_N3840_G256", 8192, 10240, 3840, 256, 2,
                                 10240 // 100, rq_group=16)
GEMV_W4A8 = GemvW4A8Workload("w4a8_gemv_K4096_N12288", (1, 4, 16), 4096, 12288, 3)
GEMV_AWQ = GemvAwqWorkload("awq_w4a16_gemv_K3072_N18432_G64", (1, 2, 4), 3072, 18432, 64, 4)

ALL = (LINEAR_M32, LINEAR_M8192, LINEAR_MLP_DOWN, GEMV_W4A8, GEMV_AWQ)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def activations(M: int, K: int, n_outlier_cols: int, g: torch.Generator,
                dtype=torch.bfloat16) -> torch.Tensor:
    """x ~ N(0, 1) with ``n_outlier_cols`` distinct columns multiplied by 20."""
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if n_outlier_cols:
        cols = torch.randperm(K, generator=g)[:n_outlier_cols]
        x[:, cols] *= 20.0
    return x.to(dtype)


def packed_weight_bytes(N: int, K: int, g: torch.Generator) -> torch.Tensor:
    """(N, K/2) bytes uniform over [0, 255]: independent uniform nibbles in [0, 15]."""
    return torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)


def uniform(shape, lo: float, hi: float, g: torch.Generator, dtype=torch.bfloat16) -> torch.Tensor:
    return (torch.rand(shape, generator=g, dtype=torch.float32) * (hi - lo) + lo).to(dtype)


def linear_inputs(w: LinearWorkload, dtype=torch.bfloat16) -> dict:
    """x (M, K), w_packed (N, K/2) u8, w_scale (N,) bf16 ~ U(0.005, 0.02)."""
    g = _gen(w.seed)
    x = activations(w.M, w.K, w.outlier_cols, g, dtype)
    wp = packed_weight_bytes(w.N, w.K, g)
    sw = uniform((w.N,), 0.005, 0.02, g)
    return {"x": x, "w_packed": wp, "w_scale": sw}


def gemv_w4a8_inputs(w: GemvW4A8Workload, M: int) -> dict:
    """x (M, K) bf16 ~ N(0, 1) (quantized rowwise by the caller), weights, scales."""
    g = _gen(w.seed * 1000 + M)
    x = activations(M, w.K, 0, g)
    wp = packed_weight_bytes(w.N, w.K, g)
    sw = uniform((w.N,), 0.005, 0.02, g)
    return {"x": x, "w_packed": wp, "w_scale": sw}


def gemv_awq_inputs(w: GemvAwqWorkload, M: int, dtype=torch.bfloat16) -> dict:
    """x (M, K), qweight (N, K/2), wscales ~ U(0.001, 0.01), wzeros ~ N(0, 0.01^2)."""
    g = _gen(w.seed * 1000 + M)
    x = activations(M, w.K, 0, g, dtype)
    qw = packed_weight_bytes(w.N, w.K, g)
    ws = uniform((w.K // w.G, w.N), 0.001, 0.01, g, dtype)
    wz = (torch.randn((w.K // w.G, w.N), generator=g, dtype=torch.float32) * 0.01).to(dtype)
    return {"x": x, "qweight": qw, "wscales": ws, "wzeros": wz}


def small_linear_inputs(M: int, K: int, N: int, seed: int, n_outlier_cols: int = 0,
                        dtype=torch.bfloat16, with_bias: bool = False) -> dict:
    """Same distributions at arbitrary (small) sizes, for parity and edge cases."""
    g = _gen(seed)
    x = activations(M, K, n_outlier_cols, g, dtype)
    wp = packed_weight_bytes(N, K, g)
    sw = uniform((N,), 0.005, 0.02, g)
    out = {"x": x, "w_packed": wp, "w_scale": sw}
    if with_bias:
        out["bias"] = uniform((N,), -1.0, 1.0, g)
    return out

"""Seeded synthetic weight matrices for the EntroPack decode workloads.

This module only draws random numbers and shapes them. It contains none of the
compression method, so the oracle tests and the GPU path can both take their
inputs from it. Every matrix comes from a CPU ``torch.Generator`` seeded as
stated, in float32 and row-major with shape (out_features, in_features). It is
cast to the container at the end.

The real weights that the pages measure on (the linear layers of the
Z-Image-Turbo diffusion transformer; EntroPack README, section 性能) are not
available. ``dit_layer_shapes()`` is a stand-in with the same layer count and
the same shapes.
"""
from __future__ import annotations

import math

import torch

CONTAINERS = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32,
              "fp8_e4m3": torch.float8_e4m3fn, "int8": torch.int8}
DTYPE_CODE = {"bf16": 1, "fp16": 2, "fp32": 3, "fp8_e4m3": 4, "int8": 5}


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed)


def quickstart_256(seed: int = 0) -> torch.Tensor:
    """256x256 BF16 with entries N(0, 0.02^2). This is the README quick-start tensor (section 快速开始)."""
    return (torch.randn(256, 256, generator=_gen(seed)) * 0.02).to(torch.bfloat16)


def lognormal_rows_with_outliers(n: int = 3072, seed: int = 1, sigma: float = 0.5,
                                 outlier_frac: float = 1e-4, outlier_mult: float = 8.0) -> torch.Tensor:
    """n x n BF16 matrix with lognormal row scales and sparse outliers.

    Draws happen in a fixed order:
    1. z ~ N(0,1)^n gives the row scales s = exp(ln 0.02 + sigma·z).
    2. The entries are s_row · N(0,1).
    3. round(outlier_frac·n²) positions are picked by randperm.
    4. Each picked position gets a random sign, times outlier_mult · s_row.
    """
    g = _gen(seed)
    z = torch.randn(n, generator=g)
    s = torch.exp(math.log(0.02) + sigma * z)
    w = s[:, None] * torch.randn(n, n, generator=g)
    k = int(round(outlier_frac * n * n))
    idx = torch.randperm(n * n, generator=g)[:k]
    sign = torch.randint(0, 2, (k,), generator=g).float() * 2 - 1
    flat = w.view(-1)
    flat[idx] = sign * outlier_mult * s[idx // n]
    return w.to(torch.bfloat16)


def dit_layer_shapes() -> list[tuple[str, int, int]]:
    """The 276 linear layers of the DiT-like set, in decode order.

    The set is 34 blocks, each of q, k, v, o (3840x3840), gate and up
    (10240x3840), down (3840x10240) and adaLN (15360x256). Four projections
    follow: 3840x64, 64x3840, 3840x2560 and 3840x3840. Shapes are
    (out_features, in_features).
    """
    shapes = []
    for blk in range(34):
        for nm in ("q", "k", "v", "o"):
            shapes.append((f"blocks.{blk}.attn.{nm}", 3840, 3840))
        shapes.append((f"blocks.{blk}.mlp.gate", 10240, 3840))
        shapes.append((f"blocks.{blk}.mlp.up", 10240, 3840))
        shapes.append((f"blocks.{blk}.mlp.down", 3840, 10240))
        shapes.append((f"blocks.{blk}.adaLN", 15360, 256))
    shapes += [("proj.a", 3840, 64), ("proj.b", 64, 3840), ("proj.c", 3840, 2560), ("proj.d", 3840, 3840)]
    assert len(shapes) == 276
    return shapes


def dit_layer(i: int, shape: tuple[int, int] | None = None, sigma: float = 0.3) -> torch.Tensor:
    """Layer i of the DiT-like set (seed i), in BF16.

    z ~ N(0,1)^M, then W = 0.02·exp(sigma·z)[:, None] · N(0,1)^(M x N).
    """
    if shape is None:
        _, M, N = dit_layer_shapes()[i]
    else:
        M, N = shape
    g = _gen(i)
    z = torch.randn(M, generator=g)
    w = (0.02 * torch.exp(sigma * z))[:, None] * torch.randn(M, N, generator=g)
    return w.to(torch.bfloat16)


def layer_sensitivity(n: int, seed: int = 20000, sigma: float = 1.0) -> list[float]:
    """A synthetic per-layer sensitivity: n draws of exp(sigma * z), z ~ N(0, 1), in layer order.

    The pages' mixed-bitrate packs rank layers by a sensitivity measured on the real model, which is
    not available; this stands in for it with a lognormal spread (sigma = 1: the middle two thirds of
    layers within a factor e of the median).
    """
    z = torch.randn(n, generator=_gen(seed), dtype=torch.float64)
    return [float(v) for v in torch.exp(sigma * z)]


def gaussian(M: int, N: int, seed: int, std: float = 0.02, container: str = "fp32") -> torch.Tensor:
    """M x N with entries N(0, std^2). Drawn in float32, then cast to the container."""
    w = torch.randn(M, N, generator=_gen(seed)) * std
    return w.to(CONTAINERS[container])


def fp8_codes(M: int = 8192, N: int = 28672, seed: int = 3) -> torch.Tensor:
    """FP8 e4m3 weight codes.

    Entries are N(0, 0.02^2). Each row is scaled so that its largest magnitude
    is 448. The result is cast to e4m3, clamped to ±448 first.
    """
    n = torch.randn(M, N, generator=_gen(seed)) * 0.02
    n = n * (448.0 / n.abs().amax(dim=1, keepdim=True))
    return n.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)


def int8_codes(M: int = 8192, N: int = 28672, seed: int = 4) -> torch.Tensor:
    """INT8 weight codes: round(clip(32·N(0,1), -127, 127))."""
    n = torch.randn(M, N, generator=_gen(seed)) * 32.0
    return torch.round(n.clamp(-127.0, 127.0)).to(torch.int8)


def container_bits(t: torch.Tensor) -> "numpy.ndarray":  # noqa: F821
    """Raw container bit patterns of t as a numpy array, for the byte-level C interfaces."""
    import numpy as np
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.contiguous().view(torch.uint8).numpy()
    return t.contiguous().numpy()


def dtype_code(t: torch.Tensor) -> int:
    for name, dt in CONTAINERS.items():
        if t.dtype == dt:
            return DTYPE_CODE[name]
    raise ValueError(f"unsupported container {t.dtype}")

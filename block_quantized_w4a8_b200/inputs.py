"""Seeded synthetic inputs for the W4A8 matmul workloads.

This module only draws random numbers; it holds none of the method's arithmetic, so the
oracle and the CUDA path can both take their inputs from it without sharing any code
that computes a result.

Recipe (every workload): ``torch.manual_seed(seed)``, then ``torch.randn`` on the CPU,
activations x (M x K) first and weights W (N x K) second, each scaled by its standard
deviation. Where a workload states bf16 activations, x is rounded to bf16 after drawing.

The shapes are those of the pages' workloads: the MiniLM intermediate projection
(64 x 384 x 1536, tract PR #2432 "Numbers"), the 4096 x 4096 decode GEMV of the same
page's follow-up, a 1024-token prefill at 4096 x 4096, the LLM MLP shapes of MLX PR #4802
"Performance" (K x N = 4096 x 14336, 14336 x 4096, 8192 x 2048) and its affine accuracy
setup (M = 1024, K = N = 4096, normal x and w).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    x_dtype: str = "f32"      # "f32" or "bf16"
    x_std: float = 1.0
    w_std: float = 0.02
    kind: str = "q4_0"        # "q4_0" or "affine"
    group: int = 0            # affine group size (64 or 128)
    seed: int = 0


MINILM = Workload("minilm_intermediate_64x384x1536", M=64, K=384, N=1536)
DECODE = Workload("decode_gemv_m1_4096x4096", M=1, K=4096, N=4096)
PREFILL = Workload("prefill_gemm_m1024_4096x4096", M=1024, K=4096, N=4096, x_dtype="bf16", w_std=1.0)
AFFINE_GS64 = Workload("affine_m1024_4096x4096_gs64", M=1024, K=4096, N=4096, x_dtype="bf16",
                       w_std=1.0, kind="affine", group=64)
AFFINE_GS128 = Workload("affine_m1024_4096x4096_gs128", M=1024, K=4096, N=4096, x_dtype="bf16",
                        w_std=1.0, kind="affine", group=128)

SWEEP_SHAPES = [(4096, 14336), (14336, 4096), (8192, 2048)]   # (K, N)
SWEEP_M = [1, 8, 16, 32, 64, 256, 1024, 4096]


def sweep_workloads() -> list[Workload]:
    out = []
    for K, N in SWEEP_SHAPES:
        for M in SWEEP_M:
            out.append(Workload(f"mlp_sweep_m{M}_k{K}_n{N}", M=M, K=K, N=N))
    return out


def make(wl: Workload, M: int | None = None, N: int | None = None, K: int | None = None):
    """Draw (x, W) for a workload, optionally at other sizes with the same distribution.

    Returns CPU tensors: x (M, K) float32 or bfloat16, W (N, K) float32.
    """
    M = wl.M if M is None else M
    N = wl.N if N is None else N
    K = wl.K if K is None else K
    g = torch.Generator().manual_seed(wl.seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32) * wl.x_std
    w = torch.randn(N, K, generator=g, dtype=torch.float32) * wl.w_std
    if wl.x_dtype == "bf16":
        x = x.to(torch.bfloat16)
    return x, w


def randn(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def sample_indices(M: int, N: int, count: int, seed: int = 1234):
    """Uniformly drawn output coordinates (m, n), always including the four corners."""
    g = torch.Generator().manual_seed(seed)
    ms = torch.randint(0, M, (count,), generator=g, dtype=torch.int32)
    ns = torch.randint(0, N, (count,), generator=g, dtype=torch.int32)
    corners_m = torch.tensor([0, 0, M - 1, M - 1], dtype=torch.int32)
    corners_n = torch.tensor([0, N - 1, 0, N - 1], dtype=torch.int32)
    return torch.cat([corners_m, ms]).numpy(), torch.cat([corners_n, ns]).numpy()


def make_q4_k(N: int, K: int, seed: int, d_scale: float = 2.0 ** -10) -> torch.Tensor:
    """Random Q4_K weights: N rows of K/256 super-blocks of 144 bytes (uint8, (N, K/256*144)).
    Every byte pattern of the 12 scale bytes and of the 128 code bytes is a valid block, so
    they are drawn uniformly; d and dmin are fp16 draws of U(0.5, 1) * d_scale and
    U(0, 1) * d_scale (bytes 0-1 and 2-3, little-endian)."""
    assert K % 256 == 0
    g = torch.Generator().manual_seed(seed)
    nb = K // 256
    blocks = torch.randint(0, 256, (N, nb, 144), generator=g, dtype=torch.int32).to(torch.uint8)
    d = ((torch.rand((N, nb), generator=g) * 0.5 + 0.5) * d_scale).to(torch.float16)
    dmin = (torch.rand((N, nb), generator=g) * d_scale).to(torch.float16)
    blocks[:, :, 0:2] = d.view(torch.uint8).reshape(N, nb, 2)
    blocks[:, :, 2:4] = dmin.view(torch.uint8).reshape(N, nb, 2)
    return blocks.reshape(N, nb * 144)

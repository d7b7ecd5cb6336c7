"""Seeded synthetic input tensors for the five block-scaled FP4 workloads.

This module only draws random numbers: it holds none of the quantisation
arithmetic, so both the CUDA library's tests/benchmark and the CPU oracle
can take their inputs from it.  Values are drawn in fp32 (fp64 where a
transform needs it), outliers are inserted in fp32, and a bf16 workload is
cast once with round-to-nearest-even.

Workloads (shapes along rows = blocks along the last dimension):
  tiny-f32      256 x 1024 fp32, N(0,1), every 512th flat element x20 (seed 0)
                -- the same outlier pattern as the block-size MAE experiment
                on the ultralytics FP4 glossary page ("Come funziona FP4").
  weight-4k     4096 x 4096 bf16, N(0, 0.02), 0.1 % of positions x50 (seed 1)
  act-8k-14k    8192 x 14336 bf16, Student-t (nu = 3) x 0.5 (seed 2)
  model-7b      32 layers x (4 x 4096x4096 + 3 x 4096x14336) bf16, N(0, 0.02),
                0.05 % of positions x30 per matrix (seed 3, per-matrix seeds)
  search-4k-14k 4096 x 14336 bf16, Laplace(0, 0.02) (seed 4)
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    rows: int
    cols: int
    dtype: torch.dtype
    seed: int
    kind: str          # "normal-outliers", "student-t", "laplace"
    std: float = 1.0
    out_frac: float = 0.0
    out_mult: float = 1.0
    every: int = 0      # every n-th flat element is an outlier (0 = random positions)
    description: str = ""

    @property
    def numel(self) -> int:
        return self.rows * self.cols


TINY_F32 = Workload("tiny-f32-256x1024", 256, 1024, torch.float32, 0, "normal-outliers",
                    std=1.0, out_mult=20.0, every=512,
                    description="fp32 256x1024 N(0,1), every 512th element x20, seed 0")
WEIGHT_4K = Workload("weight-4096x4096-bf16", 4096, 4096, torch.bfloat16, 1, "normal-outliers",
                     std=0.02, out_frac=0.001, out_mult=50.0,
                     description="bf16 4096x4096 N(0,0.02), 0.1% of positions x50, seed 1")
ACT_8K = Workload("act-8192x14336-bf16", 8192, 14336, torch.bfloat16, 2, "student-t",
                  std=0.5, description="bf16 8192x14336 Student-t(nu=3) x0.5, seed 2")
SEARCH_4K = Workload("search-4096x14336-bf16", 4096, 14336, torch.bfloat16, 4, "laplace",
                     std=0.02, description="bf16 4096x14336 Laplace(0,0.02), seed 4")

# The other block layouts: a weight grouped along its columns (Q(W^T) of a
# 4096x14336 matrix, the down-projection shape of the weight set) and an
# activation whose rows are one element short of whole blocks (14335 =
# 895 x 16 + 15: every row ends in a 15-element block padded with +0).
COLUMNS_4K = Workload("columns-4096x14336-bf16", 4096, 14336, torch.bfloat16, 5, "normal-outliers",
                      std=0.02, out_frac=0.001, out_mult=50.0,
                      description="bf16 4096x14336 N(0,0.02), 0.1% x50, seed 5; blocks down the columns")
RAGGED_8K = Workload("ragged-8192x14335-bf16", 8192, 14335, torch.bfloat16, 6, "student-t",
                     std=0.5, description="bf16 8192x14335 Student-t(nu=3) x0.5, seed 6; rows padded to "
                                          "whole blocks")

# The scale-rule variants on the activation distribution (Student-t rows of
# 14336 elements, a fresh seed).
VARIANTS_8K = Workload("variants-8192x14336-bf16", 8192, 14336, torch.bfloat16, 7, "student-t",
                       std=0.5, description="bf16 8192x14336 Student-t(nu=3) x0.5, seed 7; MXFP4 ceil rule "
                                            "and NVFP4 four over six")

# The consumer: an activation of 8192 tokens x 14336 features (as the
# activation workload) times the 4096 x 14336 down-projection weight of the
# weight set, both NVFP4 along K = 14336.
GEMM_ACT = Workload("gemm-8192x4096x14336-nvfp4", 8192, 14336, torch.bfloat16, 8, "student-t",
                    std=0.5, description="D [8192, 4096] = A [8192, 14336] x W^T, W [4096, 14336]: A bf16 "
                                         "Student-t(nu=3) x0.5 seed 8 quantised each step, W N(0,0.02) 0.05% x30 "
                                         "seed 9 quantised once")
GEMM_W = Workload("gemm-weight-4096x14336", 4096, 14336, torch.bfloat16, 9, "normal-outliers",
                  std=0.02, out_frac=0.0005, out_mult=30.0)

# The 7B-class weight set: per layer 4 square 4096x4096 and 3 4096x14336.
MODEL_LAYERS = 32
MODEL_MATRICES = [(4096, 4096)] * 4 + [(4096, 14336)] * 3


def model_matrix(layer: int, idx: int) -> Workload:
    r, c = MODEL_MATRICES[idx]
    seed = 3 * 1_000_003 + layer * 101 + idx  # distinct, reproducible per matrix
    return Workload(f"model-7b-L{layer}-M{idx}", r, c, torch.bfloat16, seed, "normal-outliers",
                    std=0.02, out_frac=0.0005, out_mult=30.0,
                    description=f"bf16 {r}x{c} N(0,0.02), 0.05% x30, layer {layer} matrix {idx}")


def model_numel() -> int:
    return MODEL_LAYERS * sum(r * c for r, c in MODEL_MATRICES)


# The whole weight set as one workload (processed with grouped calls, each
# matrix drawn from its own model_matrix seed): rows x cols is only the
# element count, 7,784,628,224 = 1,900,544 x 4096; the real shapes are
# MODEL_MATRICES per layer.
MODEL_WEIGHTS = Workload("model-7b-weights-bf16", model_numel() // 4096, 4096, torch.bfloat16, 3,
                         "normal-outliers", std=0.02, out_frac=0.0005, out_mult=30.0,
                         description="7B-class weight set: 32 layers x (4 x 4096x4096 + 3 x 4096x14336) "
                                     "bf16, N(0,0.02), 0.05% x30 per matrix, seed 3 (per-matrix seeds)")


def with_shape(w: Workload, rows: int, cols: int, seed_offset: int = 0) -> Workload:
    """Same distribution at another size (small parity cases, shards)."""
    return dataclasses.replace(w, rows=rows, cols=cols, seed=w.seed + seed_offset,
                               name=f"{w.name}@{rows}x{cols}" + (f"+{seed_offset}" if seed_offset else ""))


def for_rank(w: Workload, rank: int) -> Workload:
    """The tensor rank `rank` works on when N ranks each take their own
    tensor of the workload (independent problems, no data exchange): same
    shape and distribution, seed offset by 1000 per rank (rank 0 keeps the
    workload's own seed)."""
    return w if rank == 0 else with_shape(w, w.rows, w.cols, seed_offset=1000 * rank)


def generate(w: Workload, device: str | torch.device = "cpu") -> torch.Tensor:
    """The workload's tensor, [rows, cols] in its dtype, drawn from a
    torch.Generator seeded with w.seed on `device`."""
    n = w.numel
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    if w.kind == "normal-outliers":
        x = torch.randn(n, generator=gen, device=device, dtype=torch.float32) * w.std
        if w.every:
            x[:: w.every] *= w.out_mult
        elif w.out_frac > 0:
            k = int(round(w.out_frac * n))
            pos = torch.randperm(n, generator=gen, device=device)[:k]
            x[pos] *= w.out_mult
    elif w.kind == "student-t":
        # t_3 = z / sqrt(chi2_3 / 3), chi2_3 = sum of three squared normals.
        z = torch.randn(n, generator=gen, device=device, dtype=torch.float32)
        chi = torch.zeros(n, device=device, dtype=torch.float32)
        for _ in range(3):
            chi += torch.randn(n, generator=gen, device=device, dtype=torch.float32) ** 2
        x = z / torch.sqrt(chi / 3.0) * w.std
    elif w.kind == "laplace":
        # inverse CDF: x = -b sign(u - 1/2) log(1 - 2|u - 1/2|), u in (0, 1).
        u = torch.rand(n, generator=gen, device=device, dtype=torch.float64) - 0.5
        a = u.abs().clamp(max=0.5 - 2.0 ** -40)
        x = (-w.std * torch.sign(u) * torch.log1p(-2.0 * a)).to(torch.float32)
    else:
        raise ValueError(w.kind)
    return x.reshape(w.rows, w.cols).to(w.dtype)


def page_mae_input() -> torch.Tensor:
    """fp32 randn(4096) from seed 0 with every 512th element x20: the input of
    the block-size MAE experiment on the ultralytics FP4 glossary page."""
    return generate(Workload("mae-4096", 1, 4096, torch.float32, 0, "normal-outliers",
                             std=1.0, out_mult=20.0, every=512)).reshape(-1)


def as_oracle_array(x: torch.Tensor):
    """numpy view for the oracle: float32 as is, bf16 as uint16 bit patterns."""
    import numpy as np
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.float32:
        return x.numpy()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16)
    raise TypeError(x.dtype)


def sample_rows(rows: int, k: int, seed: int = 12345) -> list[int]:
    """k distinct row indices including the first and last row."""
    if k >= rows:
        return list(range(rows))
    gen = torch.Generator().manual_seed(seed)
    mid = torch.randperm(rows - 2, generator=gen)[: max(k - 2, 0)] + 1
    return sorted({0, rows - 1, *mid.tolist()})


ALL = {w.name: w for w in (TINY_F32, WEIGHT_4K, ACT_8K, SEARCH_4K)}

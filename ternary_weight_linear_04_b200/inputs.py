"""Seeded synthetic inputs for the BitLinear workloads.

This module holds no arithmetic of the method itself: it only draws latent
weights and activations, so that the CUDA path and the CPU oracle can be fed
the very same bytes.  Recipe (identical for every consumer):

* ``rng = np.random.default_rng(np.random.SeedSequence([seed, index]))`` per
  matrix, ``index`` its position in the workload's matrix list;
* latent weights W (N x K, row-major: out_features x in_features) are drawn
  first, in fp64, and rounded to fp32 (NumPy's cast, round to nearest);
* then activations x (M_max x K) are drawn from the same generator in fp64,
  rounded to fp32 and, for bf16 workloads, to bf16 (torch's round to nearest
  even); a smaller batch M takes the first M rows.

Distributions follow the layer shapes the pages discuss (3B/7B/70B-class
decoder projections): W ~ N(0, 0.02^2) or Laplace(0, 0.02); x ~ N(0, 1) or
Student-t(3) with 1% of channels scaled by 50 (an outlier stress case).
"""
import math
from dataclasses import dataclass
from typing import Tuple

import numpy as np


@dataclass(frozen=True)
class Matrix:
    name: str
    K: int  # in_features
    N: int  # out_features


@dataclass(frozen=True)
class Workload:
    key: str
    seed: int
    matrices: Tuple[Matrix, ...]
    batches: Tuple[int, ...]
    act_dtype: str          # "f32" or "bf16"
    out_dtype: str          # "f32" or "bf16"
    w_dist: str = "normal"  # "normal" | "laplace"
    x_dist: str = "normal"  # "normal" | "student_t_outliers"
    description: str = ""


WORKLOADS = {
    "single_256": Workload(
        "single_256", 0, (Matrix("W", 256, 256),), (1,), "f32", "f32",
        description="single BitLinear, M=1, K=256, N=256, fp32 in/out"),
    "decode_3b": Workload(
        "decode_3b", 1, (Matrix("up_3200x8640", 3200, 8640), Matrix("down_8640x3200", 8640, 3200)),
        (1, 4, 16), "bf16", "bf16",
        description="3B-class decode GEMV: K=3200->N=8640 and K=8640->N=3200, M in {1,4,16}"),
    "prefill_7b": Workload(
        "prefill_7b", 2, (Matrix("ffn_4096x11008", 4096, 11008),), (2048,), "bf16", "bf16",
        description="7B-class prefill GEMM: M=2048, K=4096, N=11008"),
    "layer_70b": Workload(
        "layer_70b", 3,
        (Matrix("Wq", 8192, 8192), Matrix("Wk", 8192, 1024), Matrix("Wv", 8192, 1024),
         Matrix("Wo", 8192, 8192), Matrix("gate", 8192, 28672), Matrix("up", 8192, 28672),
         Matrix("down", 28672, 8192)),
        (1, 32), "bf16", "bf16",
        description="one 70B-class decoder layer's 7 projections, M in {1,32}"),
    "outlier_sweep": Workload(
        "outlier_sweep", 4, (Matrix("ffn_8192x28672", 8192, 28672),), (1, 8, 64, 256, 2048),
        "bf16", "bf16", w_dist="laplace", x_dist="student_t_outliers",
        description="8192x28672, Laplace weights, Student-t(3) activations with 1% x50 "
                    "outlier channels, M in {1,8,64,256,2048}"),
}


def _rng(seed, index):
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(index)]))


def draw_weights(rng, N, K, dist="normal"):
    if dist == "normal":
        w = rng.normal(0.0, 0.02, size=(N, K))
    elif dist == "laplace":
        w = rng.laplace(0.0, 0.02, size=(N, K))
    else:
        raise ValueError(dist)
    return w.astype(np.float32)


def draw_activations(rng, M, K, dist="normal", dtype="bf16"):
    """Returns fp32 values (bf16-representable when dtype == 'bf16')."""
    if dist == "normal":
        x = rng.normal(0.0, 1.0, size=(M, K))
    elif dist == "student_t_outliers":
        x = rng.standard_t(3.0, size=(M, K))
        cols = rng.choice(K, size=int(math.ceil(0.01 * K)), replace=False)
        x[:, cols] *= 50.0
    else:
        raise ValueError(dist)
    x = x.astype(np.float32)
    if dtype == "bf16":
        x = to_bf16_values(x)
    return x


def to_bf16_values(x32):
    """Round fp32 values to bf16 (torch, nearest-even) and widen back."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).to(torch.float32).numpy()


def make_matrix_inputs(workload: Workload, index: int, m_max=None):
    """(W fp32 N x K, x fp32 M_max x K) for matrix ``index`` of a workload."""
    mat = workload.matrices[index]
    rng = _rng(workload.seed, index)
    W = draw_weights(rng, mat.N, mat.K, workload.w_dist)
    M = max(workload.batches) if m_max is None else m_max
    x = draw_activations(rng, M, mat.K, workload.x_dist, workload.act_dtype)
    return W, x


def make_case(seed, M, K, N, w_dist="normal", x_dist="normal", act_dtype="f32"):
    """A free-form seeded case (for tests at sizes of their own choosing)."""
    rng = _rng(seed, 0)
    W = draw_weights(rng, N, K, w_dist)
    x = draw_activations(rng, M, K, x_dist, act_dtype)
    return W, x

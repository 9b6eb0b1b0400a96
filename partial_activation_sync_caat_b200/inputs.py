"""Seeded synthetic input generators shared by the tests, the bench and the smoke check.

This module holds no arithmetic of the method: it only draws random tensors with the
shapes and distributions of the workloads, and random sync-index lists.  Both the CUDA
path and the float64 oracle are fed from here; neither of them is imported here.

Layouts (row-major, last dimension contiguous), bf16 stored as torch.bfloat16:

* row-parallel layer: X [P, T, K/P], W [P, H, K/P] (nn.Linear orientation, K contiguous),
  residual [P, T, H], gamma [H];
* MLP block: X [P, T, H], A [P, 2F/P, H] (gate rows first, then up rows),
  W2 [P, H, F/P], residual [P, T, H], gamma [H].
"""
from __future__ import annotations

import numpy as np
import torch


def _normal(shape, std, gen, device):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    if std == 0.0:
        return t.zero_().to(torch.bfloat16)
    t.normal_(0.0, std, generator=gen)
    return t.to(torch.bfloat16)


def _generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_rowpar_inputs(T: int, K: int, H: int, P: int, seed: int = 0, *,
                       x_std: float = 1.0, w_std: float = 0.02, r_std: float = 1.0,
                       gamma: str = "ones", device: str = "cpu") -> dict:
    """Inputs of the partially synchronized row-parallel layer.

    gamma: "ones" (gamma = 1) or "uniform" (U(0.5, 1.5), seeded).  r_std = 0 gives a zero
    residual, which makes the output depend on the GEMM alone.
    """
    if K % P:
        raise ValueError("K must be divisible by P")
    Kp = K // P
    g = _generator(seed, device)
    X = _normal((P, T, Kp), x_std, g, device)
    W = _normal((P, H, Kp), w_std, g, device)
    R = _normal((P, T, H), r_std, g, device)
    if gamma == "ones":
        gm = torch.ones(H, dtype=torch.bfloat16, device=device)
    elif gamma == "uniform":
        gm = (torch.rand(H, generator=g, device=device) + 0.5).to(torch.bfloat16)
    else:
        raise ValueError(gamma)
    return {"X": X, "W": W, "R": R, "gamma": gm}


def make_mlp_inputs(T: int, H: int, F: int, P: int, seed: int = 0, *,
                    x_std: float = 1.0, w_std: float = 0.02, r_std: float = 1.0,
                    gamma: str = "ones", device: str = "cpu") -> dict:
    """Inputs of the MLP block: per-rank X, column-parallel A (gate rows, then up rows),
    row-parallel W2, per-rank residual, shared gamma."""
    if F % P:
        raise ValueError("F must be divisible by P")
    Fp = F // P
    g = _generator(seed, device)
    X = _normal((P, T, H), x_std, g, device)
    A = _normal((P, 2 * Fp, H), w_std, g, device)
    W2 = _normal((P, H, Fp), w_std, g, device)
    R = _normal((P, T, H), r_std, g, device)
    if gamma == "ones":
        gm = torch.ones(H, dtype=torch.bfloat16, device=device)
    elif gamma == "uniform":
        gm = (torch.rand(H, generator=g, device=device) + 0.5).to(torch.bfloat16)
    else:
        raise ValueError(gamma)
    return {"X": X, "A": A, "W2": W2, "R": R, "gamma": gm}


def random_sync_idx(H: int, n_sync: int, seed: int = 0) -> np.ndarray:
    """A seeded random sync-index list: n_sync distinct channels of [0, H), sorted, int32."""
    rng = np.random.default_rng(seed)
    idx = rng.choice(H, size=n_sync, replace=False)
    return np.sort(idx).astype(np.int32)


def sample_rows(T: int, n: int, seed: int = 0) -> np.ndarray:
    """n distinct token rows of [0, T), sorted (for sampled parity checks at full size)."""
    rng = np.random.default_rng(seed + 7919)
    n = min(n, T)
    return np.sort(rng.choice(T, size=n, replace=False)).astype(np.int64)

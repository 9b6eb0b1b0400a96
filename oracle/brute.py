"""Pure-Python brute force of the partially synchronized layer, for tiny shapes only.

TEST INFRASTRUCTURE ONLY.  It checks the NumPy oracle in caat_oracle.py by writing every
sum of "Tensor-Parallelism with Partially Synchronized Activations", App. A.2 Eq. 22 as
explicit loops over (rank m, token i, channel l, contraction index k), in Python floats
(IEEE double), with no NumPy matmul, masking or broadcasting.
"""
from __future__ import annotations

import math


def _tolist(a):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).tolist()
    except ImportError:  # pragma: no cover
        pass
    return [[[float(v) for v in row] for row in mat] for mat in a] if hasattr(a, "__len__") else a


def brute_rowpar(X, W, R, gamma, P, p, sync_idx=None, eps=1e-5, private_scale=1.0):
    """Returns (Z, h, out) as nested lists [P][T][H]."""
    X = _tolist(X)
    W = _tolist(W)
    R = _tolist(R)
    g = gamma.detach().to("cpu").double().tolist() if hasattr(gamma, "detach") else list(gamma)
    T = len(X[0])
    Kp = len(X[0][0])
    H = len(W[0])
    ns = math.floor(H * p)
    if sync_idx is None:
        shared = set(range(ns))
    else:
        shared = set(int(v) for v in sync_idx)
    # Z~_{i l m} = sum_k X_{i k m} B~_{k l m}
    Zt = [[[0.0] * H for _ in range(T)] for _ in range(P)]
    for m in range(P):
        for i in range(T):
            for l in range(H):
                acc = 0.0
                for k in range(Kp):
                    acc += X[m][i][k] * W[m][l][k]
                Zt[m][i][l] = acc
    Z = [[[0.0] * H for _ in range(T)] for _ in range(P)]
    for m in range(P):
        for i in range(T):
            for l in range(H):
                if l in shared:
                    s = 0.0
                    for q in range(P):
                        s += Zt[q][i][l]
                    Z[m][i][l] = s
                else:
                    Z[m][i][l] = private_scale * Zt[m][i][l]
    h = [[[Z[m][i][l] + R[m][i][l] for l in range(H)] for i in range(T)] for m in range(P)]
    out = [[[0.0] * H for _ in range(T)] for _ in range(P)]
    for m in range(P):
        for i in range(T):
            ss = 0.0
            for l in range(H):
                ss += h[m][i][l] * h[m][i][l]
            inv = 1.0 / math.sqrt(ss / H + eps)
            for l in range(H):
                out[m][i][l] = h[m][i][l] * inv * g[l]
    return Z, h, out


def brute_swiglu(X, A):
    """Y[m][i][j] = silu(sum_k X[m][i][k] A[m][j][k]) * sum_k X[m][i][k] A[m][F/P + j][k]."""
    X = _tolist(X)
    A = _tolist(A)
    P = len(X)
    T = len(X[0])
    Hd = len(X[0][0])
    Fp = len(A[0]) // 2
    Y = [[[0.0] * Fp for _ in range(T)] for _ in range(P)]
    for m in range(P):
        for i in range(T):
            for j in range(Fp):
                gsum = 0.0
                usum = 0.0
                for k in range(Hd):
                    gsum += X[m][i][k] * A[m][j][k]
                    usum += X[m][i][k] * A[m][Fp + j][k]
                Y[m][i][j] = gsum / (1.0 + math.exp(-gsum)) * usum
    return Y

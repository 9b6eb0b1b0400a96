"""Float64 CPU oracle for the partially synchronized row-parallel layer of CAAT-Net.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU-baseline
leg may import this module.  It shares no code with the CUDA path and imports nothing
from the product package.

Source: "Tensor-Parallelism with Partially Synchronized Activations" (Lamprecht,
Karnieli, Hanani, Giladi, Soudry; arXiv 2506.19645):

* partial products of the row-parallel layer: §3.1 Eq. 4-5 and App. A.2 Eq. 21-22
  (Z~_{ilm} = sum_k Y_{ikm} B~_{klm});
* partial channel-reduce: App. A.2 Eq. 22 (channels l < floor(h p) are summed over the
  tensor-parallel ranks m, the others keep the rank's own value), §3 (the shared channels
  are the first h p channels), §3.1 Eq. 8 (the two-rank case);
* private-channel scaling: §4 "Private channel scaling", Eq. 14-15 (private channels are
  multiplied by sqrt(r) so that their variance matches the shared ones);
* residual add and norm: §4 Eq. 9 and App. B Eq. 25 (X_m = Norm(sum Z + R)); the norm is
  RMSNorm here, with gamma shared by the ranks (§4: norm parameters are synchronized);
* MLP block: §3.1 Eq. 6 (Y_m = sigma(X_m A_m), column-parallel A) with sigma = SwiGLU;
* speed-up model: App. C Eq. 31-35 (compute and exchange per layer, T(p), speed-up, p*);
* backward: §4 Eq. 10-13 (the reduction over ranks follows the norm derivative; the shared
  norm weight's gradient is summed over the ranks), chain rule through Eq. 22 and Eq. 9.

Everything is plain NumPy float64: one library matmul per partial product, no blocking,
fusion or reordering beyond the definitions above.  The inputs are the bf16 tensors
upcast exactly to float64.

Readings where the pages leave a step open (each also listed in the design notes):
* n_s = floor(H p) is evaluated in float64 (App. A.2 Eq. 22 writes floor(hp)).
* S is the first n_s channels unless an explicit sorted, unique index list of length n_s
  is given (the pages only describe the contiguous choice, §3).
* private_scale multiplies the private channels before the residual add (§4 Eq. 14-15);
  default 1.0, sqrt(P) is the paper's variant.
* RMSNorm: out = h / sqrt(mean(h^2) + eps) * gamma over all H channels of the rank,
  eps inside the square root (the pages name RMSNorm but give no epsilon).
* SwiGLU: Y = silu(X A_gate^T) * (X A_up^T), silu(x) = x / (1 + exp(-x)); A_m holds the
  F/P gate rows first, then the F/P up rows (the pages keep sigma generic).
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    """Upcast a torch tensor (any float dtype) or array to a float64 NumPy array."""
    try:
        import torch  # local import: the oracle itself needs only NumPy
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def n_sync(H: int, p: float) -> int:
    """Number of shared channels, floor(h p) (App. A.2, Eq. 22)."""
    if not (0.0 <= p <= 1.0):
        raise ValueError("p must lie in [0, 1]")
    return int(np.floor(np.float64(H) * np.float64(p)))


def sync_mask(H: int, p: float, sync_idx=None) -> np.ndarray:
    """Boolean mask of the shared channels S (App. A.2 Eq. 22; §3 "first h p channels").

    With sync_idx given it must be a sorted list of n_s distinct channels in [0, H).
    """
    ns = n_sync(H, p)
    mask = np.zeros(H, dtype=bool)
    if sync_idx is None:
        mask[:ns] = True
        return mask
    idx = np.asarray(sync_idx, dtype=np.int64).reshape(-1)
    if idx.size != ns:
        raise ValueError(f"sync_idx has {idx.size} entries, floor(H*p) = {ns}")
    if idx.size and (idx.min() < 0 or idx.max() >= H):
        raise ValueError("sync_idx out of range")
    if idx.size > 1 and np.any(np.diff(idx) <= 0):
        raise ValueError("sync_idx must be strictly increasing")
    mask[idx] = True
    return mask


def partial_products(X, W) -> np.ndarray:
    """Per-rank partial products Z~_m = X_m W_m^T (App. A.2 Eq. 22, first line).

    X [P, T, K/P], W [P, H, K/P] (W_m is B~_m transposed) -> [P, T, H] float64.
    """
    X = _f64(X)
    W = _f64(W)
    return np.stack([X[m] @ W[m].T for m in range(X.shape[0])])


def partial_channel_reduce(Zt: np.ndarray, mask: np.ndarray, private_scale: float = 1.0) -> np.ndarray:
    """Eq. 22 second line: shared channels get the sum over ranks, private channels keep
    the rank's own partial (times the §4 private-channel scale)."""
    Z = Zt * np.float64(private_scale)
    Z[:, :, mask] = Zt[:, :, mask].sum(axis=0)[None, :, :]
    return Z


def rmsnorm(h: np.ndarray, gamma, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: h / sqrt(mean(h^2) + eps) * gamma."""
    gamma = _f64(gamma)
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + np.float64(eps)) * gamma


def rowpar_forward(X, W, R, gamma, P: int, p: float, sync_idx=None, *, eps: float = 1e-5,
                   private_scale: float = 1.0, return_all: bool = False):
    """The partially synchronized row-parallel layer, residual add and per-rank RMSNorm.

    X [P,T,K/P], W [P,H,K/P], R [P,T,H], gamma [H] -> out [P,T,H] (float64).
    With return_all, returns a dict with the intermediates Zt (partials), Z (after the
    partial channel-reduce), h (pre-norm residual stream), out and mask.
    """
    X = _f64(X)
    W = _f64(W)
    R = _f64(R)
    if X.shape[0] != P or W.shape[0] != P or R.shape[0] != P:
        raise ValueError("leading dimension must be P")
    H = W.shape[1]
    mask = sync_mask(H, p, sync_idx)
    Zt = partial_products(X, W)
    Z = partial_channel_reduce(Zt, mask, private_scale)
    h = Z + R
    out = rmsnorm(h, gamma, eps)
    if return_all:
        return {"Zt": Zt, "Z": Z, "h": h, "out": out, "mask": mask}
    return out


def rmsnorm_backward(h: np.ndarray, gamma, dout: np.ndarray, eps: float):
    """Backward of out = h / sqrt(mean(h^2) + eps) * gamma over the last axis, per row:
    with r = 1 / sqrt(mean(h^2) + eps), xhat = h r and g = dout * gamma,
    dh = r (g - xhat mean(g xhat)) and dgamma_row = dout * xhat.  Returns (dh, dout * xhat)."""
    gamma = _f64(gamma)
    r = 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + np.float64(eps))
    xhat = h * r
    g = dout * gamma
    dh = r * (g - xhat * np.mean(g * xhat, axis=-1, keepdims=True))
    return dh, dout * xhat


def partial_channel_reduce_backward(dZ: np.ndarray, mask: np.ndarray, private_scale: float = 1.0) -> np.ndarray:
    """Transpose of partial_channel_reduce: a shared channel of every rank's partial receives
    the sum over ranks of dZ (the reduction after the norm derivative, §4 Eq. 10-11: the 'h'
    operation of Fig. 2b), a private channel private_scale times its own rank's dZ."""
    dZt = dZ * np.float64(private_scale)
    dZt[:, :, mask] = dZ[:, :, mask].sum(axis=0)[None, :, :]
    return dZt


def rowpar_backward(X, W, h, gamma, dout, P: int, p: float, sync_idx=None, *, eps: float = 1e-5,
                    private_scale: float = 1.0):
    """Gradients of rowpar_forward given dL/d(out) [P,T,H] and the pre-norm stream h the
    forward produced (h = Z + R).  The chain rule, step by step:
      RMSNorm per rank (§4 Eq. 9)         -> dh, and dgamma summed over ranks and tokens
                                             (gamma is shared: its gradient is reduced over
                                             the ranks, §4 Eq. 12-13)
      residual add h = Z + R              -> dR = dZ = dh
      partial channel-reduce (Eq. 22)     -> dZt (shared: sum over ranks; private: scale x own)
      partial products Zt_m = X_m W_m^T   -> dX_m = dZt_m W_m, dW_m = dZt_m^T X_m
    Returns a dict with dX [P,T,K/P], dW [P,H,K/P], dR [P,T,H], dgamma [H] and dZt."""
    X = _f64(X)
    W = _f64(W)
    h = _f64(h)
    dout = _f64(dout)
    if X.shape[0] != P or W.shape[0] != P or h.shape[0] != P:
        raise ValueError("leading dimension must be P")
    mask = sync_mask(W.shape[1], p, sync_idx)
    dh, dg_rows = rmsnorm_backward(h, gamma, dout, eps)
    dZt = partial_channel_reduce_backward(dh, mask, private_scale)
    dX = np.stack([dZt[m] @ W[m] for m in range(P)])
    dW = np.stack([dZt[m].T @ X[m] for m in range(P)])
    return {"dX": dX, "dW": dW, "dR": dh, "dgamma": dg_rows.sum(axis=(0, 1)), "dZt": dZt}


def silu(x: np.ndarray) -> np.ndarray:
    """silu(x) = x * sigmoid(x) = x / (1 + exp(-x))."""
    return x / (1.0 + np.exp(-x))


def swiglu_fc1(X, A) -> np.ndarray:
    """Column-parallel FC1 with SwiGLU per rank (§3.1 Eq. 6 with sigma = SwiGLU).

    X [P,T,H], A [P, 2F/P, H] (gate rows then up rows) -> Y [P, T, F/P] float64.
    """
    X = _f64(X)
    A = _f64(A)
    Fp = A.shape[1] // 2
    out = []
    for m in range(X.shape[0]):
        g = X[m] @ A[m, :Fp].T
        u = X[m] @ A[m, Fp:].T
        out.append(silu(g) * u)
    return np.stack(out)


def mlp_forward(X, A, W2, R, gamma, P: int, p: float, sync_idx=None, *, eps: float = 1e-5,
                private_scale: float = 1.0, return_all: bool = False):
    """MLP block: FC1 + SwiGLU (Eq. 6), then the partially synced FC2 (Eq. 22), residual
    add and RMSNorm (Eq. 9).  Y stays in float64 (no bf16 rounding)."""
    Y = swiglu_fc1(X, A)
    res = rowpar_forward(Y, W2, R, gamma, P, p, sync_idx, eps=eps,
                         private_scale=private_scale, return_all=True)
    if return_all:
        res["Y"] = Y
        return res
    return res["out"]


def _take_rows(a, rows: np.ndarray) -> np.ndarray:
    """a[:, rows, :] as float64, indexing before the upcast (full-size tensors stay bf16)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return _f64(a[:, torch.as_tensor(rows, device=a.device), :])
    except ImportError:  # pragma: no cover
        pass
    return _f64(np.asarray(a)[:, rows, :])


def rowpar_rows(X, W, R, gamma, P: int, p: float, rows, sync_idx=None, *, eps: float = 1e-5,
                private_scale: float = 1.0, return_all: bool = False):
    """The layer evaluated on a subset of token rows only (rows are independent through the
    whole path, so this is exact for those rows).  Used for sampled checks at full size."""
    rows = np.asarray(rows, dtype=np.int64)
    return rowpar_forward(_take_rows(X, rows), W, _take_rows(R, rows), gamma, P, p, sync_idx,
                          eps=eps, private_scale=private_scale, return_all=return_all)


def mlp_rows(X, A, W2, R, gamma, P: int, p: float, rows, sync_idx=None, *, eps: float = 1e-5,
             private_scale: float = 1.0, return_all: bool = False):
    """The MLP block on a subset of token rows (rows are independent)."""
    rows = np.asarray(rows, dtype=np.int64)
    return mlp_forward(_take_rows(X, rows), A, W2, _take_rows(R, rows), gamma, P, p, sync_idx,
                       eps=eps, private_scale=private_scale, return_all=return_all)


def layer_compute_ops(h: float, s: float, r: float) -> float:
    """Per-device GEMM operations of one transformer layer's forward (App. C, Eq. 31-32):
    MLP (h -> 4h, 4h -> h) 16 s h^2, attention (qkv, scores and values, out) 4 s^2 h + 8 s h^2,
    a product of m x p by p x n counted as 2 m p n; split over r tensor-parallel devices."""
    mlp = 8 * s * h * h + 8 * s * h * h
    attention = 6 * s * h * h + 4 * s * s * h + 2 * s * h * h
    return (mlp + attention) / r


def layer_exchange(h: float, s: float, p: float) -> float:
    """Activations each device sends and receives per layer (App. C, Eq. 32): two all-reduces
    of s h activations, of which the partial all-reduce keeps the fraction p."""
    return 2 * s * h * p


def speedup_model(h: float, s: float, r: float, p: float, C: float):
    """App. C Eq. 33-35 from the definitions: T(p) = G + C P(p) with C the ratio of compute
    to communication capacity (FLOP per exchanged activation), speed-up (T(1) - T(p)) / T(1),
    and p* = the p at which C P(p) = G, capped at 1.  Returns (speedup, p_star)."""
    G = layer_compute_ops(h, s, r)
    T = lambda q: G + C * layer_exchange(h, s, q)  # noqa: E731
    p_star = min(G / (C * layer_exchange(h, s, 1.0)), 1.0)
    return (T(1.0) - T(p)) / T(1.0), p_star


def within_tolerance(got, ref, atol: float = 2e-2, rtol: float = 1e-2):
    """The pass rule for floating-point outputs: |got - ref| <= atol + rtol |ref| for every
    element.  Returns (ok, max_abs_err, max_rel_err over |ref| > 1e-3)."""
    got = _f64(got)
    ref = _f64(ref)
    err = np.abs(got - ref)
    ok = bool(np.all(err <= atol + rtol * np.abs(ref)))
    big = np.abs(ref) > 1e-3
    max_rel = float(np.max(err[big] / np.abs(ref[big]))) if np.any(big) else 0.0
    return ok, float(err.max()) if err.size else 0.0, max_rel

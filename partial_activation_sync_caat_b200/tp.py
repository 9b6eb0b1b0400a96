"""The partially synchronized row-parallel layer over real devices: one tensor-parallel rank per
process and GPU, with torch.distributed (NCCL) for its one exchange step.

"Tensor-Parallelism with Partially Synchronized Activations" (App. A.2 Eq. 22; §3; App. D):
each rank computes its partial product X_r W_r^T; only the first n_s = floor(H p) channels
(the shared ones) are summed over the ranks -- an all-reduce of T x n_s values, the fraction p
of a full all-reduce of the layer's output -- and every rank finishes its residual add and
RMSNorm locally.  The arithmetic runs in the library's kernels (caat_rowpar_tp_local and
caat_rowpar_tp_finish); this module only allocates the buffers and calls the collective:

    local:  zs = (X_r W_r^T)[:, :n_s] (fp32), h[:, n_s:] = s (X_r W_r^T)[:, n_s:] + R_r[:, n_s:]
    reduce: zs <- sum over ranks of zs (fp32, all ranks receive it)
    finish: h[:, :n_s] = bf16(zs + R_r[:, :n_s]);  out = h / sqrt(mean h^2 + eps) * gamma
"""
from __future__ import annotations

import math


def n_shared(H: int, p: float) -> int:
    """floor(H p) evaluated in double, as the library does."""
    return int(math.floor(float(H) * float(p)))


def exchanged_bytes(T: int, H: int, p: float) -> int:
    """Bytes of the buffer the collective reduces per call (fp32 partials of the shared
    channels); a full all-reduce of the layer's fp32 output would be 4 T H."""
    return 4 * T * n_shared(H, p)


class TPRowParallel:
    """One rank of the layer.  local_fn / finish_fn / reduce_fn default to the library's kernels
    and torch.distributed.all_reduce (sum) on `group`; they are parameters only so that the
    orchestration can be exercised on CPU ranks (gloo) with stand-ins for the two kernels."""

    def __init__(self, H: int, p: float, *, group=None, eps: float = 1e-5, private_scale: float = 1.0,
                 local_fn=None, finish_fn=None, reduce_fn=None):
        from . import caat as C
        self.H = int(H)
        self.p = float(p)
        self.n_s = n_shared(H, p)
        self.eps = float(eps)
        self.private_scale = float(private_scale)
        self.group = group
        self.local_fn = local_fn or C.caat_rowpar_tp_local
        self.finish_fn = finish_fn or C.caat_rowpar_tp_finish
        self.reduce_fn = reduce_fn or self._all_reduce

    def _all_reduce(self, t):
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)

    def buffers(self, T: int, device):
        """The per-call buffers: zs [T, n_s] fp32 and h [T, H] bf16 (reusable across calls)."""
        import torch
        zs = torch.empty(T, self.n_s, dtype=torch.float32, device=device)
        h = torch.empty(T, self.H, dtype=torch.bfloat16, device=device)
        return zs, h

    def forward(self, X_r, W_r, R_r, gamma, out, *, zs=None, h=None, workspace=None, stream=None):
        """X_r [T, K_r], W_r [H, K_r], R_r [T, H], gamma [H] (bf16) -> out [T, H]; returns (out, h),
        h being the complete pre-norm residual stream of this rank."""
        import contextlib
        T = int(X_r.shape[0])
        if zs is None or h is None:
            zs, h = self.buffers(T, X_r.device)
        kw = {"private_scale": self.private_scale}
        if workspace is not None:
            kw["workspace"] = workspace
        # the kernels and the collective are queued on the current stream (or `stream`)
        ctx = contextlib.nullcontext()
        if stream is not None:
            import torch
            ctx = torch.cuda.stream(stream)
        with ctx:
            self.local_fn(X_r, W_r, R_r, self.p, zs, h, **kw)
            if self.n_s > 0:
                self.reduce_fn(zs)
            self.finish_fn(zs, R_r, h, gamma, self.p, out, eps=self.eps)
        return out, h

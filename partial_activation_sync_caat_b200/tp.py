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


def peer_exchange_bytes(T: int, H: int, p: float, world: int) -> int:
    """Bytes one rank sends per call with the exchange over peer memory: its fp32 partials of
    the other owners' columns ((world - 1) / world of T n_s values), then the sums of its own
    slice to the other ranks (the same amount); a ring all-reduce of zs sends as much."""
    ns = n_shared(H, p)
    return 2 * 4 * T * (ns - ns // world) if world > 1 else 0


class CudaPeerMemory:
    """Device buffers shared between the ranks' processes with CUDA IPC (the CUDA runtime through
    cuda-python).  alloc returns (handle, address): the handle (bytes) travels to the other
    ranks, which map it with open."""

    def __init__(self):
        from cuda.bindings import runtime as rt
        self.rt = rt
        self.own, self.mapped = [], []

    def _ok(self, res, what):
        err = res[0] if isinstance(res, tuple) else res
        if int(err) != 0:
            raise RuntimeError(f"{what} failed: {err}")
        return res[1] if isinstance(res, tuple) and len(res) > 1 else None

    def alloc(self, nbytes: int):
        ptr = self._ok(self.rt.cudaMalloc(int(nbytes)), "cudaMalloc")
        self._ok(self.rt.cudaMemset(ptr, 0, int(nbytes)), "cudaMemset")
        self._ok(self.rt.cudaDeviceSynchronize(), "cudaDeviceSynchronize")  # zeroed before any peer maps it
        self.own.append(ptr)
        handle = self._ok(self.rt.cudaIpcGetMemHandle(ptr), "cudaIpcGetMemHandle")
        return bytes(handle.reserved), int(ptr)

    def open(self, handle: bytes) -> int:
        h = self.rt.cudaIpcMemHandle_t()
        h.reserved = handle
        ptr = self._ok(self.rt.cudaIpcOpenMemHandle(h, self.rt.cudaIpcMemLazyEnablePeerAccess),
                       "cudaIpcOpenMemHandle")
        self.mapped.append(ptr)
        return int(ptr)

    def close_mapped(self):
        for ptr in self.mapped:
            self.rt.cudaIpcCloseMemHandle(ptr)
        self.mapped = []

    def free_own(self):
        for ptr in self.own:
            self.rt.cudaFree(ptr)
        self.own = []


class LibraryPeerOps:
    """The three steps of the exchange over peer memory: the library's kernels."""

    def __init__(self):
        from . import caat as C
        self.C = C

    def peers(self, world, rank, epoch, recv, gather, flags):
        return self.C.tp_peers(world, rank, epoch, recv, gather, flags)

    def push(self, X_r, W_r, R_r, p, h, peers, *, workspace, private_scale):
        self.C.caat_rowpar_tp_local_push(X_r, W_r, R_r, p, h, peers, workspace=workspace,
                                         private_scale=private_scale)

    def reduce(self, T, H, p, peers, *, workspace):
        self.C.caat_rowpar_tp_reduce(T, H, p, peers, workspace=workspace)

    def finish(self, R_r, h, gamma, p, out, peers, *, eps):
        self.C.caat_rowpar_tp_finish_wait(R_r, h, gamma, p, out, peers, eps=eps)


class TPRowParallelP2P:
    """One rank of the layer with the exchange over peer memory, no collective library on the
    data path (the group is used once, to trade buffer handles).  Owner q of the `world` ranks
    owns the shared columns [q w, (q + 1) w), w = n_s / world.  Per call (epoch e):

        push:    this rank's GEMM stores its fp32 partial of owner q's columns into
                 recv_q[rank] (peer memory), then raises flags_q[0][rank] = e on every q;
        reduce:  once flags_rank[0][*] = e, the sum over ranks of recv_rank (rank order, fp32)
                 goes to gather_g[:, rank w:(rank + 1) w] of every rank g, then flags_g[1][rank] = e;
        finish:  once flags_rank[1][*] = e, h[:, :n_s] = bf16(gather_rank + R[:, :n_s]), RMSNorm.

    Buffers per rank, allocated once for up to T_max tokens: recv [world][T_max][w] fp32,
    gather [T_max][n_s] fp32, flags [2][world] uint32 (zeroed).  `memory` and `ops` default to
    CUDA IPC and the library's kernels; they are parameters only so that the protocol can be
    exercised by CPU processes (gloo) with stand-ins."""

    def __init__(self, H: int, p: float, T_max: int, *, group=None, eps: float = 1e-5,
                 private_scale: float = 1.0, memory=None, ops=None):
        import torch.distributed as dist
        self.H, self.p, self.T_max = int(H), float(p), int(T_max)
        self.n_s = n_shared(H, p)
        self.eps, self.private_scale = float(eps), float(private_scale)
        self.group = group
        init = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if init else 1
        self.rank = dist.get_rank(group) if init else 0
        if self.n_s % (32 * self.world) != 0:
            raise ValueError(f"n_s = {self.n_s} must be a multiple of 32 * world = {32 * self.world}")
        self.w = self.n_s // self.world
        self.memory = memory if memory is not None else CudaPeerMemory()
        self.ops = ops if ops is not None else LibraryPeerOps()
        sizes = (4 * self.world * self.T_max * max(self.w, 4), 4 * self.T_max * max(self.n_s, 4),
                 4 * 2 * self.world)
        own = [self.memory.alloc(n) for n in sizes]  # (handle, address) of recv, gather, flags
        handles = [own[i][0] for i in range(3)]
        if self.world > 1:
            everyone = [None] * self.world
            dist.all_gather_object(everyone, handles, group=group)
        else:
            everyone = [handles]
        self.recv, self.gather, self.flags = [], [], []
        for q in range(self.world):
            if q == self.rank:
                addrs = [own[i][1] for i in range(3)]
            else:
                addrs = [self.memory.open(everyone[q][i]) for i in range(3)]
            self.recv.append(addrs[0])
            self.gather.append(addrs[1])
            self.flags.append(addrs[2])
        self.epoch = 0

    def close(self):
        """Unmaps the other ranks' buffers, waits until every rank has done so, then frees this
        rank's own (an exporter frees only after every importer has closed its mapping).  Call it
        on every rank, after the last forward has completed."""
        import torch.distributed as dist
        self.memory.close_mapped()
        if self.world > 1:
            dist.barrier(group=self.group)
        self.memory.free_own()

    def forward(self, X_r, W_r, R_r, gamma, out, *, h=None, workspace=None):
        """X_r [T, K_r], W_r [H, K_r], R_r [T, H], gamma [H] (bf16) -> out [T, H]; returns
        (out, h).  Every rank calls it with the same T <= T_max, in the same order."""
        import torch
        T = int(X_r.shape[0])
        if T > self.T_max:
            raise ValueError(f"T = {T} exceeds T_max = {self.T_max}")
        if h is None:
            h = torch.empty(T, self.H, dtype=torch.bfloat16, device=X_r.device)
        if workspace is None:
            workspace = torch.empty(256, dtype=torch.uint8, device=X_r.device)
        self.epoch += 1
        pe = self.ops.peers(self.world, self.rank, self.epoch, self.recv, self.gather, self.flags)
        self.ops.push(X_r, W_r, R_r, self.p, h, pe, workspace=workspace, private_scale=self.private_scale)
        self.ops.reduce(T, self.H, self.p, pe, workspace=workspace)
        self.ops.finish(R_r, h, gamma, self.p, out, pe, eps=self.eps)
        return out, h

"""Python binding of the C ABI in include/caat.h (argument marshalling only).

Every step of the path runs in the CUDA kernels of libcaat.so; this module only turns torch
tensors into pointers, sizes and a stream, calls the library and turns error codes into
exceptions.  There is no fallback: if libcaat.so is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcaat.so")

CAAT_OK = 0
CAAT_ERR_INVALID_ARG = 1
CAAT_ERR_UNSUPPORTED = 2
CAAT_ERR_CUDA = 3
CAAT_ERR_TIMEOUT = 4
CAAT_ERR_WORKSPACE = 5

CAAT_VARIANT_ROWPAR = 0
CAAT_VARIANT_MLP = 1
CAAT_VARIANT_ROWPAR_HOST = 2
CAAT_VARIANT_ROWPAR_BWD = 4
CAAT_BWD_FLAG_TRANSPOSED_OPERANDS = 0x1

CAAT_FLAG_FORCE_GEMM_PATH = 0x1
CAAT_FLAG_FORCE_DECODE_PATH = 0x2
CAAT_FLAG_SINGLE_CTA = 0x4
CAAT_FLAG_FUSED_NORM = 0x8
CAAT_FLAG_ORDER_ROWBLOCK = 0x10
CAAT_FLAG_OVERLAP_NORM = 0x20
CAAT_FLAG_ORDER_GROUPED = 0x40
CAAT_FLAG_W_PERMUTED = 0x80
CAAT_FLAG_TEST_STALL = 0x100
CAAT_FLAG_NORM_BESIDE_GEMM = 0x200

CAAT_NOALLOC_SCRATCH_BYTES = 1048576

# Every symbol include/caat.h declares (checked by the ABI tests).
EXPORTS = [
    "caat_rowpar_forward", "caat_rowpar_forward_ex", "caat_rowpar_forward_host",
    "caat_rowpar_forward_noalloc", "caat_mlp_forward", "caat_mlp_forward_ex",
    "caat_workspace_size", "caat_sync_mask", "caat_get_device_status", "caat_timing_create",
    "caat_timing_destroy", "caat_timing_reset", "caat_timing_read", "caat_status_string",
    "caat_version", "caat_permute_weights", "caat_speedup_model", "caat_rowpar_backward",
    "caat_plan_create", "caat_plan_execute", "caat_plan_destroy", "caat_rowpar_tp_local",
    "caat_rowpar_tp_finish", "caat_rowpar_tp_local_push", "caat_rowpar_tp_reduce", "caat_rowpar_tp_finish_wait",
]

CAAT_TP_MAX_WORLD = 8


class CaatError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


class RowparArgs(ctypes.Structure):
    _fields_ = [
        ("X", ctypes.c_void_p), ("W", ctypes.c_void_p), ("residual", ctypes.c_void_p),
        ("gamma", ctypes.c_void_p), ("sync_idx", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("h_out", ctypes.c_void_p), ("workspace", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t),
        ("stream", ctypes.c_void_p), ("timing", ctypes.c_void_p),
        ("T", ctypes.c_int64), ("K", ctypes.c_int64), ("H", ctypes.c_int64),
        ("p", ctypes.c_double), ("eps", ctypes.c_float), ("private_scale", ctypes.c_float),
        ("P", ctypes.c_int32), ("flags", ctypes.c_uint32),
    ]


class BwdArgs(ctypes.Structure):
    _fields_ = [
        ("X", ctypes.c_void_p), ("W", ctypes.c_void_p), ("h", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
        ("dout", ctypes.c_void_p), ("sync_idx", ctypes.c_void_p), ("dX", ctypes.c_void_p),
        ("dW", ctypes.c_void_p), ("dR", ctypes.c_void_p), ("dgamma", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t), ("stream", ctypes.c_void_p),
        ("timing", ctypes.c_void_p), ("T", ctypes.c_int64), ("K", ctypes.c_int64), ("H", ctypes.c_int64),
        ("p", ctypes.c_double), ("eps", ctypes.c_float), ("private_scale", ctypes.c_float),
        ("P", ctypes.c_int32), ("flags", ctypes.c_uint32),
    ]


class TpArgs(ctypes.Structure):
    _fields_ = [
        ("X", ctypes.c_void_p), ("W", ctypes.c_void_p), ("residual", ctypes.c_void_p),
        ("gamma", ctypes.c_void_p), ("zs", ctypes.c_void_p), ("h", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t), ("stream", ctypes.c_void_p),
        ("timing", ctypes.c_void_p), ("T", ctypes.c_int64), ("K_r", ctypes.c_int64), ("H", ctypes.c_int64),
        ("p", ctypes.c_double), ("eps", ctypes.c_float), ("private_scale", ctypes.c_float),
        ("flags", ctypes.c_uint32),
    ]


class TpPeers(ctypes.Structure):
    _fields_ = [
        ("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("epoch", ctypes.c_uint32),
        ("recv", ctypes.c_void_p * CAAT_TP_MAX_WORLD), ("gather", ctypes.c_void_p * CAAT_TP_MAX_WORLD),
        ("flags", ctypes.c_void_p * CAAT_TP_MAX_WORLD),
    ]


class MlpArgs(ctypes.Structure):
    _fields_ = [
        ("X", ctypes.c_void_p), ("A", ctypes.c_void_p), ("W2", ctypes.c_void_p),
        ("residual", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("sync_idx", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("h_out", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("ws_bytes", ctypes.c_size_t), ("stream", ctypes.c_void_p), ("timing", ctypes.c_void_p),
        ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("F", ctypes.c_int64),
        ("p", ctypes.c_double), ("eps", ctypes.c_float), ("private_scale", ctypes.c_float),
        ("P", ctypes.c_int32), ("flags", ctypes.c_uint32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libcaat.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libcaat.so not built ({LIB_PATH}); run `python -m partial_activation_sync_caat_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i64, i32, u32, dbl, vp, sz = (ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_double,
                                  ctypes.c_void_p, ctypes.c_size_t)
    L.caat_rowpar_forward.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, dbl, vp, i64, i64, i64, vp, sz, vp]
    L.caat_rowpar_forward.restype = ctypes.c_int
    L.caat_rowpar_forward_ex.argtypes = [ctypes.POINTER(RowparArgs)]
    L.caat_rowpar_forward_ex.restype = ctypes.c_int
    L.caat_rowpar_forward_host.argtypes = [ctypes.POINTER(RowparArgs)]
    L.caat_rowpar_forward_host.restype = ctypes.c_int
    L.caat_rowpar_forward_noalloc.argtypes = [ctypes.POINTER(RowparArgs)]
    L.caat_rowpar_forward_noalloc.restype = ctypes.c_int
    L.caat_mlp_forward.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, dbl, vp, i64, i64, i64, vp, sz, vp]
    L.caat_mlp_forward.restype = ctypes.c_int
    L.caat_mlp_forward_ex.argtypes = [ctypes.POINTER(MlpArgs)]
    L.caat_mlp_forward_ex.restype = ctypes.c_int
    L.caat_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_int]
    L.caat_workspace_size.restype = sz
    L.caat_sync_mask.argtypes = [i64, dbl, vp, vp, ctypes.POINTER(i64)]
    L.caat_plan_create.restype = ctypes.c_int
    L.caat_plan_create.argtypes = [ctypes.POINTER(RowparArgs), ctypes.POINTER(vp)]
    L.caat_plan_execute.restype = ctypes.c_int
    L.caat_plan_execute.argtypes = [vp, vp]
    L.caat_plan_destroy.restype = ctypes.c_int
    L.caat_plan_destroy.argtypes = [vp]
    L.caat_rowpar_tp_local.argtypes = [ctypes.POINTER(TpArgs)]
    L.caat_rowpar_tp_local.restype = ctypes.c_int
    L.caat_rowpar_tp_finish.argtypes = [ctypes.POINTER(TpArgs)]
    for name in ("caat_rowpar_tp_local_push", "caat_rowpar_tp_reduce", "caat_rowpar_tp_finish_wait"):
        getattr(L, name).argtypes = [ctypes.POINTER(TpArgs), ctypes.POINTER(TpPeers)]
        getattr(L, name).restype = ctypes.c_int
    L.caat_rowpar_tp_finish.restype = ctypes.c_int
    L.caat_rowpar_backward.restype = ctypes.c_int
    L.caat_rowpar_backward.argtypes = [ctypes.POINTER(BwdArgs)]
    L.caat_speedup_model.restype = ctypes.c_int
    L.caat_speedup_model.argtypes = [dbl, dbl, dbl, dbl, dbl, ctypes.POINTER(dbl), ctypes.POINTER(dbl)]
    L.caat_permute_weights.restype = ctypes.c_int
    L.caat_permute_weights.argtypes = [vp, vp, vp, dbl, ctypes.c_int, i64, i64, vp]
    L.caat_sync_mask.restype = ctypes.c_int
    L.caat_get_device_status.argtypes = [vp, ctypes.POINTER(i32)]
    L.caat_get_device_status.restype = ctypes.c_int
    L.caat_timing_create.argtypes = [ctypes.c_int, ctypes.POINTER(vp)]
    L.caat_timing_create.restype = ctypes.c_int
    L.caat_timing_destroy.argtypes = [vp]
    L.caat_timing_destroy.restype = ctypes.c_int
    L.caat_timing_reset.argtypes = [vp]
    L.caat_timing_reset.restype = ctypes.c_int
    L.caat_timing_read.argtypes = [vp, ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.c_int,
                                   ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    L.caat_timing_read.restype = ctypes.c_int
    L.caat_status_string.argtypes = [ctypes.c_int]
    L.caat_status_string.restype = ctypes.c_char_p
    L.caat_version.argtypes = []
    L.caat_version.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().caat_status_string(int(code)).decode()


def version() -> str:
    return lib().caat_version().decode()


def _check(code: int, what: str):
    if code != CAAT_OK:
        raise CaatError(code, what)


# ---------------------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------------------

def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _bf16_dev(t, name):
    import torch
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return _ptr(t)


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def _sync_idx_host(sync_idx):
    if sync_idx is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(sync_idx, dtype=np.int32))
    return arr, arr.ctypes.data


# ---------------------------------------------------------------------------------------
# host-only bookkeeping
# ---------------------------------------------------------------------------------------

def caat_sync_mask(H: int, p: float, sync_idx=None):
    """(mask uint8[H], n_s) as computed by the library on the host (no GPU needed)."""
    mask = np.zeros(int(H), dtype=np.uint8)
    ns = ctypes.c_int64(0)
    arr, ptr = _sync_idx_host(sync_idx)
    code = lib().caat_sync_mask(int(H), float(p), ptr, mask.ctypes.data, ctypes.byref(ns))
    _check(code, "caat_sync_mask")
    return mask, int(ns.value)


def caat_speedup_model(h: float, s: float, r: float, p: float, C: float):
    """(speedup, p_star) of the paper's model (App. C Eq. 34-35); host only."""
    sp, ps = ctypes.c_double(0.0), ctypes.c_double(0.0)
    _check(lib().caat_speedup_model(float(h), float(s), float(r), float(p), float(C), ctypes.byref(sp),
                                    ctypes.byref(ps)), "caat_speedup_model")
    return sp.value, ps.value


def caat_permute_weights(W, W_out, sync_idx, P: int, p: float, stream=None):
    """W_out[m, i] = W[m, perm(i)]: the shared channels first, then the private ones (both
    ascending).  W, W_out: device bf16 [P, H, K/P], not overlapping.  Asynchronous."""
    P_, H, Kp = W.shape
    if P_ != P or tuple(W_out.shape) != tuple(W.shape):
        raise CaatError(CAAT_ERR_INVALID_ARG, "caat_permute_weights: shapes")
    arr, ptr = _sync_idx_host(sync_idx)
    code = lib().caat_permute_weights(_ptr(W), _ptr(W_out), ptr, float(p), int(P), int(H), int(Kp * P),
                                      _stream_ptr(stream))
    _check(code, "caat_permute_weights")


def caat_workspace_size(T: int, K: int, H: int, P: int, variant: int = CAAT_VARIANT_ROWPAR) -> int:
    n = lib().caat_workspace_size(int(T), int(K), int(H), int(P), int(variant))
    if n == ctypes.c_size_t(-1).value:
        raise CaatError(CAAT_ERR_INVALID_ARG, "caat_workspace_size")
    return int(n)


def alloc_workspace(nbytes: int, device=None):
    """A device buffer for the workspace (allocated by torch, owned by the caller)."""
    import torch
    n = max(256, (int(nbytes) + 255) // 256 * 256)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------------------------------
# forward calls
# ---------------------------------------------------------------------------------------

def caat_rowpar_forward(X, W, residual, gamma, sync_idx, P: int, p: float, out, *, workspace=None,
                        h_out=None, eps: float = 1e-5, private_scale: float = 1.0, flags: int = 0,
                        stream=None, timing=None):
    """Queues the partially synchronized row-parallel layer + residual + RMSNorm.

    X [P,T,K/P], W [P,H,K/P], residual [P,T,H], gamma [H], out [P,T,H] (bf16 CUDA tensors);
    sync_idx: None (first floor(H p) channels) or a host int list of floor(H p) channels.
    """
    P = int(P)
    T = int(X.shape[1])
    K = int(X.shape[2]) * P
    H = int(W.shape[1])
    if workspace is None:
        workspace = alloc_workspace(caat_workspace_size(T, K, H, P, CAAT_VARIANT_ROWPAR), X.device)
    arr, idx_ptr = _sync_idx_host(sync_idx)
    a = RowparArgs()
    a.X = _bf16_dev(X, "X")
    a.W = _bf16_dev(W, "W")
    a.residual = _bf16_dev(residual, "residual")
    a.gamma = _bf16_dev(gamma, "gamma")
    a.sync_idx = idx_ptr
    a.out = _bf16_dev(out, "out")
    a.h_out = _bf16_dev(h_out, "h_out") if h_out is not None else None
    a.workspace = _ptr(workspace)
    a.ws_bytes = workspace.numel() * workspace.element_size()
    a.stream = _stream_ptr(stream)
    a.timing = timing.handle if timing is not None else None
    a.T, a.K, a.H = T, K, H
    a.p = float(p)
    a.eps = float(eps)
    a.private_scale = float(private_scale)
    a.P = P
    a.flags = int(flags)
    _check(lib().caat_rowpar_forward_ex(ctypes.byref(a)), "caat_rowpar_forward")
    return out


class Plan:
    """A caat_plan: the row-parallel call with its buffers bound once; execute() only queues
    the kernels.  The tensors given at creation must outlive the plan (they are kept here)."""

    def __init__(self, X, W, residual, gamma, sync_idx, P: int, p: float, out, *, workspace=None, h_out=None,
                 eps: float = 1e-5, private_scale: float = 1.0, flags: int = 0):
        P = int(P)
        T, K, H = int(X.shape[1]), int(X.shape[2]) * P, int(W.shape[1])
        if workspace is None:
            workspace = alloc_workspace(caat_workspace_size(T, K, H, P, CAAT_VARIANT_ROWPAR), X.device)
        self._keep = (X, W, residual, gamma, out, h_out, workspace)
        arr, idx_ptr = _sync_idx_host(sync_idx)
        a = RowparArgs()
        a.X, a.W = _bf16_dev(X, "X"), _bf16_dev(W, "W")
        a.residual, a.gamma = _bf16_dev(residual, "residual"), _bf16_dev(gamma, "gamma")
        a.sync_idx = idx_ptr
        a.out = _bf16_dev(out, "out")
        a.h_out = _bf16_dev(h_out, "h_out") if h_out is not None else None
        a.workspace = _ptr(workspace)
        a.ws_bytes = workspace.numel() * workspace.element_size()
        a.stream = None
        a.timing = None
        a.T, a.K, a.H = T, K, H
        a.p, a.eps, a.private_scale, a.P, a.flags = float(p), float(eps), float(private_scale), P, int(flags)
        h = ctypes.c_void_p(None)
        _check(lib().caat_plan_create(ctypes.byref(a), ctypes.byref(h)), "caat_plan_create")
        self.handle = h.value

    def execute(self, stream=None):
        _check(lib().caat_plan_execute(self.handle, _stream_ptr(stream)), "caat_plan_execute")

    def close(self):
        if self.handle:
            lib().caat_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _f32_dev(t, name):
    import torch
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return _ptr(t)


def _tp_args(T, K_r, H, p, eps, private_scale, stream, timing):
    a = TpArgs()
    a.T, a.K_r, a.H = int(T), int(K_r), int(H)
    a.p = float(p)
    a.eps = float(eps)
    a.private_scale = float(private_scale)
    a.stream = _stream_ptr(stream)
    a.timing = timing.handle if timing is not None else None
    a.flags = 0
    return a


def caat_rowpar_tp_local(X, W, residual, p: float, zs, h, *, workspace=None, private_scale: float = 1.0,
                         stream=None, timing=None):
    """Local step of one rank of the layer over real devices: X [T,K_r], W [H,K_r], residual
    [T,H] (bf16, this rank's); writes zs [T, floor(H p)] (fp32, this rank's partial of the shared
    channels) and the private channels of h [T,H] (bf16)."""
    T, K_r = int(X.shape[0]), int(X.shape[1])
    H = int(W.shape[0])
    if workspace is None:
        workspace = alloc_workspace(256, X.device)
    a = _tp_args(T, K_r, H, p, 1e-5, private_scale, stream, timing)
    a.X = _bf16_dev(X, "X")
    a.W = _bf16_dev(W, "W")
    a.residual = _bf16_dev(residual, "residual")
    a.zs = _f32_dev(zs, "zs") if zs is not None and zs.numel() else None
    a.h = _bf16_dev(h, "h")
    a.workspace = _ptr(workspace)
    a.ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().caat_rowpar_tp_local(ctypes.byref(a)), "caat_rowpar_tp_local")
    return zs, h


def caat_rowpar_tp_finish(zs, residual, h, gamma, p: float, out, *, eps: float = 1e-5, stream=None, timing=None):
    """Finishing step after the exchange: zs [T, floor(H p)] holds the sum over the ranks;
    writes the shared channels of h [T,H] and out [T,H] = RMSNorm(h) * gamma."""
    T, H = int(h.shape[0]), int(h.shape[1])
    a = _tp_args(T, 0, H, p, eps, 1.0, stream, timing)
    a.residual = _bf16_dev(residual, "residual")
    a.gamma = _bf16_dev(gamma, "gamma")
    a.zs = _f32_dev(zs, "zs") if zs is not None and zs.numel() else None
    a.h = _bf16_dev(h, "h")
    a.out = _bf16_dev(out, "out")
    _check(lib().caat_rowpar_tp_finish(ctypes.byref(a)), "caat_rowpar_tp_finish")
    return out


def tp_peers(world: int, rank: int, epoch: int, recv, gather, flags) -> TpPeers:
    """Descriptor of the peer-memory exchange for one rank and call: recv[q], gather[q], flags[q]
    are rank q's buffers (CUDA tensors, or device addresses as ints, valid in this process):
    recv [world, T, n_s / world] fp32, gather [T, n_s] fp32, flags [2, world] int32 zeroed once."""
    world = int(world)
    if not 1 <= world <= CAAT_TP_MAX_WORLD:
        raise ValueError(f"world must be 1..{CAAT_TP_MAX_WORLD}")
    pe = TpPeers()
    pe.world, pe.rank, pe.epoch = world, int(rank), int(epoch)

    def addr(x):
        return int(x) if isinstance(x, int) else _ptr(x)
    for q in range(world):
        pe.recv[q] = addr(recv[q])
        pe.gather[q] = addr(gather[q])
        pe.flags[q] = addr(flags[q])
    return pe


def caat_rowpar_tp_local_push(X, W, residual, p: float, h, peers: TpPeers, *, workspace=None,
                              private_scale: float = 1.0, stream=None, timing=None):
    """Local step of the peer-memory exchange: as caat_rowpar_tp_local, with this rank's fp32
    partials of the shared channels stored into their owners' receive buffers (peers.recv)."""
    T, K_r = int(X.shape[0]), int(X.shape[1])
    H = int(W.shape[0])
    if workspace is None:
        workspace = alloc_workspace(256, X.device)
    a = _tp_args(T, K_r, H, p, 1e-5, private_scale, stream, timing)
    a.X = _bf16_dev(X, "X")
    a.W = _bf16_dev(W, "W")
    a.residual = _bf16_dev(residual, "residual")
    a.h = _bf16_dev(h, "h")
    a.workspace = _ptr(workspace)
    a.ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().caat_rowpar_tp_local_push(ctypes.byref(a), ctypes.byref(peers)), "caat_rowpar_tp_local_push")
    return h


def caat_rowpar_tp_reduce(T: int, H: int, p: float, peers: TpPeers, *, workspace, stream=None, timing=None):
    """Owner step of the peer-memory exchange: sums this rank's slice of the shared channels over
    the ranks and writes it into every rank's gather buffer.  workspace: >= 256 bytes, device."""
    a = _tp_args(T, 0, H, p, 1e-5, 1.0, stream, timing)
    a.workspace = _ptr(workspace)
    a.ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().caat_rowpar_tp_reduce(ctypes.byref(a), ctypes.byref(peers)), "caat_rowpar_tp_reduce")


def caat_rowpar_tp_finish_wait(residual, h, gamma, p: float, out, peers: TpPeers, *, eps: float = 1e-5, stream=None,
                               timing=None):
    """Finishing step of the peer-memory exchange: waits for every owner's slice, then as
    caat_rowpar_tp_finish with zs = this rank's gather buffer."""
    T, H = int(h.shape[0]), int(h.shape[1])
    a = _tp_args(T, 0, H, p, eps, 1.0, stream, timing)
    a.residual = _bf16_dev(residual, "residual")
    a.gamma = _bf16_dev(gamma, "gamma")
    a.h = _bf16_dev(h, "h")
    a.out = _bf16_dev(out, "out")
    _check(lib().caat_rowpar_tp_finish_wait(ctypes.byref(a), ctypes.byref(peers)), "caat_rowpar_tp_finish_wait")
    return out


def caat_rowpar_backward(X, W, h, gamma, dout, sync_idx, P: int, p: float, dX, dW, dgamma, *, dR=None,
                         workspace=None, eps: float = 1e-5, private_scale: float = 1.0, stream=None, timing=None,
                         flags: int = 0):
    """Queues the backward of the layer: dX [P,T,K/P], dW [P,H,K/P] (bf16), dgamma [H] (fp32)
    and optionally dR [P,T,H] (bf16), from the forward's inputs, its pre-norm stream h and
    dout = dL/d(out).  flags: 0, or CAAT_BWD_FLAG_TRANSPOSED_OPERANDS (test hook: the gradient
    GEMMs on transposed K-major copies, bit-identical to the default MN-major reads)."""
    P = int(P)
    T = int(X.shape[1])
    K = int(X.shape[2]) * P
    H = int(W.shape[1])
    if workspace is None:
        workspace = alloc_workspace(caat_workspace_size(T, K, H, P, CAAT_VARIANT_ROWPAR_BWD), X.device)
    arr, idx_ptr = _sync_idx_host(sync_idx)
    a = BwdArgs()
    a.X, a.W, a.h = _bf16_dev(X, "X"), _bf16_dev(W, "W"), _bf16_dev(h, "h")
    a.gamma, a.dout = _bf16_dev(gamma, "gamma"), _bf16_dev(dout, "dout")
    a.sync_idx = idx_ptr
    a.dX, a.dW = _bf16_dev(dX, "dX"), _bf16_dev(dW, "dW")
    a.dR = _bf16_dev(dR, "dR") if dR is not None else None
    if dgamma.dtype.__str__() != "torch.float32" or not dgamma.is_cuda:
        raise TypeError("dgamma must be a float32 CUDA tensor")
    a.dgamma = _ptr(dgamma)
    a.workspace = _ptr(workspace)
    a.ws_bytes = workspace.numel() * workspace.element_size()
    a.stream = _stream_ptr(stream)
    a.timing = timing.handle if timing is not None else None
    a.T, a.K, a.H = T, K, H
    a.p = float(p)
    a.eps = float(eps)
    a.private_scale = float(private_scale)
    a.P = P
    a.flags = int(flags)
    _check(lib().caat_rowpar_backward(ctypes.byref(a)), "caat_rowpar_backward")


def caat_rowpar_forward_host(X, W, residual, gamma, sync_idx, P: int, p: float, out, workspace, *,
                             h_out=None, eps: float = 1e-5, private_scale: float = 1.0, flags: int = 0,
                             stream=None, timing=None):
    """The layer on HOST tensors (pinned CPU bf16 tensors): the library copies the inputs into
    `workspace` (a device buffer of caat_workspace_size(..., CAAT_VARIANT_ROWPAR_HOST) bytes),
    runs the kernels and copies out (and h_out) back, all queued on `stream`."""
    import torch
    P = int(P)
    T = int(X.shape[1])
    K = int(X.shape[2]) * P
    H = int(W.shape[1])
    for name, t in (("X", X), ("W", W), ("residual", residual), ("gamma", gamma), ("out", out)):
        if t.dtype != torch.bfloat16 or t.is_cuda:
            raise ValueError(f"{name} must be a bfloat16 CPU tensor")
    arr, idx_ptr = _sync_idx_host(sync_idx)
    a = RowparArgs()
    a.X, a.W, a.residual, a.gamma, a.out = _ptr(X), _ptr(W), _ptr(residual), _ptr(gamma), _ptr(out)
    a.h_out = _ptr(h_out) if h_out is not None else None
    a.sync_idx = idx_ptr
    a.workspace = _ptr(workspace)
    a.ws_bytes = workspace.numel() * workspace.element_size()
    a.stream = _stream_ptr(stream)
    a.timing = timing.handle if timing is not None else None
    a.T, a.K, a.H = T, K, H
    a.p = float(p)
    a.eps = float(eps)
    a.private_scale = float(private_scale)
    a.P = P
    a.flags = int(flags)
    _check(lib().caat_rowpar_forward_host(ctypes.byref(a)), "caat_rowpar_forward_host")
    return out


def caat_rowpar_forward_noalloc(X, W, residual, gamma, sync_idx, P: int, p: float, out, *, h_out=None,
                                eps: float = 1e-5, private_scale: float = 1.0, flags: int = 0,
                                stream=None, timing=None):
    """The layer without any device allocation, for callers that cannot allocate device memory:
    the library's built-in scratch array (CAAT_NOALLOC_SCRATCH_BYTES per GPU) replaces the
    workspace.  Calls that overlap on the GPU share that array and race; serialize them."""
    P = int(P)
    T = int(X.shape[1])
    K = int(X.shape[2]) * P
    H = int(W.shape[1])
    arr, idx_ptr = _sync_idx_host(sync_idx)
    a = RowparArgs()
    a.X = _bf16_dev(X, "X")
    a.W = _bf16_dev(W, "W")
    a.residual = _bf16_dev(residual, "residual")
    a.gamma = _bf16_dev(gamma, "gamma")
    a.sync_idx = idx_ptr
    a.out = _bf16_dev(out, "out")
    a.h_out = _bf16_dev(h_out, "h_out") if h_out is not None else None
    a.workspace = None
    a.ws_bytes = 0
    a.stream = _stream_ptr(stream)
    a.timing = timing.handle if timing is not None else None
    a.T, a.K, a.H = T, K, H
    a.p = float(p)
    a.eps = float(eps)
    a.private_scale = float(private_scale)
    a.P = P
    a.flags = int(flags)
    _check(lib().caat_rowpar_forward_noalloc(ctypes.byref(a)), "caat_rowpar_forward_noalloc")
    return out


def caat_mlp_forward(X, A, W2, residual, gamma, sync_idx, P: int, p: float, out, *, workspace=None,
                     h_out=None, eps: float = 1e-5, private_scale: float = 1.0, flags: int = 0,
                     stream=None, timing=None):
    """Queues the MLP block: FC1 + SwiGLU, partially synced FC2, residual, RMSNorm.

    X [P,T,H], A [P,2F/P,H], W2 [P,H,F/P], residual [P,T,H], gamma [H], out [P,T,H].
    """
    P = int(P)
    T = int(X.shape[1])
    H = int(X.shape[2])
    F = int(W2.shape[2]) * P
    if workspace is None:
        workspace = alloc_workspace(caat_workspace_size(T, F, H, P, CAAT_VARIANT_MLP), X.device)
    arr, idx_ptr = _sync_idx_host(sync_idx)
    a = MlpArgs()
    a.X = _bf16_dev(X, "X")
    a.A = _bf16_dev(A, "A")
    a.W2 = _bf16_dev(W2, "W2")
    a.residual = _bf16_dev(residual, "residual")
    a.gamma = _bf16_dev(gamma, "gamma")
    a.sync_idx = idx_ptr
    a.out = _bf16_dev(out, "out")
    a.h_out = _bf16_dev(h_out, "h_out") if h_out is not None else None
    a.workspace = _ptr(workspace)
    a.ws_bytes = workspace.numel() * workspace.element_size()
    a.stream = _stream_ptr(stream)
    a.timing = timing.handle if timing is not None else None
    a.T, a.H, a.F = T, H, F
    a.p = float(p)
    a.eps = float(eps)
    a.private_scale = float(private_scale)
    a.P = P
    a.flags = int(flags)
    _check(lib().caat_mlp_forward_ex(ctypes.byref(a)), "caat_mlp_forward")
    return out


def caat_get_device_status(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the device status word."""
    v = ctypes.c_int32(0)
    lib().caat_get_device_status(_stream_ptr(stream), ctypes.byref(v))
    return int(v.value)


class Timing:
    """Per-kernel CUDA-event recorder of the library (caat_timing_*)."""

    MAX_KERNELS = 8

    def __init__(self, capacity: int = 256):
        h = ctypes.c_void_p()
        _check(lib().caat_timing_create(int(capacity), ctypes.byref(h)), "caat_timing_create")
        self.handle = h.value
        self.capacity = capacity

    def reset(self):
        _check(lib().caat_timing_reset(self.handle), "caat_timing_reset")

    def read(self):
        """List of per-call lists of kernel durations in ms."""
        buf = (ctypes.c_float * (self.capacity * self.MAX_KERNELS))()
        nr, nk = ctypes.c_int(0), ctypes.c_int(0)
        _check(lib().caat_timing_read(self.handle, buf, self.capacity, self.MAX_KERNELS,
                                      ctypes.byref(nr), ctypes.byref(nk)), "caat_timing_read")
        return [[buf[r * self.MAX_KERNELS + k] for k in range(nk.value)] for r in range(nr.value)]

    def close(self):
        if self.handle:
            lib().caat_timing_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

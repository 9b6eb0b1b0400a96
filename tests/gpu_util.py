"""Helpers shared by the GPU parity tests (no arithmetic of the method lives here)."""
import numpy as np
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import build as B
from partial_activation_sync_caat_b200 import caat as C

# The pass rule for the normalized output (floating point): |gpu - oracle| <= ATOL + RTOL |oracle|.
ATOL = 2e-2
RTOL = 1e-2


def ensure_built():
    B.build()
    C.lib()


def to_dev(d):
    return {k: v.cuda() for k, v in d.items()}


def assert_out_close(got, ref, what=""):
    ok, max_abs, max_rel = O.within_tolerance(got, ref, ATOL, RTOL)
    assert ok, f"{what}: max_abs={max_abs:.3e} max_rel={max_rel:.3e}"
    return max_abs, max_rel


def assert_h_close(got, ref, what=""):
    """The pre-norm residual stream h is stored in bf16: relative rounding 2^-9 plus fp32
    accumulation.  Pass rule: |gpu - oracle| <= 8e-3 |oracle| + 2e-3 rms(oracle row)."""
    got = O._f64(got)
    ref = O._f64(ref)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    err = np.abs(got - ref)
    bound = 8e-3 * np.abs(ref) + 2e-3 * rms
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of bound, max err {err.max():.3e}"


def run_rowpar(d, P, p, sync_idx=None, *, eps=1e-5, private_scale=1.0, h_out=True, flags=0,
               out_alias_residual=False):
    """Runs the CUDA path on CPU-generated inputs; returns (out, h) on the CPU."""
    g = to_dev(d)
    out = g["R"] if out_alias_residual else torch.empty_like(g["R"])
    hb = torch.empty_like(g["R"]) if h_out else None
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], sync_idx, P, p, out, h_out=hb, eps=eps,
                          private_scale=private_scale, flags=flags)
    torch.cuda.synchronize()
    status = C.caat_get_device_status()
    assert status == 0, f"device status {status:#x}"
    return out.cpu(), (hb.cpu() if hb is not None else None)

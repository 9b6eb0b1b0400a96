"""C-ABI tests that need no GPU: the library loads, exports every symbol include/caat.h
declares, the host-side sync-set bookkeeping is bit-exact against the oracle, and invalid
calls are rejected with the documented codes before any device work."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import build as B
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return C.lib()


def header_symbols():
    with open(os.path.join(ROOT, "include", "caat.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^CAAT_API[^;(]*?\b(caat_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_what_binding_lists():
    assert header_symbols() == sorted(C.EXPORTS)


def header_constants():
    """Every numeric #define and enum value of include/caat.h named CAAT_*."""
    with open(os.path.join(ROOT, "include", "caat.h")) as f:
        text = f.read()
    consts = {}
    for name, val in re.findall(r"^#define (CAAT_\w+) (0x[0-9a-fA-F]+|\d+)u?\b", text, flags=re.M):
        consts[name] = int(val, 0)
    for name, val in re.findall(r"^\s+(CAAT_\w+) = (\d+),?", text, flags=re.M):
        consts[name] = int(val)
    return consts


def test_binding_constants_match_header():
    consts = header_constants()
    assert len(consts) >= 20
    for name, val in consts.items():
        if name in ("CAAT_MAX_H", "CAAT_MAX_P", "CAAT_DECODE_MAX_T") and not hasattr(C, name):
            continue  # limits the binding does not restate
        assert getattr(C, name) == val, name


def test_library_exports_every_declared_symbol(L):
    for name in header_symbols():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", C.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (caat_\w+)", out))
    assert set(header_symbols()) <= exported
    # nothing else of ours leaks out of the shared object
    assert all(s.startswith("caat_") for s in exported)


def test_version_and_status_strings(L):
    assert "sm_100a" in C.version()
    for code, name in [(0, "CAAT_OK"), (1, "CAAT_ERR_INVALID_ARG"), (2, "CAAT_ERR_UNSUPPORTED"),
                       (3, "CAAT_ERR_CUDA"), (4, "CAAT_ERR_TIMEOUT"), (5, "CAAT_ERR_WORKSPACE")]:
        assert C.status_string(code) == name


@pytest.mark.parametrize("H,p", [(768, 0.5), (768, 0.7), (768, 0.703125), (4096, 0.25), (4096, 0.0),
                                 (4096, 1.0), (2048, 0.5), (776, 0.333), (8, 0.5), (65536, 0.1)])
def test_sync_mask_contiguous_bit_exact(L, H, p):
    mask, ns = C.caat_sync_mask(H, p)
    ref = O.sync_mask(H, p)
    assert ns == O.n_sync(H, p)
    np.testing.assert_array_equal(mask.astype(bool), ref)


@pytest.mark.parametrize("H,p,seed", [(2048, 0.5, 0), (768, 0.25, 3), (4096, 0.75, 1), (16, 0.5, 9)])
def test_sync_mask_list_bit_exact(L, H, p, seed):
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed)
    mask, ns = C.caat_sync_mask(H, p, idx)
    np.testing.assert_array_equal(mask.astype(bool), O.sync_mask(H, p, idx))


@pytest.mark.parametrize("bad", [[1, 1, 2, 3], [3, 2, 1, 0], [0, 1, 2, 16], [-1, 0, 1, 2]])
def test_sync_mask_rejects_bad_lists(L, bad):
    with pytest.raises(C.CaatError) as e:
        C.caat_sync_mask(16, 0.25, bad)
    assert e.value.code == C.CAAT_ERR_INVALID_ARG


def test_sync_mask_rejects_bad_p(L):
    for p in (-0.01, 1.01, float("nan")):
        with pytest.raises(C.CaatError):
            C.caat_sync_mask(16, p)


def test_workspace_size(L):
    assert C.caat_workspace_size(8192, 11008, 4096, 8) >= 4
    with pytest.raises(C.CaatError):
        C.caat_workspace_size(8192, 11007, 4096, 8)   # K % P != 0


def _call(L, **kw):
    """Direct ABI call with fake (never dereferenced) pointers: validation runs first."""
    base = dict(X=0x10000, W=0x20000, R=0x30000, g=0x40000, idx=None, P=2, p=0.5, out=0x50000,
                T=256, K=768, H=768, ws=0x60000, ws_bytes=1 << 20, stream=None)
    base.update(kw)
    return L.caat_rowpar_forward(base["X"], base["W"], base["R"], base["g"], base["idx"], base["P"],
                                 base["p"], base["out"], base["T"], base["K"], base["H"], base["ws"],
                                 base["ws_bytes"], base["stream"])


def test_rejects_invalid_arguments_without_device_work(L):
    assert _call(L, P=0) == C.CAAT_ERR_INVALID_ARG
    assert _call(L, P=65) == C.CAAT_ERR_INVALID_ARG
    assert _call(L, T=-1) == C.CAAT_ERR_INVALID_ARG
    assert _call(L, p=1.5) == C.CAAT_ERR_INVALID_ARG
    assert _call(L, p=float("nan")) == C.CAAT_ERR_INVALID_ARG
    assert _call(L, X=None) == C.CAAT_ERR_INVALID_ARG
    assert _call(L, out=None) == C.CAAT_ERR_INVALID_ARG
    assert _call(L, K=770) == C.CAAT_ERR_UNSUPPORTED          # K % P != 0
    assert _call(L, K=772, P=2) == C.CAAT_ERR_UNSUPPORTED     # (K/P) % 8 != 0
    assert _call(L, H=770) == C.CAAT_ERR_UNSUPPORTED          # H % 8 != 0
    assert _call(L, H=65544) == C.CAAT_ERR_UNSUPPORTED        # H > CAAT_MAX_H
    assert _call(L, X=0x10008) == C.CAAT_ERR_UNSUPPORTED      # misaligned pointer
    assert _call(L, ws=None) == C.CAAT_ERR_WORKSPACE
    assert _call(L, ws_bytes=0) == C.CAAT_ERR_WORKSPACE
    assert _call(L, ws=0x60010) == C.CAAT_ERR_WORKSPACE       # not 256-byte aligned
    bad = np.array([5, 3], dtype=np.int32)
    assert _call(L, H=8, K=16, p=0.25, idx=bad.ctypes.data) == C.CAAT_ERR_INVALID_ARG


def test_empty_token_count_is_a_no_op(L):
    assert _call(L, T=0, X=None, W=None, R=None, g=None, out=None, ws=None, ws_bytes=0) == C.CAAT_OK


def test_ex_rejects_null_and_bad_eps(L):
    assert L.caat_rowpar_forward_ex(None) == C.CAAT_ERR_INVALID_ARG
    a = C.RowparArgs()
    a.X, a.W, a.residual, a.gamma, a.out = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    a.workspace, a.ws_bytes = 0x60000, 1 << 20
    a.T, a.K, a.H, a.P, a.p, a.eps, a.private_scale = 128, 256, 256, 2, 0.5, -1.0, 1.0
    assert L.caat_rowpar_forward_ex(ctypes.byref(a)) == C.CAAT_ERR_INVALID_ARG
    a.eps = float("inf")
    assert L.caat_rowpar_forward_ex(ctypes.byref(a)) == C.CAAT_ERR_INVALID_ARG
    a.eps, a.private_scale = 1e-5, float("nan")
    assert L.caat_rowpar_forward_ex(ctypes.byref(a)) == C.CAAT_ERR_INVALID_ARG


def test_permute_weights_rejects_invalid_arguments_without_device_work(L):
    def call(W=0x100000, Wo=0x900000, idx=None, p=0.5, P=2, H=768, K=768):
        return L.caat_permute_weights(W, Wo, idx, p, P, H, K, None)
    assert call(P=0) == C.CAAT_ERR_INVALID_ARG
    assert call(p=-0.1) == C.CAAT_ERR_INVALID_ARG
    assert call(H=770) == C.CAAT_ERR_UNSUPPORTED
    assert call(K=770) == C.CAAT_ERR_UNSUPPORTED
    assert call(W=None) == C.CAAT_ERR_INVALID_ARG
    assert call(Wo=0x100008) == C.CAAT_ERR_UNSUPPORTED          # misaligned
    assert call(Wo=0x100000 + 768 * 768) == C.CAAT_ERR_INVALID_ARG  # overlaps W (W is 768*768*2 bytes)
    bad = np.array([5, 3], dtype=np.int32)
    assert call(H=8, K=16, p=0.25, idx=bad.ctypes.data) == C.CAAT_ERR_INVALID_ARG


def test_plan_validation_without_device_work(L):
    a = C.RowparArgs()
    a.X, a.W, a.residual, a.gamma, a.out = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    a.workspace, a.ws_bytes = 0x60000, 1 << 20
    a.T, a.K, a.H, a.P, a.p, a.eps, a.private_scale = 128, 256, 256, 2, 0.5, 1e-5, 1.0
    h = ctypes.c_void_p(None)
    a.P = 0
    assert L.caat_plan_create(ctypes.byref(a), ctypes.byref(h)) == C.CAAT_ERR_INVALID_ARG and h.value is None
    a.P, a.ws_bytes = 2, 0
    assert L.caat_plan_create(ctypes.byref(a), ctypes.byref(h)) == C.CAAT_ERR_WORKSPACE and h.value is None
    assert L.caat_plan_create(None, ctypes.byref(h)) == C.CAAT_ERR_INVALID_ARG
    assert L.caat_plan_create(ctypes.byref(a), None) == C.CAAT_ERR_INVALID_ARG
    assert L.caat_plan_execute(None, None) == C.CAAT_ERR_INVALID_ARG
    assert L.caat_plan_destroy(None) == C.CAAT_OK
    # an empty call plans and executes as a no-op without a device
    a.T, a.X, a.W, a.residual, a.gamma, a.out, a.workspace = 0, None, None, None, None, None, None
    assert L.caat_plan_create(ctypes.byref(a), ctypes.byref(h)) == C.CAAT_OK and h.value
    assert L.caat_plan_execute(h, None) == C.CAAT_OK
    assert L.caat_plan_destroy(h) == C.CAAT_OK

"""The entry point that allocates no device memory (caat_rowpar_forward_noalloc).

It exists for callers that cannot call cudaMalloc (an embedding whose allocator belongs to
someone else, code that must not grow its memory footprint or enter an allocator in a hot
loop): its scratch is a fixed array inside the library instead of a caller-supplied
workspace.  This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it must pass alone in a fresh process too.

Each case runs the entry point twice in a row (the calls share the array and must re-clear
what has to start at zero) and compares both results with the float64 oracle and with the
workspace entry point (caat_rowpar_forward), within the tolerance of the other parity tests.
"""
import pytest
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I

from gpu_util import assert_out_close, ensure_built, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _check_twice(d, P, p, idx=None, flags=0, what=""):
    g = to_dev(d)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, idx)
    ws_out = torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, ws_out, flags=flags)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    ws_cpu = ws_out.cpu()
    assert_out_close(ws_cpu, ref, f"{what} workspace entry point vs oracle")
    for call in range(2):
        out = torch.full_like(g["R"], float("nan"))
        C.caat_rowpar_forward_noalloc(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out, flags=flags)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        got = out.cpu()
        assert_out_close(got, ref, f"{what} no-alloc call {call} vs oracle")
        assert_out_close(got, ws_cpu, f"{what} no-alloc call {call} vs workspace entry point")


@pytest.mark.parametrize("T,K,H,P,p,random_idx", [
    (300, 800, 776, 4, 0.5, False),     # GEMM path, norm beside the GEMM (job list in the array)
    (256, 1024, 1024, 4, 0.5, True),    # every column block mixed: completion flags in the array
    (1024, 4096, 2048, 8, 0.75, False),
    (8, 1024, 1024, 4, 0.5, False),     # decode path: fp32 partials (128 KiB) in the array
])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(T, K, H, P, p, random_idx):
    d = I.make_rowpar_inputs(T, K, H, P, seed=21, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=2) if random_idx else None
    _check_twice(d, P, p, idx, what=f"T={T} H={H} P={P}")


@pytest.mark.parametrize("T", [1, 8, 64])
def test_noalloc_decode_shapes_7b(T):
    """The 7B decode shapes (H=4096, K=11008, P=8, p=0.5).  T=1: the decode partials (128 KiB)
    fit in the array; T=8 and 64 need 1 MiB + and 8 MiB, so those calls take the GEMM path,
    which needs only the unit counter and the job list."""
    d = I.make_rowpar_inputs(T, 11008, 4096, 8, seed=22, x_std=1.0, w_std=0.02, r_std=1.0)
    _check_twice(d, 8, 0.5, what=f"decode T={T}")


def test_noalloc_fused_norm_falls_back_to_separate_norm():
    """With CAAT_FLAG_FUSED_NORM, T=2048, H=4096, P=8 the fused norm's partials (8.4 MB) do not
    fit in the array: the call runs the separate norm instead and still matches."""
    d = I.make_rowpar_inputs(2048, 1024, 4096, 8, seed=23, x_std=1.0, w_std=0.05, r_std=1.0)
    _check_twice(d, 8, 0.5, flags=C.CAAT_FLAG_FUSED_NORM, what="fused fallback")


def test_noalloc_rejects_what_does_not_fit():
    """A forced decode path whose partials exceed the array (T=64, H=4096, P=8: 8 MiB) is
    rejected with CAAT_ERR_WORKSPACE and queues nothing."""
    g = to_dev(I.make_rowpar_inputs(64, 1024, 4096, 8, seed=24))
    out = torch.full_like(g["R"], 7.0)
    with pytest.raises(C.CaatError) as e:
        C.caat_rowpar_forward_noalloc(g["X"], g["W"], g["R"], g["gamma"], None, 8, 0.5, out,
                                      flags=C.CAAT_FLAG_FORCE_DECODE_PATH)
    assert e.value.code == C.CAAT_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())


def test_noalloc_rejects_invalid_like_the_workspace_entry_point():
    g = to_dev(I.make_rowpar_inputs(64, 256, 256, 2, seed=0))
    out = torch.empty_like(g["R"])
    with pytest.raises(C.CaatError) as e:
        C.caat_rowpar_forward_noalloc(g["X"], g["W"], g["R"], g["gamma"], None, 2, 1.5, out)
    assert e.value.code == C.CAAT_ERR_INVALID_ARG

"""The entry point that allocates no device memory (caat_rowpar_forward_noalloc).

It exists for callers that cannot call cudaMalloc (an embedding whose allocator belongs to
someone else, code that must not grow its memory footprint or enter an allocator in a hot
loop): its scratch is a fixed array inside the library instead of a caller-supplied
workspace.  This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it must pass alone in a fresh process too.
"""
import numpy as np
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


@pytest.mark.parametrize("T,K,H,P,p,random_idx", [(300, 800, 776, 4, 0.5, False),
                                                   (256, 1024, 1024, 4, 0.5, True),
                                                   (1024, 4096, 2048, 8, 0.75, False)])
def test_noalloc_matches_workspace_entry_point_twice(T, K, H, P, p, random_idx):
    d = I.make_rowpar_inputs(T, K, H, P, seed=21, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=2) if random_idx else None
    g = to_dev(d)
    ref = torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, ref)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    ref_cpu = ref.cpu()
    for call in range(2):   # two calls in a row share (and must re-clear) the scratch array
        out = torch.full_like(g["R"], float("nan"))
        C.caat_rowpar_forward_noalloc(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        assert_out_close(out.cpu(), ref_cpu, f"no-alloc call {call}")


def test_noalloc_rejects_invalid_like_the_workspace_entry_point():
    g = to_dev(I.make_rowpar_inputs(64, 256, 256, 2, seed=0))
    out = torch.empty_like(g["R"])
    with pytest.raises(C.CaatError) as e:
        C.caat_rowpar_forward_noalloc(g["X"], g["W"], g["R"], g["gamma"], None, 2, 1.5, out)
    assert e.value.code == C.CAAT_ERR_INVALID_ARG

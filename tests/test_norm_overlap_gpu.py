"""The row norm running beside the GEMM kernel (CAAT_FLAG_NORM_BESIDE_GEMM, CTA-pair path,
H <= 4096): the GEMM counts its finished tiles per (128-token block, rank) and the norm kernel,
launched as its programmatic dependent on the SMs the GEMM leaves free, normalizes complete
blocks while the GEMM computes the rest.  Same arithmetic as the norm kernel that runs after
the GEMM (the default), so both give the same bits; both match the float64 oracle
("Tensor-Parallelism with Partially Synchronized Activations", App. A.2 Eq. 22, §4 Eq. 9)."""
import pytest
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I

from gpu_util import assert_h_close, assert_out_close, ensure_built, run_rowpar, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _kernels_per_call(d, P, p, idx=None, flags=0):
    """Number of timed intervals the library records for one call: the overlapped GEMM + norm
    are one interval (no event may sit between them), the sequential path two."""
    g = to_dev(d)
    out = torch.empty_like(g["R"])
    tm = C.Timing(capacity=4)
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out, flags=flags, timing=tm)
    torch.cuda.synchronize()
    r = tm.read()
    tm.close()
    return len(r[0])


CASES = [
    # T, K, H, P, p, random S
    (300, 800, 776, 4, 0.5, False),      # ragged T (3 row blocks of 128), H with an 8-wide tail
    (1000, 768, 768, 2, 0.7, False),     # mixed column block at the sync boundary
    (520, 1024, 1024, 4, 0.5, True),     # every column block mixed (merge epilogue)
    (2304, 512, 1032, 4, 0.25, False),   # 9 row blocks of 256: more than the stagger distance
    (1536, 2048, 2048, 8, 1.0, False),   # all shared
    (1536, 2048, 2048, 8, 0.0, False),   # all private
    (640, 11008, 4096, 8, 0.5, False),   # the 7B FC2 shape at 640 tokens
    (257, 256, 264, 1, 0.5, False),      # one rank, one token past a pair row block
]


@pytest.mark.parametrize("T,K,H,P,p,rand", CASES)
def test_overlapped_norm_matches_sequential_and_oracle(T, K, H, P, p, rand):
    d = I.make_rowpar_inputs(T, K, H, P, seed=40 + T % 17, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=5) if rand else None
    B = C.CAAT_FLAG_NORM_BESIDE_GEMM
    assert _kernels_per_call(d, P, p, idx, B) == 1, "the overlapped norm did not run"
    assert _kernels_per_call(d, P, p, idx) == 2
    out_o, h_o = run_rowpar(d, P, p, idx, flags=B)
    out_s, h_s = run_rowpar(d, P, p, idx)
    assert torch.equal(h_o, h_s), "pre-norm stream differs"
    assert torch.equal(out_o, out_s), "overlapped norm differs from the sequential norm"
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, idx, return_all=True)
    assert_h_close(h_o, ref["h"], "h")
    assert_out_close(out_o, ref["out"], "out")


@pytest.mark.parametrize("alias", ["out=residual", "no h_out", "h_out=residual"])
def test_overlapped_norm_in_place(alias):
    """out may alias the residual and h may live in out: the norm of a row block starts only
    after every tile of that block (which reads the residual of those rows) is stored."""
    T, K, H, P, p = 700, 1024, 1024, 4, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=44, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p)
    g = to_dev(d)
    if alias == "out=residual":
        out, hb = g["R"], torch.empty_like(g["R"])
    elif alias == "no h_out":
        out, hb = torch.empty_like(g["R"]), None
    else:
        out, hb = torch.empty_like(g["R"]), g["R"]
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out, h_out=hb,
                          flags=C.CAAT_FLAG_NORM_BESIDE_GEMM)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    assert_out_close(out.cpu(), ref, alias)


def test_overlapped_norm_repeated_calls_deterministic():
    """Back-to-back calls reuse the workspace counters (cleared on the stream before each GEMM):
    every call gives the same bits, the same as the norm after the GEMM."""
    T, K, H, P, p = 1100, 1024, 2048, 4, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=45, x_std=1.0, w_std=0.05, r_std=1.0)
    g = to_dev(d)
    ws = C.alloc_workspace(C.caat_workspace_size(T, K, H, P))
    outs = []
    for _ in range(4):
        out = torch.empty_like(g["R"])
        C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out, workspace=ws,
                              flags=C.CAAT_FLAG_NORM_BESIDE_GEMM)
        outs.append(out)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    ref_out, _ = run_rowpar(d, P, p, h_out=False)
    assert torch.equal(outs[0].cpu(), ref_out)


def test_minimal_workspace_runs_norm_after_gemm():
    """A workspace of only the 256-byte counter block has no room for the tile counters: the
    norm runs after the GEMM (two recorded kernels) even when asked to run beside it, with the
    same result."""
    T, K, H, P, p = 600, 1024, 1024, 4, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=46, x_std=1.0, w_std=0.05, r_std=1.0)
    g = to_dev(d)
    ws = C.alloc_workspace(256)
    out = torch.empty_like(g["R"])
    tm = C.Timing(capacity=2)
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out, workspace=ws, timing=tm,
                          flags=C.CAAT_FLAG_NORM_BESIDE_GEMM)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    assert len(tm.read()[0]) == 2
    out_full, _ = run_rowpar(d, P, p, h_out=False)
    assert torch.equal(out.cpu(), out_full)

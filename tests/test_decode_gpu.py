"""GPU parity of the decode path (T <= 64: weight-streaming partial products, then the
cluster kernel for the partial channel-reduce, residual and RMSNorm) against the oracle, and
agreement with the tensor-core GEMM path on the same inputs."""
import math

import numpy as np
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


@pytest.mark.parametrize("T,K,H,P,p", [(1, 1024, 512, 8, 0.5), (5, 800, 776, 4, 0.7), (8, 2048, 1024, 2, 0.25),
                                       (33, 512, 264, 16, 0.5), (64, 1376 * 2, 1032, 2, 1.0), (17, 256, 256, 1, 0.0)])
def test_decode_matches_oracle(T, K, H, P, p):
    d = I.make_rowpar_inputs(T, K, H, P, seed=T * 7 + P, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    out, h = run_rowpar(d, P, p, flags=C.CAAT_FLAG_FORCE_DECODE_PATH)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
    assert_h_close(h, ref["h"], f"decode h T={T}")
    assert_out_close(out, ref["out"], f"decode T={T} K={K} H={H} P={P} p={p}")


def test_decode_random_sync_idx_scale_eps():
    d = I.make_rowpar_inputs(8, 1024, 1024, 4, seed=11, x_std=1.0, w_std=0.05, r_std=1.0)
    idx = I.random_sync_idx(1024, O.n_sync(1024, 0.5), seed=9)
    out, _ = run_rowpar(d, 4, 0.5, idx, private_scale=2.0, eps=1e-3)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 4, 0.5, idx, private_scale=2.0, eps=1e-3)
    assert_out_close(out, ref, "decode random S")


@pytest.mark.parametrize("T", [1, 8, 64])
def test_decode_agrees_with_gemm_path(T):
    d = I.make_rowpar_inputs(T, 2048, 1024, 8, seed=T, x_std=1.0, w_std=0.05, r_std=1.0)
    o_dec, h_dec = run_rowpar(d, 8, 0.5)
    o_gem, h_gem = run_rowpar(d, 8, 0.5, flags=C.CAAT_FLAG_FORCE_GEMM_PATH)
    # both are within the oracle tolerance; against each other they differ only by fp32
    # summation order and bf16 rounding
    assert_out_close(o_dec, o_gem.double(), f"decode vs gemm T={T}")


def test_decode_integer_construction_bit_exact():
    P, T, H, Kp = 4, 3, 520, 16
    X = torch.zeros(P, T, Kp, dtype=torch.bfloat16)
    W = torch.zeros(P, H, Kp, dtype=torch.bfloat16)
    a = torch.tensor([1.0 + (t % 4) for t in range(T)])
    for m in range(P):
        X[m, :, 5] = a
        W[m, :, 5] = float(2 ** m)
    d = {"X": X, "W": W, "R": torch.zeros(P, T, H, dtype=torch.bfloat16), "gamma": torch.ones(H, dtype=torch.bfloat16)}
    for p in (0.5, 0.3):
        _, h = run_rowpar(d, P, p)
        mask = O.sync_mask(H, p)
        for m in range(P):
            want = np.where(mask[None, :], (2 ** P - 1) * a.numpy()[:, None], (2 ** m) * a.numpy()[:, None])
            np.testing.assert_array_equal(h[m].double().numpy(), want)


@pytest.mark.parametrize("T", [1, 64])
def test_decode_repeat_and_in_place(T):
    """Back-to-back decode calls (the reduce kernel is a programmatic dependent of the
    partials kernel) give identical bits, and normalizing h in place (no h_out) gives the same
    out as with a separate h buffer."""
    P, K, H = 8, 2048, 1032
    d = I.make_rowpar_inputs(T, K, H, P, seed=40 + T, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    o1, h1 = run_rowpar(d, P, 0.5)
    o2, h2 = run_rowpar(d, P, 0.5)
    o3, _ = run_rowpar(d, P, 0.5, h_out=False)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    assert torch.equal(o1, o3)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, 0.5)
    assert_out_close(o1, ref, f"decode T={T}")


@pytest.mark.parametrize("T", [1, 64, 300])
def test_call_captured_in_cuda_graph(T):
    """One call of the device entry point captured in a CUDA graph (decode path: the reduce
    kernel's programmatic-dependent launch becomes a graph edge; GEMM path at T=300: the
    counter memset becomes a memset node) replays to the same bits as the eager call."""
    P, K, H = 8, 2048, 1032
    d = I.make_rowpar_inputs(T, K, H, P, seed=50 + T, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    o_ref, h_ref = run_rowpar(d, P, 0.5)
    g = to_dev(d)
    out = torch.empty_like(g["R"])
    hb = torch.empty_like(g["R"])
    ws = C.alloc_workspace(C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR))
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, 0.5, out, h_out=hb, workspace=ws)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, 0.5, out, h_out=hb, workspace=ws,
                              stream=torch.cuda.current_stream())
    for _ in range(2):
        out.zero_()
        hb.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        assert torch.equal(out.cpu(), o_ref) and torch.equal(hb.cpu(), h_ref)
    del graph


@pytest.mark.parametrize("T,rand", [(1, False), (300, False), (300, True)])
def test_plan_execute_matches_forward_and_captures(T, rand):
    """A plan (buffers bound once) gives the forward call's bits, again after its buffers'
    contents change, and inside a CUDA graph; with a random sync list also on permuted W."""
    P, K, H, p = 4, 1024, 1032, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=60 + T, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=3) if rand else None
    g = to_dev(d)
    flags = 0
    if rand:
        Wp = torch.empty_like(g["W"])
        C.caat_permute_weights(g["W"], Wp, idx, P, p)
        g["W"], flags = Wp, C.CAAT_FLAG_W_PERMUTED
    ref_out, ref_h = torch.empty_like(g["R"]), torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, ref_out, h_out=ref_h, flags=flags)
    out, hb = torch.empty_like(g["R"]), torch.empty_like(g["R"])
    plan = C.Plan(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out, h_out=hb, flags=flags)
    plan.execute()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(hb, ref_h)
    # new contents in the bound buffers
    g["X"].copy_(torch.flip(g["X"], dims=[1]))
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, ref_out, h_out=ref_h, flags=flags)
    plan.execute()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(hb, ref_h)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        plan.execute(stream=torch.cuda.current_stream())
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    assert torch.equal(out, ref_out)
    del graph
    plan.close()
    ref = O.rowpar_forward(d["X"].flip(1), d["W"], d["R"], d["gamma"], P, p, idx)
    assert_out_close(out.cpu(), ref, "plan")

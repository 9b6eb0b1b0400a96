"""The largest shapes each path accepts: hidden size CAAT_MAX_H = 65536 and CAAT_MAX_P = 64 ranks
on the GEMM path, H = 8192 with P = 16 on the decode path and the backward."""
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


@pytest.mark.parametrize("rand", [False, True])
def test_max_hidden_size(rand):
    """H = 65536 (256 column blocks, the two-pass norm), T = 300 (ragged pair tiles)."""
    T, K, H, P, p = 300, 256, 65536, 2, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=7, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=1) if rand else None
    out, h = run_rowpar(d, P, p, idx)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, idx, return_all=True)
    assert_h_close(h, ref["h"], "h H=65536")
    assert_out_close(out, ref["out"], "H=65536")


def test_max_ranks():
    """P = 64 ranks with K/P = 8 (one 16-wide MMA step per rank, zero-filled), p = 0.3."""
    T, K, H, P, p = 300, 512, 520, 64, 0.3
    d = I.make_rowpar_inputs(T, K, H, P, seed=8, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    out, h = run_rowpar(d, P, p)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
    assert_h_close(h, ref["h"], "h P=64")
    assert_out_close(out, ref["out"], "P=64")


@pytest.mark.parametrize("T", [1, 64])
def test_decode_limits(T):
    """The decode path at its limits: H = 8192, P = 16."""
    K, H, P, p = 2048, 8192, 16, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=9, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    out, h = run_rowpar(d, P, p, flags=C.CAAT_FLAG_FORCE_DECODE_PATH)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
    assert_h_close(h, ref["h"], f"decode h T={T}")
    assert_out_close(out, ref["out"], f"decode T={T} H=8192 P=16")


def test_backward_limits():
    """The backward at its limits: H = 8192, P = 16 (the shared-memory norm backward holds
    P H 4 = 512 KB > its staging budget, so the kernel that re-reads the token from cache runs)."""
    T, K, H, P, p = 130, 512, 8192, 16, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=10, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    g = to_dev(d)
    out, h = torch.empty_like(g["R"]), torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out, h_out=h)
    dout = torch.randn(P, T, H, generator=torch.Generator().manual_seed(11)).to(torch.bfloat16).cuda()
    dX, dW, dR = torch.empty_like(g["X"]), torch.empty_like(g["W"]), torch.empty_like(g["R"])
    dg = torch.empty(H, dtype=torch.float32, device="cuda")
    C.caat_rowpar_backward(g["X"], g["W"], h, g["gamma"], dout, None, P, p, dX, dW, dg, dR=dR)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    ref = O.rowpar_backward(d["X"], d["W"], h.cpu(), d["gamma"], dout.cpu(), P, p)
    for name, got, rel in (("dR", dR, 8e-3), ("dgamma", dg, 1e-3)):
        r = ref[name]
        err = np.abs(O._f64(got.cpu()) - r)
        assert (err <= rel * np.abs(r) + 2e-3 * np.sqrt(np.mean(r * r))).all(), name
    for name, got, sq in (("dX", dX, np.stack([(ref["dZt"][m] ** 2) @ (O._f64(d["W"][m]) ** 2) for m in range(P)])),
                          ("dW", dW, np.stack([(ref["dZt"][m] ** 2).T @ (O._f64(d["X"][m]) ** 2) for m in range(P)]))):
        err = np.abs(O._f64(got.cpu()) - ref[name])
        assert (err <= 8e-3 * np.sqrt(sq) + 4e-3 * np.abs(ref[name]) + 1e-6).all(), name


@pytest.mark.parametrize("H", [8192, 12288, 24576])
def test_wide_rows_norm(H):
    """H > 4096: the norm runs one CTA per row (256, 512 or 1024 threads) with the row in
    registers; ragged T, contiguous and listed sync sets."""
    T, K, P, p = 300, 256, 2, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=H, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    for idx in (None, I.random_sync_idx(H, O.n_sync(H, p), seed=2)):
        out, h = run_rowpar(d, P, p, idx)
        ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, idx, return_all=True)
        assert_h_close(h, ref["h"], f"h H={H}")
        assert_out_close(out, ref["out"], f"H={H}")

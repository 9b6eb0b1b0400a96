"""Parity at the full workload sizes, in the launch configuration the bench times, checked on
sampled token rows against the float64 oracle (rows are independent through the path)."""
import numpy as np
import pytest
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I

from gpu_util import assert_out_close, ensure_built, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


@pytest.fixture(scope="module")
def fc2_7b():
    return I.make_rowpar_inputs(8192, 11008, 4096, 8, seed=1000, x_std=1.0, w_std=0.02, r_std=1.0)


def _run(g, P, p, idx=None, flags=0):
    out = torch.empty_like(g["R"])
    ws = C.alloc_workspace(C.caat_workspace_size(g["X"].shape[1], g["X"].shape[2] * P, g["W"].shape[1], P))
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    return out.cpu()


@pytest.mark.parametrize("p", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_fc2_7b_p_sweep_sampled(fc2_7b, p):
    g = to_dev(fc2_7b)
    out = _run(g, 8, p)
    rows = I.sample_rows(8192, 128, seed=int(p * 100))
    ref = O.rowpar_rows(fc2_7b["X"], fc2_7b["W"], fc2_7b["R"], fc2_7b["gamma"], 8, p, rows)
    assert_out_close(out[:, torch.as_tensor(rows), :], ref, f"fc2-7b p={p}")


def test_fc2_7b_fused_norm_sampled(fc2_7b):
    g = to_dev(fc2_7b)
    out = _run(g, 8, 0.5, flags=C.CAAT_FLAG_FUSED_NORM)
    rows = I.sample_rows(8192, 128, seed=7)
    ref = O.rowpar_rows(fc2_7b["X"], fc2_7b["W"], fc2_7b["R"], fc2_7b["gamma"], 8, 0.5, rows)
    assert_out_close(out[:, torch.as_tensor(rows), :], ref, "fc2-7b fused")


def test_fc2_1b_random_sync_idx_full():
    """The 1.1B FC2 workload (T=4096, H=2048, K=5632, P=4, p=0.5, seeded random S), compared on
    every element (the float64 oracle runs it in seconds)."""
    d = I.make_rowpar_inputs(4096, 5632, 2048, 4, seed=2000, x_std=1.0, w_std=0.02, r_std=1.0)
    idx = I.random_sync_idx(2048, O.n_sync(2048, 0.5), seed=0)
    out = _run(to_dev(d), 4, 0.5, idx)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 4, 0.5, idx)
    assert_out_close(out, ref, "fc2-1b random S")
    # the channel-permuted path on the same inputs (W permuted once, as the bench does)
    g = to_dev(d)
    Wp = torch.empty_like(g["W"])
    C.caat_permute_weights(g["W"], Wp, idx, 4, 0.5)
    g["W"] = Wp
    out_p = _run(g, 4, 0.5, idx, flags=C.CAAT_FLAG_W_PERMUTED)
    assert_out_close(out_p, ref, "fc2-1b random S, permuted W")


@pytest.mark.parametrize("T", [1, 8, 64])
def test_decode_shapes_full(T):
    """Decode-shaped calls: T in {1, 8, 64} tokens at H=4096, K=11008, P=8, p=0.5."""
    d = I.make_rowpar_inputs(T, 11008, 4096, 8, seed=3000 + T, x_std=1.0, w_std=0.02, r_std=1.0)
    out = _run(to_dev(d), 8, 0.5)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 8, 0.5)
    assert_out_close(out, ref, f"decode T={T}")


def test_attention_out_projection_7b_sampled():
    """The attention output projection of App. A.1 Eq. 24 is the same row-parallel layer with
    X_m = rank m's head outputs and K = heads x head_dim: Llama-2-7B shape (32 heads of 128,
    4 per rank), T = 8192, H = 4096, P = 8, p = 0.5, checked on sampled rows."""
    d = I.make_rowpar_inputs(8192, 4096, 4096, 8, seed=4000, x_std=1.0, w_std=0.02, r_std=1.0)
    out = _run(to_dev(d), 8, 0.5)
    rows = I.sample_rows(8192, 128, seed=11)
    ref = O.rowpar_rows(d["X"], d["W"], d["R"], d["gamma"], 8, 0.5, rows)
    assert_out_close(out[:, torch.as_tensor(rows), :], ref, "attention out-projection 7B")

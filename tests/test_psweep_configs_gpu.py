"""Every workload at its own shape over the sync factors p in {0, 0.25, 0.5, 0.75, 1} against the
float64 oracle ("Tensor-Parallelism with Partially Synchronized Activations", App. A.2 Eq. 22,
§4 Eq. 9; the MLP block §3.1 Eq. 6): the tiny sanity shape, the 1.1B FC2 (seeded random sync
list, plain and channel-permuted W), the 7B MLP block (128 sampled token rows per p) and the
decode shapes T in {1, 8, 64}.  The 7B FC2 sweep is in test_fullsize_gpu.py."""
import pytest
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I

from gpu_util import assert_out_close, ensure_built, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

P_SWEEP = [0.0, 0.25, 0.5, 0.75, 1.0]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _rowpar(g, P, p, idx=None, flags=0):
    T, K, H = g["X"].shape[1], g["X"].shape[2] * P, g["W"].shape[1]
    out = torch.empty_like(g["R"])
    ws = C.alloc_workspace(C.caat_workspace_size(T, K, H, P))
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    return out.cpu()


@pytest.mark.parametrize("p", P_SWEEP)
def test_tiny_p_sweep(p):
    """T=256, K=H=768, P=2; X, W ~ N(0,0.02), R ~ N(0,1), gamma=1; and with R = 0, gamma ~ U(0.5,1.5)
    (the residual no longer dominates, so the GEMM decides the output)."""
    for seed, r_std, gamma in ((0, 1.0, "ones"), (1, 0.0, "uniform")):
        d = I.make_rowpar_inputs(256, 768, 768, 2, seed=seed, x_std=0.02, w_std=0.02, r_std=r_std, gamma=gamma)
        out = _rowpar(to_dev(d), 2, p)
        ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 2, p)
        assert_out_close(out, ref, f"tiny p={p} r_std={r_std}")


@pytest.fixture(scope="module")
def fc2_1b():
    return I.make_rowpar_inputs(4096, 5632, 2048, 4, seed=2000, x_std=1.0, w_std=0.02, r_std=1.0)


@pytest.mark.parametrize("p", P_SWEEP)
def test_fc2_1b_p_sweep_full(fc2_1b, p):
    """T=4096, H=2048, K=5632, P=4, a seeded random sync list of floor(2048 p) channels; every
    element, on the original W (mixed column blocks) and on W permuted once for the list."""
    d = fc2_1b
    idx = I.random_sync_idx(2048, O.n_sync(2048, p), seed=0)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 4, p, idx)
    g = to_dev(d)
    assert_out_close(_rowpar(g, 4, p, idx), ref, f"fc2-1b p={p}")
    Wp = torch.empty_like(g["W"])
    C.caat_permute_weights(g["W"], Wp, idx, 4, p)
    g["W"] = Wp
    assert_out_close(_rowpar(g, 4, p, idx, flags=C.CAAT_FLAG_W_PERMUTED), ref, f"fc2-1b p={p} permuted W")


@pytest.fixture(scope="module")
def mlp_7b():
    return I.make_mlp_inputs(4096, 4096, 11008, 8, seed=4, x_std=1.0, w_std=0.02, r_std=1.0)


@pytest.mark.parametrize("p", P_SWEEP)
def test_mlp_7b_p_sweep_sampled(mlp_7b, p):
    """The 7B MLP block (T=4096, H=4096, F=11008, P=8) at full size, 128 sampled token rows."""
    d = mlp_7b
    g = to_dev(d)
    out = torch.empty_like(g["R"])
    C.caat_mlp_forward(g["X"], g["A"], g["W2"], g["R"], g["gamma"], None, 8, p, out)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    rows = I.sample_rows(4096, 128, seed=int(p * 100) + 3)
    ref = O.mlp_rows(d["X"], d["A"], d["W2"], d["R"], d["gamma"], 8, p, rows)
    assert_out_close(out.cpu()[:, torch.as_tensor(rows), :], ref, f"mlp-7b p={p}")


@pytest.mark.parametrize("T", [1, 8, 64])
@pytest.mark.parametrize("p", P_SWEEP)
def test_decode_p_sweep_full(T, p):
    """Decode shapes (H=4096, K=11008, P=8) over p, every element."""
    d = I.make_rowpar_inputs(T, 11008, 4096, 8, seed=3000 + T, x_std=1.0, w_std=0.02, r_std=1.0)
    out = _rowpar(to_dev(d), 8, p)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 8, p)
    assert_out_close(out, ref, f"decode T={T} p={p}")

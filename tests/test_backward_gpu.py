"""GPU parity of the layer's backward (caat_rowpar_backward) against the oracle's
rowpar_backward, on the pre-norm stream h the GPU forward produced (both sides start from the
same bf16 h, X, W, gamma and dout).

Tolerances, from the arithmetic: dR is dh rounded to bf16 (relative 2^-9) from fp32 math on
exact inputs: |err| <= 8e-3 |ref| + 2e-3 rms(ref).  dX and dW are GEMMs of dZt rounded to bf16
(each element off by at most 2^-9 relative, uniformly: standard deviation <= 2^-9/sqrt(3)
|dZt|), with fp32 accumulation and a bf16 output: for C = sum_j A_j B_j the error has standard
deviation <= 1.13e-3 sqrt(sum_j A_j^2 B_j^2), so each element is checked against
8e-3 sqrt(sum_j A_j^2 B_j^2) (about 7 standard deviations) + 4e-3 |ref| (output rounding).
dgamma is an fp32 sum over the ranks and tokens: |err| <= 1e-3 (rms(ref) + |ref|)."""
import numpy as np
import pytest
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I

from gpu_util import ensure_built, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _close(got, ref, rel, atol_rms, what):
    got = O._f64(got)
    ref = O._f64(ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(got - ref)
    bound = rel * np.abs(ref) + atol_rms * rms
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {err.size} out of bound, max err {err.max():.3e}, rms {rms:.3e}"


def _close_gemm(got, ref, sq_scale, what):
    """|got - ref| <= 8e-3 sqrt(sq_scale) + 4e-3 |ref|, sq_scale = sum_j A_j^2 B_j^2 per element."""
    got = O._f64(got)
    bound = 8e-3 * np.sqrt(sq_scale) + 4e-3 * np.abs(ref) + 1e-6
    err = np.abs(got - ref)
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {err.size} out of bound, max err/bound {float((err / bound).max()):.3f}"


def _setup(T, K, H, P, p, idx, seed, private_scale=1.0, eps=1e-5):
    d = I.make_rowpar_inputs(T, K, H, P, seed=seed, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    g = to_dev(d)
    out = torch.empty_like(g["R"])
    h = torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out, h_out=h, eps=eps,
                          private_scale=private_scale)
    dout = torch.randn(P, T, H, generator=torch.Generator().manual_seed(seed + 1)).to(torch.bfloat16)
    g["h"], g["dout"] = h, dout.cuda()
    return d, g


def _backward(g, P, p, idx, private_scale=1.0, eps=1e-5, with_dR=True):
    X, W = g["X"], g["W"]
    dX, dW = torch.empty_like(X), torch.empty_like(W)
    dR = torch.empty_like(g["R"]) if with_dR else None
    dgamma = torch.empty(W.shape[1], dtype=torch.float32, device="cuda")
    C.caat_rowpar_backward(X, W, g["h"], g["gamma"], g["dout"], idx, P, p, dX, dW, dgamma, dR=dR,
                           private_scale=private_scale, eps=eps)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    return dX.cpu(), dW.cpu(), (dR.cpu() if dR is not None else None), dgamma.cpu()


@pytest.mark.parametrize("T,K,H,P,p,rand", [
    (1, 1024, 776, 4, 0.5, False), (37, 1024, 776, 4, 0.3, True), (300, 2048, 1288, 4, 0.5, False),
    (600, 1024, 776, 2, 0.0, False), (257, 1024, 520, 8, 1.0, False), (130, 512, 1032, 16, 0.5, True),
    # H % 16 == 0 and few tokens (fewer tokens than CTAs in the first)
    (5, 1024, 1024, 4, 0.5, True), (300, 2048, 2048, 8, 0.25, False), (200, 512, 1024, 16, 0.5, False)])
def test_backward_matches_oracle(T, K, H, P, p, rand):
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=T) if rand else None
    s = 1.5 if rand else 1.0
    d, g = _setup(T, K, H, P, p, idx, seed=100 + T, private_scale=s)
    dX, dW, dR, dgamma = _backward(g, P, p, idx, private_scale=s)
    ref = O.rowpar_backward(d["X"], d["W"], g["h"].cpu(), d["gamma"], g["dout"].cpu(), P, p, idx,
                            private_scale=s)
    _close(dR, ref["dR"], 8e-3, 2e-3, f"dR T={T}")
    Z2, X2, W2 = ref["dZt"] ** 2, O._f64(d["X"]) ** 2, O._f64(d["W"]) ** 2
    _close_gemm(dX, ref["dX"], np.stack([Z2[m] @ W2[m] for m in range(P)]), f"dX T={T}")
    _close_gemm(dW, ref["dW"], np.stack([Z2[m].T @ X2[m] for m in range(P)]), f"dW T={T}")
    _close(dgamma, ref["dgamma"], 1e-3, 1e-3, f"dgamma T={T}")


def test_backward_deterministic_and_dR_optional():
    T, K, H, P, p = 300, 1024, 776, 4, 0.5
    _, g = _setup(T, K, H, P, p, None, seed=7)
    a = _backward(g, P, p, None)
    b = _backward(g, P, p, None, with_dR=False)
    c = _backward(g, P, p, None)
    for x, y in zip(a, c):
        assert torch.equal(x, y)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[3], b[3])


def test_backward_full_size_fc2_7b_sampled():
    """fc2-7b shape (T=8192, H=4096, K=11008, P=8, p=0.5): dR, dgamma on every element; dX
    and dW rows checked on samples against the oracle's formulas restricted to them."""
    T, K, H, P, p = 8192, 11008, 4096, 8, 0.5
    d, g = _setup(T, K, H, P, p, None, seed=9)
    dX, dW, dR, dgamma = _backward(g, P, p, None)
    h = g["h"].cpu()
    dout = g["dout"].cpu()
    rows = I.sample_rows(T, 16, seed=3)
    rows_t = torch.as_tensor(rows)
    # dh / dZt of the sampled tokens (tokens are independent through the norm and the reduce)
    dh, _ = O.rmsnorm_backward(O._f64(h[:, rows_t]), d["gamma"], O._f64(dout[:, rows_t]), 1e-5)
    _close(dR[:, rows_t], dh, 8e-3, 2e-3, "dR sampled")
    mask = O.sync_mask(H, p)
    dZt = O.partial_channel_reduce_backward(dh, mask)
    Wf = O._f64(d["W"])
    dX_ref = np.stack([dZt[m] @ Wf[m] for m in range(P)])
    _close_gemm(dX[:, rows_t], dX_ref, np.stack([(dZt[m] ** 2) @ (Wf[m] ** 2) for m in range(P)]), "dX sampled")
    # dW rows (channels) need every token: a few channels in float64, rank by rank (memory)
    chans = np.array([0, 1, 2047, 2048, 4095])
    dh_c = np.zeros((P, T, len(chans)))
    dg_ref = np.zeros(H)
    for q in range(P):
        dh_q, dg_q = O.rmsnorm_backward(O._f64(h[q]), d["gamma"], O._f64(dout[q]), 1e-5)
        dh_c[q] = dh_q[:, chans]
        dg_ref += dg_q.sum(axis=0)
    dZt_c = O.partial_channel_reduce_backward(dh_c, mask[chans])
    Xf = O._f64(d["X"])
    dW_ref = np.stack([dZt_c[m].T @ Xf[m] for m in range(P)])
    dW_sq = np.stack([(dZt_c[m] ** 2).T @ (Xf[m] ** 2) for m in range(P)])
    _close_gemm(dW[:, torch.as_tensor(chans)], dW_ref, dW_sq, "dW sampled channels")
    _close(dgamma, dg_ref, 1e-3, 1e-3, "dgamma")


@pytest.mark.parametrize("T,K,H,P,p,rand", [(300, 2048, 1288, 4, 0.5, False), (600, 1024, 776, 2, 0.0, False),
                                            (2048, 5632, 2048, 4, 0.5, True)])
def test_backward_mn_major_equals_transposed_bitwise(T, K, H, P, p, rand):
    """The gradient GEMMs reading W, dZt and X in place (MN-major) give the same bits as the
    same GEMMs on transposed K-major copies: identical MMA steps on identical values."""
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=T) if rand else None
    _, g = _setup(T, K, H, P, p, idx, seed=200 + T)
    outs = []
    for flags in (0, C.CAAT_BWD_FLAG_TRANSPOSED_OPERANDS):
        X, W = g["X"], g["W"]
        dX, dW = torch.empty_like(X), torch.empty_like(W)
        dR = torch.empty_like(g["R"])
        dgamma = torch.empty(H, dtype=torch.float32, device="cuda")
        C.caat_rowpar_backward(X, W, g["h"], g["gamma"], g["dout"], idx, P, p, dX, dW, dgamma, dR=dR, flags=flags)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        outs.append((dX, dW, dR, dgamma))
    for name, a, b in zip(("dX", "dW", "dR", "dgamma"), outs[0], outs[1]):
        assert torch.equal(a, b), name

"""GPU parity of the channel-permuted path (caat_permute_weights + CAAT_FLAG_W_PERMUTED): a
sync set given as an arbitrary sorted list is made contiguous by permuting W's output
channels; the norm kernel restores the original channel order.  Compared with the oracle on
the original (unpermuted) weights."""
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


def _perm(H, p, idx):
    """perm(i): shared channels ascending, then private channels ascending (numpy)."""
    mask = O.sync_mask(H, p, idx)
    return np.concatenate([np.nonzero(mask)[0], np.nonzero(~mask)[0]])


def _permuted_W(g, P, p, idx):
    Wp = torch.empty_like(g["W"])
    C.caat_permute_weights(g["W"], Wp, idx, P, p)
    return Wp


def _run(g, Wp, P, p, idx, *, h_mode="separate", out_alias_residual=False, private_scale=1.0, eps=1e-5,
         flags=0):
    R = g["R"].clone()
    out = R if out_alias_residual else torch.empty_like(R)
    if h_mode == "separate":
        hb = torch.empty_like(R)
    elif h_mode == "residual":
        hb = R
    else:
        hb = None
    C.caat_rowpar_forward(g["X"], Wp, R, g["gamma"], idx, P, p, out, h_out=hb, private_scale=private_scale,
                          eps=eps, flags=C.CAAT_FLAG_W_PERMUTED | flags)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    return out.cpu(), (hb.cpu() if hb is not None else None)


def _assert_h_permuted(got, ref_all, what):
    """h on the permuted path: Z' is rounded to bf16 before the residual add and h after it,
    so |err| <= 2^-9 (|Z| + |h|) plus fp32 accumulation; checked with twice that margin."""
    got = O._f64(got)
    h = ref_all["h"]
    Z = ref_all["Z"]
    rms = np.sqrt(np.mean(h * h, axis=-1, keepdims=True))
    bound = 4e-3 * (np.abs(Z) + np.abs(h)) + 2e-3 * rms
    bad = np.abs(got - h) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of bound"


def test_permute_weights_matches_definition():
    P, H, Kp = 4, 776, 200
    W = torch.randn(P, H, Kp, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    for p, idx in [(0.5, I.random_sync_idx(H, O.n_sync(H, 0.5), seed=1)), (0.3, None), (0.0, None), (1.0, None)]:
        Wp = torch.empty_like(W).cuda()
        C.caat_permute_weights(W.cuda(), Wp, idx, P, p)
        torch.cuda.synchronize()
        perm = _perm(H, p, idx)
        assert torch.equal(Wp.cpu(), W[:, torch.from_numpy(perm)]), f"p={p}"


@pytest.mark.parametrize("T", [1, 8, 100, 300, 600])
@pytest.mark.parametrize("p,H", [(0.5, 1288), (0.3, 776)])
def test_permuted_forward_matches_oracle(T, p, H):
    """T = 1, 8: decode path; 100: single-CTA GEMM; 300, 600: CTA-pair GEMM (ragged)."""
    P, K = 4, 1024
    d = I.make_rowpar_inputs(T, K, H, P, seed=60 + T, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=T)
    g = to_dev(d)
    Wp = _permuted_W(g, P, p, idx)
    out, h = _run(g, Wp, P, p, idx, private_scale=0.75)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, sync_idx=idx, private_scale=0.75,
                           return_all=True)
    _assert_h_permuted(h, ref, f"h T={T} p={p}")
    assert_out_close(out, ref["out"], f"out T={T} p={p}")


@pytest.mark.parametrize("T", [8, 300])
def test_permuted_output_buffers(T):
    """Z' lands in h_out (distinct from residual) or in out; h_out may alias the residual and
    out may alias the residual when h_out is separate: every arrangement gives the same bits."""
    P, K, H, p = 4, 1024, 776, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=70 + T, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=2)
    g = to_dev(d)
    Wp = _permuted_W(g, P, p, idx)
    o_sep, h_sep = _run(g, Wp, P, p, idx, h_mode="separate")
    o_none, _ = _run(g, Wp, P, p, idx, h_mode="none")
    o_res, h_res = _run(g, Wp, P, p, idx, h_mode="residual")
    o_alias, h_alias = _run(g, Wp, P, p, idx, h_mode="separate", out_alias_residual=True)
    for o in (o_none, o_res, o_alias):
        assert torch.equal(o, o_sep)
    assert torch.equal(h_res, h_sep) and torch.equal(h_alias, h_sep)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, sync_idx=idx)
    assert_out_close(o_sep, ref, "buffers")


@pytest.mark.parametrize("T", [3, 100, 130])
def test_permuted_integer_construction_bit_exact(T):
    """partial_m[t, c] = 2^m a(t) through the permuted path: shared channels read exactly
    (2^P - 1) a(t), private channels of rank m exactly 2^m a(t) (exact in bf16, so Z'
    rounding changes nothing)."""
    P, H, Kp = 4, 520, 16
    X = torch.zeros(P, T, Kp, dtype=torch.bfloat16)
    W = torch.zeros(P, H, Kp, dtype=torch.bfloat16)
    a = torch.tensor([1.0 + (t % 4) for t in range(T)])
    for m in range(P):
        X[m, :, 3] = a
        W[m, :, 3] = float(2 ** m)
    d = {"X": X, "W": W, "R": torch.zeros(P, T, H, dtype=torch.bfloat16), "gamma": torch.ones(H, dtype=torch.bfloat16)}
    g = to_dev(d)
    for p, seed in ((0.5, 1), (0.3, 2)):
        idx = I.random_sync_idx(H, O.n_sync(H, p), seed=seed)
        Wp = _permuted_W(g, P, p, idx)
        _, h = _run(g, Wp, P, p, idx)
        mask = O.sync_mask(H, p, idx)
        hv = h.double().numpy()
        for m in range(P):
            want = np.where(mask[None, :], (2 ** P - 1) * a.numpy()[:, None], (2 ** m) * a.numpy()[:, None])
            np.testing.assert_array_equal(hv[m], want)


def test_permuted_contiguous_set_is_identity():
    """With the first n_s channels shared the permutation is the identity: W_out == W, and the
    permuted call agrees with the plain call within the tolerance (Z' rounding only)."""
    P, T, K, H, p = 4, 300, 1024, 776, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=80, x_std=1.0, w_std=0.05, r_std=1.0)
    g = to_dev(d)
    Wp = _permuted_W(g, P, p, None)
    torch.cuda.synchronize()
    assert torch.equal(Wp, g["W"])
    o_perm, _ = _run(g, Wp, P, p, None)
    out = torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out)
    torch.cuda.synchronize()
    assert_out_close(o_perm, out.cpu().double(), "permuted vs plain")


def test_permuted_unsupported_combinations():
    P, T, K, H, p = 2, 300, 512, 776, 0.5
    d = to_dev(I.make_rowpar_inputs(T, K, H, P, seed=81))
    out = torch.empty_like(d["R"])
    with pytest.raises(C.CaatError) as e:
        C.caat_rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], None, P, p, out,
                              flags=C.CAAT_FLAG_W_PERMUTED | C.CAAT_FLAG_FUSED_NORM)
    assert e.value.code == C.CAAT_ERR_UNSUPPORTED
    with pytest.raises(C.CaatError) as e:   # Z' would overwrite the residual
        C.caat_rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], None, P, p, d["R"], flags=C.CAAT_FLAG_W_PERMUTED)
    assert e.value.code == C.CAAT_ERR_UNSUPPORTED
    d2 = to_dev(I.make_rowpar_inputs(T, K, 4104, P, seed=82))
    with pytest.raises(C.CaatError) as e:   # GEMM path: H <= 4096
        C.caat_rowpar_forward(d2["X"], d2["W"], d2["R"], d2["gamma"], None, P, p, torch.empty_like(d2["R"]),
                              flags=C.CAAT_FLAG_W_PERMUTED)
    assert e.value.code == C.CAAT_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0


def test_permuted_host_entry_matches_device_entry():
    """caat_rowpar_forward_host with the permuted W and flag gives the device entry's bits."""
    P, T, K, H, p = 4, 1300, 1024, 776, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=90, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=4)
    g = to_dev(d)
    Wp = _permuted_W(g, P, p, idx)
    out_dev, h_dev = _run(g, Wp, P, p, idx)
    hX, hR, hg = (d[k].contiguous().pin_memory() for k in ("X", "R", "gamma"))
    hW = Wp.cpu().pin_memory()
    hout = torch.empty(P, T, H, dtype=torch.bfloat16).pin_memory()
    hh = torch.empty(P, T, H, dtype=torch.bfloat16).pin_memory()
    ws = C.alloc_workspace(C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR_HOST))
    C.caat_rowpar_forward_host(hX, hW, hR, hg, idx, P, p, hout, ws, h_out=hh, flags=C.CAAT_FLAG_W_PERMUTED)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    assert torch.equal(hout, out_dev) and torch.equal(hh, h_dev)

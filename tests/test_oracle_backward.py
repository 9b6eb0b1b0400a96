"""Pins of the oracle's backward (rowpar_backward) against central finite differences of the
oracle's own forward on tiny shapes, plus special cases.  No GPU."""
import numpy as np
import pytest

from oracle import caat_oracle as O


def _loss(X, W, R, gamma, G, P, p, idx, eps, s):
    return float(np.sum(O.rowpar_forward(X, W, R, gamma, P, p, idx, eps=eps, private_scale=s) * G))


def _fd(f, A, step=1e-6):
    g = np.zeros_like(A)
    it = np.nditer(A, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        a0 = A[i]
        A[i] = a0 + step
        up = f()
        A[i] = a0 - step
        dn = f()
        A[i] = a0
        g[i] = (up - dn) / (2 * step)
    return g


@pytest.mark.parametrize("P,T,Kp,H,p,idx,s", [
    (2, 3, 4, 6, 0.5, None, 1.0),
    (3, 2, 3, 8, 0.375, [1, 4, 6], 1.7),
    (2, 2, 2, 5, 0.0, None, 1.0),
    (2, 2, 3, 5, 1.0, None, 1.0),
    (1, 3, 2, 4, 0.5, None, 1.0),
])
def test_backward_matches_finite_differences(P, T, Kp, H, p, idx, s):
    rng = np.random.default_rng(P * 100 + H)
    X = rng.standard_normal((P, T, Kp))
    W = rng.standard_normal((P, H, Kp)) * 0.5
    R = rng.standard_normal((P, T, H))
    gamma = rng.uniform(0.5, 1.5, H)
    G = rng.standard_normal((P, T, H))
    eps = 1e-3
    f = lambda: _loss(X, W, R, gamma, G, P, p, idx, eps, s)  # noqa: E731
    fw = O.rowpar_forward(X, W, R, gamma, P, p, idx, eps=eps, private_scale=s, return_all=True)
    g = O.rowpar_backward(X, W, fw["h"], gamma, G, P, p, idx, eps=eps, private_scale=s)
    for name, A in (("dX", X), ("dW", W), ("dR", R), ("dgamma", gamma)):
        num = _fd(f, A)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_planted_mistakes_fail_the_pin():
    """Two plausible errors in the reduction step change the gradients: reducing before the
    norm derivative (the full-sync placement of Fig. 2a), and forgetting the sum over ranks."""
    P, T, Kp, H, p = 2, 2, 3, 6, 0.5
    rng = np.random.default_rng(5)
    X, W = rng.standard_normal((P, T, Kp)), rng.standard_normal((P, H, Kp))
    R, gamma, G = rng.standard_normal((P, T, H)), rng.uniform(0.5, 1.5, H), rng.standard_normal((P, T, H))
    fw = O.rowpar_forward(X, W, R, gamma, P, p, return_all=True)
    good = O.rowpar_backward(X, W, fw["h"], gamma, G, P, p)
    mask = fw["mask"]
    # reduce dout over ranks before the norm derivative, then back-propagate through each norm
    Gs = G.copy()
    Gs[:, :, mask] = G[:, :, mask].sum(axis=0)[None]
    dh_wrong, _ = O.rmsnorm_backward(fw["h"], gamma, Gs, 1e-5)
    dX_wrong = np.stack([dh_wrong[m] @ W[m] for m in range(P)])
    assert not np.allclose(dX_wrong, good["dX"], rtol=1e-3)
    # no sum over ranks for the shared channels
    dh, _ = O.rmsnorm_backward(fw["h"], gamma, G, 1e-5)
    dX_nosum = np.stack([dh[m] @ W[m] for m in range(P)])
    assert not np.allclose(dX_nosum, good["dX"], rtol=1e-3)


def test_shared_channel_gradient_identical_across_ranks_and_private_is_own():
    P, T, Kp, H, p, s = 4, 3, 2, 8, 0.5, 2.0
    rng = np.random.default_rng(9)
    h, gamma, G = rng.standard_normal((P, T, H)), rng.uniform(0.5, 1.5, H), rng.standard_normal((P, T, H))
    X, W = rng.standard_normal((P, T, Kp)), rng.standard_normal((P, H, Kp))
    g = O.rowpar_backward(X, W, h, gamma, G, P, p, private_scale=s)
    mask = O.sync_mask(H, p)
    for m in range(1, P):
        np.testing.assert_array_equal(g["dZt"][m][:, mask], g["dZt"][0][:, mask])
    np.testing.assert_allclose(g["dZt"][:, :, ~mask], s * g["dR"][:, :, ~mask], rtol=1e-15)
    np.testing.assert_allclose(g["dZt"][0][:, mask], g["dR"][:, :, mask].sum(axis=0), rtol=1e-12)

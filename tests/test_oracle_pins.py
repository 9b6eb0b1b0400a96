"""Pins of the float64 oracle against what the paper and the mathematics fix.

Each test pins the oracle to something other than itself: hand-worked values from the
paper's equations (tests/golden), a library routine on the unsharded matrices (p = 1 and
p = 0 special cases), a pure-Python brute force on tiny shapes, exact integer
constructions, closed forms and the variance relation of the paper's §4.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import caat_oracle as O
from oracle import brute as B
from partial_activation_sync_caat_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------
# Sync-set bookkeeping (App. A.2 Eq. 22: l < floor(h p))
# ---------------------------------------------------------------------------------------

def test_n_sync_floor_golden():
    for H, p, ns in _load("n_sync_floor.json")["cases"]:
        assert O.n_sync(H, p) == ns, (H, p)


def test_sync_mask_contiguous_and_list():
    m = O.sync_mask(16, 0.25)
    assert m.tolist() == [True] * 4 + [False] * 12
    m = O.sync_mask(16, 0.25, [1, 5, 9, 15])
    assert np.flatnonzero(m).tolist() == [1, 5, 9, 15]


@pytest.mark.parametrize("bad", [[1, 1, 2, 3], [3, 2, 1, 0], [0, 1, 2, 16], [-1, 0, 1, 2], [0, 1, 2]])
def test_sync_mask_rejects_bad_lists(bad):
    with pytest.raises(ValueError):
        O.sync_mask(16, 0.25, bad)


def test_sync_mask_rejects_bad_p():
    with pytest.raises(ValueError):
        O.n_sync(16, 1.5)
    with pytest.raises(ValueError):
        O.n_sync(16, -0.1)


# ---------------------------------------------------------------------------------------
# The worked two-rank example (§3.1 Eq. 7-8), hand-computed values
# ---------------------------------------------------------------------------------------

def test_eq8_two_rank_golden():
    g = _load("eq8_two_rank.json")
    Y1, Y2 = np.array(g["Y1"], float), np.array(g["Y2"], float)
    B1 = np.hstack([np.array(g["B11"], float), np.array(g["B21"], float)])  # device 1 rows
    B2 = np.hstack([np.array(g["B12"], float), np.array(g["B22"], float)])  # device 2 rows
    X = np.stack([Y1, Y2])                # [P, T, f/P]
    W = np.stack([B1.T, B2.T])            # [P, h, f/P]  (nn.Linear orientation)
    R = np.zeros((2, 2, 4))
    res = O.rowpar_forward(X, W, R, np.ones(4), g["P"], g["p"], return_all=True)
    assert res["Z"][0].tolist() == g["Z1"]
    assert res["Z"][1].tolist() == g["Z2"]


# ---------------------------------------------------------------------------------------
# Special cases that reduce to a library routine on the unsharded matrices
# ---------------------------------------------------------------------------------------

def _small_inputs(T=5, K=24, H=16, P=4, seed=3, **kw):
    return I.make_rowpar_inputs(T, K, H, P, seed, **kw)


def test_p1_equals_full_allreduce_unsharded_matmul():
    """p = 1 is a full all-reduce (§3): every rank's Z equals X_cat W_full^T (Eq. 21)."""
    P, T, K, H = 4, 7, 32, 24
    d = _small_inputs(T, K, H, P, seed=11, w_std=0.5)
    X = d["X"].double().numpy()
    W = d["W"].double().numpy()
    Xcat = np.concatenate([X[m] for m in range(P)], axis=1)     # [T, K]
    Wfull = np.concatenate([W[m] for m in range(P)], axis=1)    # [H, K]
    Zfull = np.matmul(Xcat, Wfull.T)
    res = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, 1.0, return_all=True)
    for m in range(P):
        np.testing.assert_allclose(res["Z"][m], Zfull, rtol=1e-12, atol=1e-12)
        h = Zfull + d["R"][m].double().numpy()
        ref = h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + 1e-5)
        np.testing.assert_allclose(res["out"][m], ref, rtol=1e-12, atol=1e-12)


def test_p0_gives_independent_ranks():
    """p = 0: no channel is shared, each rank is an independent local layer (§1)."""
    P, T, K, H = 3, 6, 18, 16
    d = _small_inputs(T, K, H, P, seed=5, w_std=0.5)
    res = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, 0.0, return_all=True)
    for m in range(P):
        Zm = np.matmul(d["X"][m].double().numpy(), d["W"][m].double().numpy().T)
        np.testing.assert_allclose(res["Z"][m], Zm, rtol=1e-12, atol=1e-12)


def test_private_channels_keep_own_partial_and_shared_are_equal():
    P, T, K, H = 4, 5, 16, 20
    d = _small_inputs(T, K, H, P, seed=9, w_std=0.5)
    for p in (0.25, 0.5, 0.75, 0.7):
        res = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
        mask = res["mask"]
        for m in range(P):
            Zm = np.matmul(d["X"][m].double().numpy(), d["W"][m].double().numpy().T)
            np.testing.assert_allclose(res["Z"][m][:, ~mask], Zm[:, ~mask], rtol=1e-12, atol=1e-12)
            np.testing.assert_array_equal(res["Z"][m][:, mask], res["Z"][0][:, mask])


# ---------------------------------------------------------------------------------------
# Brute force on tiny shapes
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("P,T,K,H,p,scale,idx", [
    (1, 3, 4, 8, 0.5, 1.0, None),
    (2, 4, 8, 8, 0.5, 1.0, None),
    (2, 3, 6, 12, 0.7, math.sqrt(2), None),
    (4, 2, 16, 16, 0.25, 2.0, [1, 6, 11, 14]),
    (4, 4, 8, 10, 1.0, 1.0, None),
    (4, 3, 8, 10, 0.0, 1.5, None),
])
def test_oracle_matches_brute_force(P, T, K, H, p, scale, idx):
    d = I.make_rowpar_inputs(T, K, H, P, seed=P * 100 + T, w_std=0.7, gamma="uniform")
    Zb, hb, ob = B.brute_rowpar(d["X"], d["W"], d["R"], d["gamma"], P, p, idx,
                                eps=1e-5, private_scale=scale)
    res = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, idx,
                           private_scale=scale, return_all=True)
    np.testing.assert_allclose(res["Z"], np.array(Zb), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["h"], np.array(hb), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["out"], np.array(ob), rtol=1e-12, atol=1e-12)


def test_swiglu_matches_brute_force():
    d = I.make_mlp_inputs(3, 8, 12, 2, seed=4, w_std=0.5)
    Yb = B.brute_swiglu(d["X"], d["A"])
    np.testing.assert_allclose(O.swiglu_fc1(d["X"], d["A"]), np.array(Yb), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Exact integer construction of the reduce bookkeeping
# ---------------------------------------------------------------------------------------

def integer_construction(P, T, H, Kp, a_of_t):
    """X_m[t, 0] = a(t), W_m[c, 0] = 2^m, everything else 0: partial_m[t, c] = 2^m a(t)."""
    X = torch.zeros(P, T, Kp, dtype=torch.bfloat16)
    W = torch.zeros(P, H, Kp, dtype=torch.bfloat16)
    for m in range(P):
        X[m, :, 0] = torch.tensor([float(a_of_t(t)) for t in range(T)])
        W[m, :, 0] = float(2 ** m)
    return X, W


def test_integer_construction_exact():
    P, T, H, Kp = 4, 6, 24, 8
    X, W = integer_construction(P, T, H, Kp, lambda t: 1 + t % 4)
    R = torch.zeros(P, T, H, dtype=torch.bfloat16)
    for p, idx in ((0.5, None), (0.25, [0, 7, 8, 23, 3, 5][:6]), (1.0, None), (0.0, None)):
        if idx is not None:
            idx = sorted(idx)
        res = O.rowpar_forward(X, W, R, torch.ones(H), P, p, idx, return_all=True)
        mask = res["mask"]
        for m in range(P):
            for t in range(T):
                a = 1 + t % 4
                row = res["h"][m][t]
                assert np.all(row[mask] == (2 ** P - 1) * a)
                assert np.all(row[~mask] == (2 ** m) * a)


# ---------------------------------------------------------------------------------------
# RMSNorm closed form (constant rows), hand-worked values
# ---------------------------------------------------------------------------------------

def test_rmsnorm_constant_rows_golden():
    for c in _load("rmsnorm_constant_row.json")["cases"]:
        h = np.full((1, 1, c["H"]), c["c"])
        out = O.rmsnorm(h, np.full(c["H"], c["gamma"]), c["eps"])
        np.testing.assert_allclose(out, c["out"], rtol=1e-15, atol=1e-15)


def test_rmsnorm_scale_invariance_and_unit_rms():
    rng = np.random.default_rng(0)
    h = rng.standard_normal((2, 3, 64))
    out = O.rmsnorm(h, np.ones(64), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, axis=-1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(O.rmsnorm(7.5 * h, np.ones(64), 0.0), out, rtol=1e-13)


# ---------------------------------------------------------------------------------------
# Private-channel scaling: variance relation of §4 Eq. 14-15
# ---------------------------------------------------------------------------------------

def test_private_scaling_matches_shared_variance():
    """With independent zero-mean partials of variance s^2, shared channels have variance
    P s^2 (Eq. 14) and private ones s^2 (Eq. 15); scaling private channels by sqrt(P)
    equalises them (§4)."""
    P, T, K, H = 4, 512, 256, 64
    d = I.make_rowpar_inputs(T, K, H, P, seed=21, x_std=1.0, w_std=1.0, r_std=0.0)
    for scale, ratio in ((1.0, P), (math.sqrt(P), 1.0)):
        res = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, 0.5,
                               private_scale=scale, return_all=True)
        Z = res["Z"]
        mask = res["mask"]
        v_shared = Z[:, :, mask].var()
        v_private = Z[:, :, ~mask].var()
        assert abs(v_shared / v_private / ratio - 1.0) < 0.15


# ---------------------------------------------------------------------------------------
# MLP block: at p = 1 with identical per-rank inputs it is the unsharded SwiGLU MLP
# (Eq. 20-21: Z = sigma(X A) B with A split by columns, B by rows)
# ---------------------------------------------------------------------------------------

def test_mlp_p1_equals_unsharded_swiglu_mlp():
    P, T, H, F = 4, 5, 16, 32
    d = I.make_mlp_inputs(T, H, F, P, seed=8, w_std=0.3)
    X0 = d["X"][0:1].expand(P, T, H).contiguous()
    Fp = F // P
    A = d["A"].double().numpy()
    W2 = d["W2"].double().numpy()
    Ag = np.concatenate([A[m, :Fp] for m in range(P)], axis=0)   # [F, H]
    Au = np.concatenate([A[m, Fp:] for m in range(P)], axis=0)   # [F, H]
    Bf = np.concatenate([W2[m] for m in range(P)], axis=1)       # [H, F]
    x = X0[0].double().numpy()
    g = x @ Ag.T
    u = x @ Au.T
    Zfull = ((g / (1.0 + np.exp(-g))) * u) @ Bf.T
    res = O.mlp_forward(X0, d["A"], d["W2"], d["R"], d["gamma"], P, 1.0, return_all=True)
    for m in range(P):
        np.testing.assert_allclose(res["Z"][m], Zfull, rtol=1e-11, atol=1e-12)


def test_silu_values():
    assert O.silu(np.array(0.0)) == 0.0
    np.testing.assert_allclose(O.silu(np.array(1.0)), 1.0 / (1.0 + math.exp(-1.0)), rtol=1e-15)
    np.testing.assert_allclose(O.silu(np.array(40.0)), 40.0, rtol=1e-15)
    assert abs(O.silu(np.array(-40.0))) < 1e-15


# ---------------------------------------------------------------------------------------
# Planted mistakes: each pin above must catch a plausible error in the oracle
# ---------------------------------------------------------------------------------------

def test_pins_catch_planted_mistakes(monkeypatch):
    g = _load("eq8_two_rank.json")
    Y1, Y2 = np.array(g["Y1"], float), np.array(g["Y2"], float)
    B1 = np.hstack([np.array(g["B11"], float), np.array(g["B21"], float)])
    B2 = np.hstack([np.array(g["B12"], float), np.array(g["B22"], float)])
    X = np.stack([Y1, Y2])
    W = np.stack([B1.T, B2.T])
    R = np.zeros((2, 2, 4))

    def wrong_reduce(Zt, mask, private_scale=1.0):  # private channels take rank 0's value
        Z = Zt * private_scale
        Z[:, :, mask] = Zt[:, :, mask].sum(axis=0)[None]
        Z[:, :, ~mask] = Zt[0][:, ~mask][None]
        return Z

    monkeypatch.setattr(O, "partial_channel_reduce", wrong_reduce)
    res = O.rowpar_forward(X, W, R, np.ones(4), 2, 0.5, return_all=True)
    assert res["Z"][1].tolist() != g["Z2"]
    monkeypatch.undo()

    def wrong_partials(X_, W_):  # transposed operand
        X_ = O._f64(X_)
        W_ = O._f64(W_)
        return np.stack([X_[m] @ W_[m][:, ::-1].T for m in range(X_.shape[0])])

    monkeypatch.setattr(O, "partial_products", wrong_partials)
    res = O.rowpar_forward(X, W, R, np.ones(4), 2, 0.5, return_all=True)
    assert res["Z"][0].tolist() != g["Z1"]


# ---------------------------------------------------------------------------------------
# Helpers: the backward's channel reduce is the adjoint of the forward's; sampled-row
# evaluation equals the full evaluation restricted to those rows; the pass rule's boundary
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("P,s", [(1, 1.0), (2, 1.0), (4, 1.5), (8, 0.5)])
def test_channel_reduce_backward_is_the_adjoint(P, s):
    rng = np.random.default_rng(P)
    T, H = 5, 24
    mask = np.zeros(H, dtype=bool)
    mask[rng.choice(H, size=H // 3, replace=False)] = True
    Z = rng.standard_normal((P, T, H))
    G = rng.standard_normal((P, T, H))
    lhs = float(np.sum(O.partial_channel_reduce(Z, mask, s) * G))
    rhs = float(np.sum(Z * O.partial_channel_reduce_backward(G, mask, s)))
    assert lhs == pytest.approx(rhs, rel=1e-12, abs=1e-12)
    # and as a matrix: the backward is the transpose of the forward's linear map
    n = P * T * H
    F = np.stack([O.partial_channel_reduce(e.reshape(P, T, H), mask, s).ravel() for e in np.eye(n)], axis=1)
    Bm = np.stack([O.partial_channel_reduce_backward(e.reshape(P, T, H), mask, s).ravel() for e in np.eye(n)],
                  axis=1)
    assert np.array_equal(F.T, Bm)


def test_sampled_rows_equal_the_full_layer_restricted():
    T, K, H, P, p = 12, 64, 40, 4, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=5, x_std=1.0, w_std=0.1, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=1)
    rows = np.array([0, 3, 7, 11])
    full = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, idx, private_scale=1.5)
    part = O.rowpar_rows(d["X"], d["W"], d["R"], d["gamma"], P, p, rows, idx, private_scale=1.5)
    assert np.array_equal(part, full[:, rows, :])
    m = I.make_mlp_inputs(T, 32, 48, P, seed=6, x_std=1.0, w_std=0.1)
    full = O.mlp_forward(m["X"], m["A"], m["W2"], m["R"], m["gamma"], P, p)
    part = O.mlp_rows(m["X"], m["A"], m["W2"], m["R"], m["gamma"], P, p, rows)
    assert np.array_equal(part, full[:, rows, :])


def test_within_tolerance_boundary():
    ref = np.array([0.0, 1.0, -4.0, 1e-4])
    bound = 2e-2 + 1e-2 * np.abs(ref)
    sign = np.array([1.0, 1.0, -1.0, 1.0])
    # errors just inside atol + rtol |ref| pass; one element just outside fails
    inside = ref + sign * bound * (1 - 1e-9)
    ok, max_abs, _ = O.within_tolerance(inside, ref)
    assert ok and max_abs == pytest.approx(6e-2)
    for i in range(4):
        over = inside.copy()
        over[i] = ref[i] + sign[i] * bound[i] * (1 + 1e-9)
        assert not O.within_tolerance(over, ref)[0], i
    # the reported relative error ignores |ref| <= 1e-3
    _, _, max_rel = O.within_tolerance(ref + 1e-2, ref)
    assert max_rel == pytest.approx(1e-2)

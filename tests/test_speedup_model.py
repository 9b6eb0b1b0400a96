"""The paper's speed-up model (App. C, Eq. 31-35): the oracle's definition-based version is
pinned against the closed forms and against operations counted on real (tiny) matrix
products; the library's host-only caat_speedup_model is checked against the oracle."""
import itertools

import numpy as np
import pytest

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import build as B
from partial_activation_sync_caat_b200 import caat as C


class _CountingMatmul:
    """m x p by p x n product done with explicit multiply-adds, counting them (2 per term)."""
    def __init__(self):
        self.ops = 0

    def __call__(self, a, b):
        m, p = a.shape
        p2, n = b.shape
        assert p == p2
        out = np.zeros((m, n))
        for i, j in itertools.product(range(m), range(n)):
            acc = 0.0
            for k in range(p):
                acc += a[i, k] * b[k, j]
                self.ops += 2
            out[i, j] = acc
        return out


@pytest.mark.parametrize("s,h", [(3, 4), (5, 2), (2, 6)])
def test_compute_ops_counted_on_a_tiny_layer(s, h):
    """Run one layer's GEMMs (qkv, scores, values, out projection, h -> 4h, 4h -> h) with a
    counting matmul: the count equals the oracle's G for r = 1, and G scales as 1/r."""
    rng = np.random.default_rng(0)
    mm = _CountingMatmul()
    x = rng.standard_normal((s, h))
    qkv = mm(x, rng.standard_normal((h, 3 * h)))
    q, k, v = qkv[:, :h], qkv[:, h:2 * h], qkv[:, 2 * h:]
    scores = mm(q, k.T)
    att = mm(scores, v)
    y = mm(att, rng.standard_normal((h, h)))
    f = mm(y, rng.standard_normal((h, 4 * h)))
    mm(f, rng.standard_normal((4 * h, h)))
    assert mm.ops == O.layer_compute_ops(h, s, 1)
    assert O.layer_compute_ops(h, s, 4) == pytest.approx(mm.ops / 4)


def test_closed_forms_match_definitions():
    rng = np.random.default_rng(1)
    for _ in range(200):
        h, s, r = rng.integers(64, 16384), rng.integers(1, 32768), rng.integers(1, 64)
        p, Cc = rng.uniform(0, 1), 10 ** rng.uniform(1, 6)
        sp, ps = O.speedup_model(h, s, r, p, Cc)
        x = (12 * h + 2 * s) / (Cc * r)
        assert sp == pytest.approx((1 - p) / (1 + x), rel=1e-12)      # Eq. 34
        assert ps == pytest.approx(min(x, 1.0), rel=1e-12)             # Eq. 35


def test_special_cases():
    h, s, r, Cc = 4096, 2048, 8, 3000.0
    assert O.speedup_model(h, s, r, 1.0, Cc)[0] == 0.0                  # full synchronization
    sp0, ps = O.speedup_model(h, s, r, 0.0, Cc)
    G, P1 = O.layer_compute_ops(h, s, r), O.layer_exchange(h, s, 1.0)
    assert sp0 == pytest.approx(Cc * P1 / (G + Cc * P1))                # all communication removed
    # below the cap, p* makes the exchange time equal the compute time
    Cbig = 1e6
    ps = O.speedup_model(h, s, r, 0.5, Cbig)[1]
    assert ps < 1 and Cbig * O.layer_exchange(h, s, ps) == pytest.approx(G)
    # speed-up is linear in (1 - p)
    a, b = O.speedup_model(h, s, r, 0.25, Cc)[0], O.speedup_model(h, s, r, 0.75, Cc)[0]
    assert a == pytest.approx(3 * b)


@pytest.fixture(scope="module")
def L():
    B.build()
    return C.lib()


def test_library_model_matches_oracle(L):
    rng = np.random.default_rng(2)
    for _ in range(50):
        h, s, r = float(rng.integers(64, 16384)), float(rng.integers(1, 32768)), float(rng.integers(1, 64))
        p, Cc = float(rng.uniform(0, 1)), float(10 ** rng.uniform(1, 6))
        got = C.caat_speedup_model(h, s, r, p, Cc)
        want = O.speedup_model(h, s, r, p, Cc)
        assert got[0] == pytest.approx(want[0], rel=1e-12) and got[1] == pytest.approx(want[1], rel=1e-12)
    for bad in [(0, 1, 1, 0.5, 1), (1, 1, 1, 1.5, 1), (1, 1, 1, 0.5, 0), (1, -1, 1, 0.5, 1)]:
        with pytest.raises(C.CaatError):
            C.caat_speedup_model(*bad)

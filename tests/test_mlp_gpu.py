"""GPU parity of the MLP block (column-parallel FC1 + SwiGLU kernel, then the partially
synchronized FC2, residual and RMSNorm) against the float64 oracle."""
import os
import subprocess
import sys

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


def run_mlp(d, P, p, idx=None, flags=0):
    g = to_dev(d)
    out = torch.empty_like(g["R"])
    C.caat_mlp_forward(g["X"], g["A"], g["W2"], g["R"], g["gamma"], idx, P, p, out, flags=flags)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    return out.cpu()


@pytest.mark.parametrize("T,H,F,P,p", [(300, 512, 1024, 4, 0.5), (130, 264, 272, 2, 0.7),
                                       (64, 512, 2048, 8, 0.25), (257, 776, 1600, 4, 1.0),
                                       (300, 512, 1408, 4, 0.5), (520, 512, 1536, 4, 0.5)])
def test_mlp_small(T, H, F, P, p):
    """F/P = 256, 136 (a last feature block of 8), 400, 352 and 384 (odd counts of 128-feature
    blocks, the last one partial or whole); p from 0.25 to 1."""
    d = I.make_mlp_inputs(T, H, F, P, seed=T + H, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    out = run_mlp(d, P, p)
    ref = O.mlp_forward(d["X"], d["A"], d["W2"], d["R"], d["gamma"], P, p)
    assert_out_close(out, ref, f"mlp T={T} H={H} F={F} P={P} p={p}")


def test_mlp_random_sync_idx_and_fused_norm():
    d = I.make_mlp_inputs(300, 512, 1024, 4, seed=3, x_std=1.0, w_std=0.05, r_std=1.0)
    idx = I.random_sync_idx(512, O.n_sync(512, 0.5), seed=5)
    ref = O.mlp_forward(d["X"], d["A"], d["W2"], d["R"], d["gamma"], 4, 0.5, idx)
    for flags in (0, C.CAAT_FLAG_FUSED_NORM):
        assert_out_close(run_mlp(d, 4, 0.5, idx, flags), ref, f"mlp random S flags={flags:#x}")


@pytest.mark.slow
def test_mlp_7b_block_sampled_rows():
    """The 7B MLP block workload (T=4096, H=4096, F=11008, P=8, p=0.5) at full size, checked on
    sampled token rows (rows are independent through the whole block)."""
    T, H, F, P, p = 4096, 4096, 11008, 8, 0.5
    d = I.make_mlp_inputs(T, H, F, P, seed=4, x_std=1.0, w_std=0.02, r_std=1.0)
    out = run_mlp(d, P, p)
    rows = I.sample_rows(T, 24, seed=1)
    ref = O.mlp_rows(d["X"], d["A"], d["W2"], d["R"], d["gamma"], P, p, rows)
    assert_out_close(out[:, torch.as_tensor(rows), :], ref, "mlp-7b sampled")


@pytest.mark.skipif(os.environ.get("CAAT_WIDE") is not None, reason="already the child run")
def test_mlp_without_wide_units():
    """The small MLP cases with the FC2's shared units all 256 x 256 (CAAT_WIDE=0, read once per
    process: a child pytest); the default takes 256 x 512 shared units where two whole shared
    blocks pair up and K >= 8192."""
    env = dict(os.environ, CAAT_WIDE="0")
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        "-k", "mlp_small or random_sync_idx"], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]

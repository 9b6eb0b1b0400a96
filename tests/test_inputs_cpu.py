"""The seeded input generators: shapes, layouts, reproducibility and the distributions of
the stated input recipe (X, R ~ N(0, 1) or N(0, 0.02); W ~ N(0, 0.02); gamma = 1 or
U(0.5, 1.5); random sync lists sorted, unique, in range)."""
import numpy as np
import pytest
import torch

from partial_activation_sync_caat_b200 import inputs as I


def _std(t):
    return float(t.float().std())


def test_rowpar_shapes_dtypes_and_layout():
    d = I.make_rowpar_inputs(64, 96, 40, 4, seed=3)
    assert d["X"].shape == (4, 64, 24) and d["W"].shape == (4, 40, 24)
    assert d["R"].shape == (4, 64, 40) and d["gamma"].shape == (40,)
    for t in d.values():
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    assert torch.all(d["gamma"] == 1)


def test_rowpar_rejects_k_not_divisible_by_p():
    with pytest.raises(ValueError):
        I.make_rowpar_inputs(8, 10, 8, 4)
    with pytest.raises(ValueError):
        I.make_rowpar_inputs(8, 8, 8, 2, gamma="bogus")


def test_same_seed_same_tensors_other_seed_differs():
    a = I.make_rowpar_inputs(32, 64, 48, 2, seed=5, gamma="uniform")
    b = I.make_rowpar_inputs(32, 64, 48, 2, seed=5, gamma="uniform")
    c = I.make_rowpar_inputs(32, 64, 48, 2, seed=6, gamma="uniform")
    for k in a:
        assert torch.equal(a[k], b[k])
        assert not torch.equal(a[k], c[k])


def test_tensors_drawn_in_sequence_are_not_copies():
    d = I.make_rowpar_inputs(64, 64, 64, 1, seed=0, x_std=1.0, w_std=1.0, r_std=1.0)
    assert not torch.equal(d["X"][0], d["W"][0])
    assert not torch.equal(d["X"][0], d["R"][0])


def test_distribution_moments():
    d = I.make_rowpar_inputs(512, 1024, 256, 2, seed=1, x_std=1.0, w_std=0.02, r_std=1.0,
                             gamma="uniform")
    # about 2.6e5 draws each: the sample std is within 1% of the target, the mean near 0
    assert abs(_std(d["X"]) - 1.0) < 0.01 and abs(float(d["X"].float().mean())) < 0.01
    assert abs(_std(d["W"]) / 0.02 - 1.0) < 0.02
    assert abs(_std(d["R"]) - 1.0) < 0.01
    g = d["gamma"].float()
    assert float(g.min()) >= 0.5 and float(g.max()) <= 1.5
    assert abs(float(g.mean()) - 1.0) < 0.05


def test_zero_std_gives_zero_tensor():
    d = I.make_rowpar_inputs(16, 32, 16, 2, seed=0, r_std=0.0)
    assert torch.count_nonzero(d["R"]) == 0
    assert torch.count_nonzero(d["X"]) > 0


def test_mlp_shapes_gate_rows_then_up_rows():
    d = I.make_mlp_inputs(16, 32, 48, 4, seed=2)
    assert d["X"].shape == (4, 16, 32)
    assert d["A"].shape == (4, 24, 32)       # 2·F/P rows: 12 gate rows, then 12 up rows
    assert d["W2"].shape == (4, 32, 12)
    assert d["R"].shape == (4, 16, 32) and d["gamma"].shape == (32,)
    with pytest.raises(ValueError):
        I.make_mlp_inputs(16, 32, 50, 4)


@pytest.mark.parametrize("H,n", [(2048, 1024), (768, 0), (768, 768), (4096, 1)])
def test_random_sync_idx_sorted_unique_in_range(H, n):
    s = I.random_sync_idx(H, n, seed=0)
    assert s.dtype == np.int32 and s.shape == (n,)
    assert np.all(np.diff(s) > 0)
    assert n == 0 or (s[0] >= 0 and s[-1] < H)
    assert np.array_equal(s, I.random_sync_idx(H, n, seed=0))
    if n == H:
        assert np.array_equal(s, np.arange(H, dtype=np.int32))


def test_random_sync_idx_is_spread_over_the_channels():
    # a random half of 2048 channels: each 256-channel block holds about 128 of them
    s = I.random_sync_idx(2048, 1024, seed=0)
    per_block = np.bincount(s // 256, minlength=8)
    assert per_block.min() > 64 and per_block.max() < 192


def test_sample_rows():
    r = I.sample_rows(8192, 128, seed=0)
    assert r.dtype == np.int64 and r.shape == (128,)
    assert np.all(np.diff(r) > 0) and r[0] >= 0 and r[-1] < 8192
    assert np.array_equal(I.sample_rows(10, 50), np.arange(10))

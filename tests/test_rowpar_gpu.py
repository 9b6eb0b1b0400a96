"""GPU parity of the row-parallel layer (tcgen05 GEMM + partial channel-reduce epilogue +
RMSNorm kernels, called through the C ABI) against the float64 oracle."""
import math
import os
import subprocess
import sys

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


def _compare(d, P, p, idx=None, *, eps=1e-5, scale=1.0, what="", flags=0):
    out, h = run_rowpar(d, P, p, idx, eps=eps, private_scale=scale, flags=flags)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, idx, eps=eps,
                           private_scale=scale, return_all=True)
    assert_h_close(h, ref["h"], what + " h")
    return assert_out_close(out, ref["out"], what + " out")


# ------------------------------------------------------------------ tiny sanity workload
def test_tiny_config_full():
    """T=256, K=H=768, P=2, p=0.5 (S = first 384), X,W ~ N(0,0.02), R ~ N(0,1), gamma=1."""
    d = I.make_rowpar_inputs(256, 768, 768, 2, seed=0, x_std=0.02, w_std=0.02, r_std=1.0)
    _compare(d, 2, 0.5, what="tiny")


def test_tiny_config_zero_residual_random_gamma():
    """Same shape with R = 0 and gamma ~ U(0.5,1.5): the output is the normalized GEMM."""
    d = I.make_rowpar_inputs(256, 768, 768, 2, seed=1, x_std=0.02, w_std=0.02, r_std=0.0, gamma="uniform")
    _compare(d, 2, 0.5, what="tiny R=0")


# ------------------------------------------------------------------ p sweep, ragged multi-tile
@pytest.mark.parametrize("p", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_p_sweep_ragged(p):
    """T=300 (3 row blocks, ragged), H=776 (4 column blocks, 8-wide tail), K/P=200 (4 k-blocks,
    8-wide tail), P=4."""
    d = I.make_rowpar_inputs(300, 800, 776, 4, seed=2, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    _compare(d, 4, p, what=f"p={p}")


@pytest.mark.parametrize("p", [0.7, 0.703125, 0.333])
def test_unaligned_shared_boundary(p):
    """n_s not a multiple of the tile width (537, 540, 255 of 768): mixed column blocks."""
    d = I.make_rowpar_inputs(200, 768, 768, 2, seed=3, x_std=1.0, w_std=0.05, r_std=1.0)
    _compare(d, 2, p, what=f"p={p}")


def test_random_sync_idx_small():
    d = I.make_rowpar_inputs(260, 1024, 1024, 4, seed=4, x_std=1.0, w_std=0.05, r_std=0.5)
    idx = I.random_sync_idx(1024, O.n_sync(1024, 0.5), seed=0)
    _compare(d, 4, 0.5, idx, what="random S")


def test_private_scale_sqrt_p_and_eps():
    d = I.make_rowpar_inputs(192, 512, 512, 4, seed=5, x_std=1.0, w_std=0.05, r_std=1.0)
    _compare(d, 4, 0.5, scale=math.sqrt(4), eps=1e-3, what="scale")


@pytest.mark.parametrize("T", [1, 8, 64, 127, 129])
def test_small_token_counts(T):
    d = I.make_rowpar_inputs(T, 1024, 512, 8, seed=6, x_std=1.0, w_std=0.05, r_std=1.0)
    _compare(d, 8, 0.5, what=f"T={T}")


def test_single_rank():
    d = I.make_rowpar_inputs(150, 256, 264, 1, seed=7, x_std=1.0, w_std=0.05, r_std=1.0)
    for p in (0.0, 0.5, 1.0):
        _compare(d, 1, p, what=f"P=1 p={p}")


@pytest.mark.parametrize("p", [0.0, 0.5, 0.7, 1.0])
def test_single_cta_kernel(p):
    """The single-CTA GEMM kernel (128-token tiles), forced for a shape the pair kernel would take."""
    d = I.make_rowpar_inputs(300, 800, 776, 4, seed=12, x_std=1.0, w_std=0.05, r_std=1.0)
    _compare(d, 4, p, flags=C.CAAT_FLAG_SINGLE_CTA, what=f"single-CTA p={p}")


def test_single_cta_random_sync_idx():
    d = I.make_rowpar_inputs(260, 1024, 1024, 4, seed=13, x_std=1.0, w_std=0.05, r_std=0.5)
    idx = I.random_sync_idx(1024, O.n_sync(1024, 0.5), seed=3)
    _compare(d, 4, 0.5, idx, flags=C.CAAT_FLAG_SINGLE_CTA, what="single-CTA random S")


@pytest.mark.parametrize("flags", [C.CAAT_FLAG_FUSED_NORM, C.CAAT_FLAG_ORDER_ROWBLOCK, C.CAAT_FLAG_ORDER_GROUPED,
                                   C.CAAT_FLAG_FUSED_NORM | C.CAAT_FLAG_SINGLE_CTA,
                                   C.CAAT_FLAG_ORDER_ROWBLOCK | C.CAAT_FLAG_SINGLE_CTA])
@pytest.mark.parametrize("p", [0.5, 0.7])
def test_norm_and_order_variants(flags, p):
    """The fused RMSNorm and the row-block-major tile order give the same result."""
    d = I.make_rowpar_inputs(520, 1024, 1032, 4, seed=14, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    _compare(d, 4, p, flags=flags, what=f"flags={flags:#x} p={p}")


@pytest.mark.parametrize("flags", [C.CAAT_FLAG_FUSED_NORM, C.CAAT_FLAG_FUSED_NORM | C.CAAT_FLAG_SINGLE_CTA])
def test_fused_norm_several_row_block_groups(flags):
    """T = 2304: more row blocks than one group of the grouped tile order (fused norm)."""
    d = I.make_rowpar_inputs(2304, 512, 1032, 4, seed=16, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    _compare(d, 4, 0.5, flags=flags, what=f"fused groups flags={flags:#x}")


def test_without_h_out_normalizes_in_place():
    d = I.make_rowpar_inputs(300, 800, 776, 4, seed=15, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 4, 0.5)
    for flags in (0, C.CAAT_FLAG_SINGLE_CTA, C.CAAT_FLAG_FUSED_NORM,
                  C.CAAT_FLAG_FUSED_NORM | C.CAAT_FLAG_SINGLE_CTA):
        out, _ = run_rowpar(d, 4, 0.5, h_out=False, flags=flags)
        assert_out_close(out, ref, f"no h_out flags={flags:#x}")


# ------------------------------------------------------------------ bit-exact bookkeeping
def _integer_inputs(P, T, H, Kp):
    X = torch.zeros(P, T, Kp, dtype=torch.bfloat16)
    W = torch.zeros(P, H, Kp, dtype=torch.bfloat16)
    a = torch.tensor([1.0 + (t % 4) for t in range(T)])
    for m in range(P):
        X[m, :, 3] = a
        W[m, :, 3] = float(2 ** m)
    return {"X": X, "W": W, "R": torch.zeros(P, T, H, dtype=torch.bfloat16),
            "gamma": torch.ones(H, dtype=torch.bfloat16)}


@pytest.mark.parametrize("P,p,random_idx", [(4, 0.5, False), (4, 0.3, True), (4, 0.0, False),
                                            (4, 1.0, False), (2, 0.7, False), (3, 0.5, True)])
def test_integer_construction_bit_exact(P, p, random_idx):
    """partial_m[t, c] = 2^m a(t): every shared channel must read exactly (2^P - 1) a(t), every
    private channel of rank m exactly 2^m a(t) (exact in fp32 and bf16)."""
    T, H, Kp = 130, 520, 16
    d = _integer_inputs(P, T, H, Kp)
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=P) if random_idx else None
    _, h = run_rowpar(d, P, p, idx)
    mask, ns = C.caat_sync_mask(H, p, idx)
    mask = mask.astype(bool)
    np.testing.assert_array_equal(mask, O.sync_mask(H, p, idx))
    a = np.array([1.0 + (t % 4) for t in range(T)])
    hv = h.double().numpy()
    for m in range(P):
        want = np.where(mask[None, :], (2 ** P - 1) * a[:, None], (2 ** m) * a[:, None])
        np.testing.assert_array_equal(hv[m], want)


# ------------------------------------------------------------------ aliasing, determinism
def test_out_aliases_residual():
    d = I.make_rowpar_inputs(140, 512, 512, 2, seed=8, x_std=1.0, w_std=0.05, r_std=1.0)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 2, 0.5)
    out, _ = run_rowpar(d, 2, 0.5, out_alias_residual=True)
    assert_out_close(out, ref, "in-place")


def test_deterministic():
    d = I.make_rowpar_inputs(300, 1024, 768, 4, seed=9, x_std=1.0, w_std=0.05, r_std=1.0)
    o1, h1 = run_rowpar(d, 4, 0.5)
    o2, h2 = run_rowpar(d, 4, 0.5)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_empty_tokens():
    g = to_dev(I.make_rowpar_inputs(0, 256, 256, 2, seed=0))
    out = torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, 2, 0.5, out)
    torch.cuda.synchronize()


# ------------------------------------------------------------------ bounded waits
@pytest.mark.parametrize("flags", [0, C.CAAT_FLAG_SINGLE_CTA])
def test_stall_reports_timeout_and_context_survives(flags):
    """The test hook makes the MMA warp withhold its accumulator signal: every consumer wait
    must run out (bounded), the status word must read CAAT_ERR_TIMEOUT, and the next call
    must work normally."""
    d = I.make_rowpar_inputs(256, 512, 512, 2, seed=10, x_std=1.0, w_std=0.05, r_std=1.0)
    g = to_dev(d)
    out = torch.empty_like(g["R"])
    C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, 2, 0.5, out,
                          flags=C.CAAT_FLAG_TEST_STALL | flags)
    st = C.caat_get_device_status()
    assert st & 0xFF == C.CAAT_ERR_TIMEOUT
    assert C.caat_get_device_status() == 0     # cleared by the read
    _compare(d, 2, 0.5, what="after timeout")


# ------------------------------------------------------------------ host-buffer entry point
@pytest.mark.parametrize("T", [300, 1060, 2500])
def test_host_buffer_entry_matches_device_entry(T):
    """caat_rowpar_forward_host (pipelined over chunks of up to 1024 tokens, the last ones
    smaller, none below 256: 300 -> one chunk, 1060 -> 768 + 292, 2500 -> 1024 + 768 + 708) gives
    the same bits as the device entry point: rows are independent and every kernel is
    deterministic per row."""
    P, K, H = 4, 1024, 776
    d = I.make_rowpar_inputs(T, K, H, P, seed=17, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    out_dev, h_dev = run_rowpar(d, P, 0.5)
    hX, hW, hR, hg = (d[k].contiguous().pin_memory() for k in ("X", "W", "R", "gamma"))
    hout = torch.empty(P, T, H, dtype=torch.bfloat16).pin_memory()
    hh = torch.empty(P, T, H, dtype=torch.bfloat16).pin_memory()
    ws = C.alloc_workspace(C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR_HOST))
    for _ in range(2):   # a second call reuses the workspace and the copy streams
        hout.zero_()
        C.caat_rowpar_forward_host(hX, hW, hR, hg, None, P, 0.5, hout, ws, h_out=hh)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        assert torch.equal(hout, out_dev)
        assert torch.equal(hh, h_dev)


def test_overlapped_norm_chunks_match():
    """CAAT_FLAG_OVERLAP_NORM (GEMM in 2048-token launches, each launch's row norm on a side
    stream) gives the same bits as the single launch, and matches the oracle."""
    T, K, H, P = 4352, 512, 776, 2
    d = I.make_rowpar_inputs(T, K, H, P, seed=18, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    o1, h1 = run_rowpar(d, P, 0.5)
    o2, h2 = run_rowpar(d, P, 0.5, flags=C.CAAT_FLAG_OVERLAP_NORM)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, 0.5)
    assert_out_close(o2, ref, "overlap")


# ------------------------------------------------------------------ mixed column blocks
@pytest.mark.parametrize("p,random_idx", [(0.3, True), (0.703125, False), (0.5, True)])
def test_mixed_block_tma_merge_matches_register_epilogue(p, random_idx):
    """Column blocks holding shared and private channels: with the full workspace the CTA-pair
    kernel stores them with TMA boxes (the private unit merges its channels into the boxes its
    shared unit stored first, behind per-row-group flags); with only the 256-byte minimum
    workspace they take the register epilogue.  Same bits either way, and both match the
    oracle.  T = 600: three 256-token row blocks, the last one ragged."""
    T, K, H, P = 600, 1024, 1288, 4
    d = I.make_rowpar_inputs(T, K, H, P, seed=21, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    idx = I.random_sync_idx(H, O.n_sync(H, p), seed=5) if random_idx else None
    g = to_dev(d)
    res = []
    for ws_bytes in (C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR), 256):
        ws = C.alloc_workspace(ws_bytes)
        out = torch.empty_like(g["R"])
        hb = torch.empty_like(g["R"])
        C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], idx, P, p, out, h_out=hb, workspace=ws,
                              private_scale=0.75)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        res.append((out.cpu(), hb.cpu()))
    assert torch.equal(res[0][1], res[1][1]) and torch.equal(res[0][0], res[1][0])
    r = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, sync_idx=idx, private_scale=0.75,
                         return_all=True)
    assert_h_close(res[0][1], r["h"], "h merged")
    assert_out_close(res[0][0], r["out"], "out merged")


# ------------------------------------------------------------------ shared sums stored once
@pytest.mark.parametrize("T,H,p,with_h", [(600, 1024, 0.5, True), (300, 776, 1.0, True),
                                          (600, 1280, 0.375, True), (600, 1280, 0.375, False),
                                          (129, 512, 0.25, True), (520, 2048, 0.625, True),
                                          (520, 2048, 0.625, False)])
def test_shared_sums_once_match_per_rank_stores(T, H, p, with_h):
    """S the first n_s channels with n_s % 8 == 0: with the full workspace the GEMM stores the
    shared channels' cross-rank sums once (fp32) and the norm kernel adds each rank's residual;
    with the 256-byte minimum every shared tile stores h for all P ranks.  h has the same bits
    either way (one fp32 sum plus the residual, one rounding); both match the oracle.  Covers
    tile-aligned and mixed shared boundaries (480 of 1280), p = 1, a ragged last row block and
    h written in place into out.  Pairs of whole shared column blocks run as 256 x 512 units:
    1024 x 0.5 has one, 776 x 1.0 two (the second ending in an 8-channel block), 2048 x 0.625
    two and one ordinary shared unit."""
    K, P = 1024, 4
    d = I.make_rowpar_inputs(T, K, H, P, seed=31, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    g = to_dev(d)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
    res = []
    for ws_bytes in (C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR), 256):
        ws = C.alloc_workspace(ws_bytes)
        out = torch.empty_like(g["R"])
        hb = torch.empty_like(g["R"]) if with_h else None
        C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out, h_out=hb, workspace=ws)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        res.append((out.cpu(), hb.cpu() if with_h else None))
        assert_out_close(res[-1][0], ref["out"], f"out ws={ws_bytes}")
    if with_h:
        assert torch.equal(res[0][1], res[1][1])
        assert_h_close(res[0][1], ref["h"], "h shared sums")


def test_shared_sums_wide_units_long_k():
    """K = 8192 with private channels: the default takes the 256 x 512 shared units (two whole
    shared column blocks per unit) for S = the first 512 of 1024 channels.  Same h bits as the
    per-rank-store path; both match the oracle."""
    T, K, H, P, p = 520, 8192, 1024, 4, 0.5
    d = I.make_rowpar_inputs(T, K, H, P, seed=32, x_std=1.0, w_std=0.02, r_std=1.0, gamma="uniform")
    g = to_dev(d)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
    hs = []
    for ws_bytes in (C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR), 256):
        ws = C.alloc_workspace(ws_bytes)
        out, hb = torch.empty_like(g["R"]), torch.empty_like(g["R"])
        C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out, h_out=hb, workspace=ws)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        assert_out_close(out.cpu(), ref["out"], f"out ws={ws_bytes}")
        hs.append(hb.cpu())
    assert torch.equal(hs[0], hs[1])
    assert_h_close(hs[0], ref["h"], "h wide")


@pytest.mark.skipif(os.environ.get("CAAT_WIDE") is not None, reason="already the child run")
def test_shared_sums_with_wide_units_forced():
    """The shared-sum cases above with 256 x 512 units wherever two whole shared blocks pair up
    (CAAT_WIDE=1, read once per process: a child pytest), also at p = 1 and short K."""
    env = dict(os.environ, CAAT_WIDE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", __file__, "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        "-k", "shared_sums_once or p_sweep_ragged or single_rank"],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


def test_shared_sums_all_shared_schedule_chosen_wide_units():
    """p = 1 (no private channels) with K = 8192 and 24 row blocks of 4 shared column blocks: on
    the 74 CTA pairs of a B200 the host's simulated schedule runs one of each row block's two
    pairs of blocks as a 256 x 512 unit and the other two blocks as ordinary units after every
    wide one.  h has the per-rank-store path's bits (the 256-byte workspace); out matches the
    oracle on sampled rows."""
    T, K, H, P, p = 6144, 8192, 1024, 4, 1.0
    d = I.make_rowpar_inputs(T, K, H, P, seed=33, x_std=1.0, w_std=0.02, r_std=1.0, gamma="uniform")
    g = to_dev(d)
    outs, hs = [], []
    for ws_bytes in (C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR), 256):
        ws = C.alloc_workspace(ws_bytes)
        out, hb = torch.empty_like(g["R"]), torch.empty_like(g["R"])
        C.caat_rowpar_forward(g["X"], g["W"], g["R"], g["gamma"], None, P, p, out, h_out=hb, workspace=ws)
        torch.cuda.synchronize()
        assert C.caat_get_device_status() == 0
        outs.append(out.cpu())
        hs.append(hb.cpu())
    assert torch.equal(hs[0], hs[1])
    rows = I.sample_rows(T, 48, seed=3)
    ref = O.rowpar_rows(d["X"], d["W"], d["R"], d["gamma"], P, p, rows)
    assert_out_close(outs[0][:, torch.as_tensor(rows), :], ref, "p=1 schedule-chosen wide units")

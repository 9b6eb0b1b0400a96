"""The layer over real devices (one tensor-parallel rank per process), its orchestration on two
gloo CPU ranks: every rank computes its local step, the shared channels' fp32 partials are
summed by the collective, and the finishing step completes h and the RMSNorm.  The two GPU
kernels are replaced here by test-only float64 stand-ins with the same buffer conventions
(zs [T, n_s] fp32; h [T, H] with the private channels after the local step), so that this test
covers the exchange (which buffer, which dtype, which ranks) and the data flow, and compares
every rank's output with the float64 oracle of the whole layer (App. A.2 Eq. 22, §4 Eq. 9)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local_standin(X_r, W_r, R_r, p, zs, h, private_scale=1.0, **_):
    """float64 stand-in for caat_rowpar_tp_local (test only)."""
    H = W_r.shape[0]
    ns = zs.shape[1]
    Z = X_r.double() @ W_r.double().T
    zs.copy_(Z[:, :ns].float())
    h[:, ns:] = (private_scale * Z[:, ns:] + R_r[:, ns:].double()).to(h.dtype)
    assert ns == int(np.floor(H * p))


def _finish_standin(zs, R_r, h, gamma, p, out, eps=1e-5, **_):
    """float64 stand-in for caat_rowpar_tp_finish (test only)."""
    ns = zs.shape[1]
    h[:, :ns] = (zs.double() + R_r[:, :ns].double()).to(h.dtype)
    hd = h.double()
    rstd = 1.0 / torch.sqrt((hd * hd).mean(dim=1, keepdim=True) + eps)
    out.copy_((hd * rstd * gamma.double()).to(out.dtype))


def _worker(rank, world, port, p, out_q):
    sys.path.insert(0, ROOT)
    import datetime
    from oracle import caat_oracle as O
    from partial_activation_sync_caat_b200 import inputs as I
    from partial_activation_sync_caat_b200.tp import TPRowParallel, exchanged_bytes
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        T, K, H, P = 24, 64, 40, world
        # every rank draws the whole layer's inputs from the same seed and keeps its own slice
        d = I.make_rowpar_inputs(T, K, H, P, seed=11, x_std=1.0, w_std=0.1, r_std=1.0, gamma="uniform")
        layer = TPRowParallel(H, p, local_fn=_local_standin, finish_fn=_finish_standin)
        X_r, W_r, R_r = d["X"][rank].contiguous(), d["W"][rank].contiguous(), d["R"][rank].contiguous()
        out = torch.empty(T, H, dtype=torch.bfloat16)
        zs, h = layer.buffers(T, "cpu")
        layer.forward(X_r, W_r, R_r, d["gamma"], out, zs=zs, h=h)
        ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
        ok, max_abs, _ = O.within_tolerance(out.float(), ref["out"][rank])
        h_err = float(np.max(np.abs(O._f64(h.float()) - ref["h"][rank])))
        out_q[rank] = (ok, max_abs, h_err, layer.n_s, exchanged_bytes(T, H, p))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("p", [0.0, 0.5, 1.0])
def test_two_gloo_ranks_partial_channel_reduce(p):
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()  # no fork of this (threaded) process
    res = manager.dict()
    mp.start_processes(_worker, args=(world, port, p, res), nprocs=world, start_method="spawn")
    for rank in range(world):
        ok, max_abs, h_err, ns, nbytes = res[rank]
        assert ok, f"rank {rank}: max_abs {max_abs}"
        assert h_err < 0.05
        assert ns == int(np.floor(40 * p))
        assert nbytes == 4 * 24 * ns      # only the shared channels cross devices


def test_exchange_is_p_of_a_full_all_reduce():
    sys.path.insert(0, ROOT)
    from partial_activation_sync_caat_b200.tp import exchanged_bytes, n_shared
    T, H = 8192, 4096
    full = 4 * T * H
    for p in (0.0, 0.25, 0.5, 0.75, 1.0):
        assert exchanged_bytes(T, H, p) == int(p * full)
    assert n_shared(768, 0.7) == 537

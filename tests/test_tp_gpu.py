"""The layer over real devices (caat_rowpar_tp_local / caat_rowpar_tp_finish), emulated on one
GPU: every rank's local step runs on its own slice, the shared channels' fp32 partials are
summed over the ranks in rank order (standing in for the all-reduce between devices), and every
rank finishes.  Compared with the float64 oracle (App. A.2 Eq. 22, §4 Eq. 9): the local partials
of the shared channels, h and out."""
import numpy as np
import pytest
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I
from partial_activation_sync_caat_b200.tp import TPRowParallel

from gpu_util import assert_h_close, assert_out_close, ensure_built, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _emulate(d, P, p, scale=1.0):
    g = to_dev(d)
    T, H = d["R"].shape[1], d["R"].shape[2]
    ns = O.n_sync(H, p)
    zs = [torch.empty(T, ns, dtype=torch.float32, device="cuda") for _ in range(P)]
    hs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    for r in range(P):
        C.caat_rowpar_tp_local(g["X"][r].contiguous(), g["W"][r].contiguous(), g["R"][r].contiguous(), p, zs[r],
                               hs[r], private_scale=scale)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    local = [z.cpu().clone() for z in zs]
    total = torch.zeros(T, ns, dtype=torch.float32, device="cuda")
    for r in range(P):           # the exchange: a sum over ranks, every rank receives it
        total += zs[r]
    outs = []
    for r in range(P):
        z = total.clone()
        out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        C.caat_rowpar_tp_finish(z, g["R"][r].contiguous(), hs[r], g["gamma"], p, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    return local, torch.stack([h.cpu() for h in hs]), torch.stack([o.cpu() for o in outs])


@pytest.mark.parametrize("T,K,H,P,p", [
    (300, 800, 784, 4, 0.5),     # n_s = 392: a 64-channel chunk straddles the sync boundary
    (1024, 2048, 2048, 8, 0.25),
    (200, 2752, 4096, 2, 0.75),  # the 7B row width
    (64, 1024, 1024, 4, 0.0),
    (64, 1024, 1024, 4, 1.0),
    (1, 512, 512, 2, 0.5),
    (257, 256, 272, 1, 0.5),     # one rank: the exchange is the identity
])
def test_tp_layer_emulated_matches_oracle(T, K, H, P, p):
    d = I.make_rowpar_inputs(T, K, H, P, seed=60 + T % 13, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    local, h, out = _emulate(d, P, p)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
    ns = O.n_sync(H, p)
    Zt = O.partial_products(d["X"], d["W"])          # [P, T, H] float64
    for r in range(P):
        z = Zt[r][:, :ns]
        err = np.abs(local[r].double().numpy() - z)
        bound = 1e-4 * np.sqrt(np.mean(z * z) + 1e-30) + 1e-5 * np.abs(z)
        assert (err <= bound).all(), f"rank {r}: local partial max err {err.max():.3e}"
    assert_h_close(h, ref["h"], "tp h")
    assert_out_close(out, ref["out"], "tp out")


def test_tp_layer_private_scale():
    d = I.make_rowpar_inputs(192, 512, 512, 4, seed=66, x_std=1.0, w_std=0.05, r_std=1.0)
    _, h, out = _emulate(d, 4, 0.5, scale=2.0)
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 4, 0.5, private_scale=2.0, return_all=True)
    assert_h_close(h, ref["h"], "tp scale h")
    assert_out_close(out, ref["out"], "tp scale out")


def test_tp_module_single_rank_group():
    """TPRowParallel on a one-rank process group (P = 1): the collective is the identity and the
    result equals the single-device layer with P = 1."""
    import os
    import socket
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        T, K, H, p = 500, 1024, 1024, 0.5
        d = I.make_rowpar_inputs(T, K, H, 1, seed=67, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
        g = to_dev(d)
        layer = TPRowParallel(H, p)
        out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        layer.forward(g["X"][0].contiguous(), g["W"][0].contiguous(), g["R"][0].contiguous(), g["gamma"], out)
        torch.cuda.synchronize()
        ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 1, p)
        assert_out_close(out.cpu().unsqueeze(0), ref, "tp module")
    finally:
        dist.destroy_process_group()


def test_tp_rejects_unaligned_sync_count():
    g = to_dev(I.make_rowpar_inputs(64, 256, 776, 1, seed=68))
    zs = torch.empty(64, 388, dtype=torch.float32, device="cuda")
    h = torch.empty(64, 776, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(C.CaatError) as e:   # floor(776 * 0.5) = 388, not a multiple of 8
        C.caat_rowpar_tp_local(g["X"][0].contiguous(), g["W"][0].contiguous(), g["R"][0].contiguous(), 0.5, zs, h)
    assert e.value.code == C.CAAT_ERR_UNSUPPORTED

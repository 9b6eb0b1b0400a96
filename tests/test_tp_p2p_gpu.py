"""The layer over real devices with the exchange over peer memory (caat_rowpar_tp_local_push /
caat_rowpar_tp_reduce / caat_rowpar_tp_finish_wait), emulated on one GPU: every rank's buffers
live on this device, each rank's local GEMM pushes its fp32 partials of the shared channels into
the owners' receive buffers, every owner reduces its slice into every rank's gather buffer, and
every rank finishes.  The steps run one after another on one stream, so no kernel waits on
another one that runs at the same time: every flag a step waits for was raised by an earlier
launch.  Compared with the float64 oracle (App. A.2 Eq. 22, §4 Eq. 9): the pushed partials, the
reduced sums, h and out."""
import numpy as np
import pytest
import torch

from oracle import caat_oracle as O
from partial_activation_sync_caat_b200 import caat as C
from partial_activation_sync_caat_b200 import inputs as I

from gpu_util import assert_h_close, assert_out_close, ensure_built, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


class _Buffers:
    """Every rank's exchange buffers, all on this GPU."""

    def __init__(self, T, H, P, p):
        self.ns = O.n_sync(H, p)
        self.w = self.ns // P
        wb = max(self.w, 4)
        self.recv = [torch.full((P, T, wb), float("nan"), dtype=torch.float32, device="cuda") for _ in range(P)]
        self.gather = [torch.full((T, max(self.ns, 4)), float("nan"), dtype=torch.float32, device="cuda")
                       for _ in range(P)]
        self.flags = [torch.zeros(2, P, dtype=torch.int32, device="cuda") for _ in range(P)]
        self.ws = [C.alloc_workspace(256, "cuda") for _ in range(P)]
        self.P = P

    def peers(self, rank, epoch):
        return C.tp_peers(self.P, rank, epoch, self.recv, self.gather, self.flags)


def _call(bufs, g, P, p, epoch, scale=1.0):
    T, H = g["R"].shape[1], g["R"].shape[2]
    hs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    for r in range(P):
        C.caat_rowpar_tp_local_push(g["X"][r].contiguous(), g["W"][r].contiguous(), g["R"][r].contiguous(), p, hs[r],
                                    bufs.peers(r, epoch), workspace=bufs.ws[r], private_scale=scale)
    for q in range(P):
        C.caat_rowpar_tp_reduce(T, H, p, bufs.peers(q, epoch), workspace=bufs.ws[q])
    for r in range(P):
        C.caat_rowpar_tp_finish_wait(g["R"][r].contiguous(), hs[r], g["gamma"], p, outs[r], bufs.peers(r, epoch))
    torch.cuda.synchronize()
    assert C.caat_get_device_status() == 0
    return torch.stack([h.cpu() for h in hs]), torch.stack([o.cpu() for o in outs])


def _check(d, bufs, h, out, P, p, scale=1.0):
    ns, w = bufs.ns, bufs.w
    ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, private_scale=scale, return_all=True)
    if ns:
        Zt = O.partial_products(d["X"], d["W"])  # [P, T, H] float64
        for r in range(P):
            # rank r's partial of owner q's columns sits in recv[q][r]
            pushed = torch.cat([bufs.recv[q][r, :, :w].cpu() for q in range(P)], dim=1).double().numpy()
            z = Zt[r][:, :ns]
            err = np.abs(pushed - z)
            bound = 1e-4 * np.sqrt(np.mean(z * z) + 1e-30) + 1e-5 * np.abs(z)
            assert (err <= bound).all(), f"rank {r}: pushed partial max err {err.max():.3e}"
        zsum = Zt[:, :, :ns].sum(axis=0)
        for r in range(P):
            got = bufs.gather[r][:, :ns].cpu().double().numpy()
            err = np.abs(got - zsum)
            bound = 1e-4 * np.sqrt(np.mean(zsum * zsum) + 1e-30) + 1e-5 * np.abs(zsum)
            assert (err <= bound).all(), f"rank {r}: gathered sum max err {err.max():.3e}"
    assert_h_close(h, ref["h"], "tp p2p h")
    assert_out_close(out, ref["out"], "tp p2p out")


@pytest.mark.parametrize("T,K,H,P,p", [
    (300, 800, 1024, 4, 0.5),
    (1024, 2048, 2048, 8, 0.25),
    (200, 2752, 4096, 2, 0.75),      # the 7B row width
    (200, 768, 1024, 3, 0.28125),    # n_s = 288: a 64-channel chunk straddles the sync boundary
    (64, 1024, 1024, 4, 0.0),        # nothing exchanged
    (64, 1024, 1024, 4, 1.0),
    (1, 512, 512, 2, 0.5),
    (257, 256, 256, 1, 0.5),         # one rank: the owner of every column is itself
])
def test_tp_peer_exchange_emulated_matches_oracle(T, K, H, P, p):
    d = I.make_rowpar_inputs(T, K, H, P, seed=70 + T % 11, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    bufs = _Buffers(T, H, P, p)
    h, out = _call(bufs, to_dev(d), P, p, epoch=1)
    _check(d, bufs, h, out, P, p)


def test_tp_peer_exchange_reuses_buffers_across_calls():
    """Three calls on the same buffers with epochs 1, 2, 3 and new inputs each time."""
    T, K, H, P, p = 256, 1024, 1024, 4, 0.5
    bufs = _Buffers(T, H, P, p)
    for epoch in (1, 2, 3):
        d = I.make_rowpar_inputs(T, K, H, P, seed=80 + epoch, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
        h, out = _call(bufs, to_dev(d), P, p, epoch=epoch, scale=1.5)
        _check(d, bufs, h, out, P, p, scale=1.5)
        assert torch.equal(bufs.flags[0].cpu(), torch.full((2, P), epoch, dtype=torch.int32))


def test_tp_peer_exchange_wait_runs_out():
    """A finishing step whose owners never reduce (nothing raises its flags): the bounded wait
    ends with CAAT_ERR_TIMEOUT in the device status word, nothing is written, and the context
    stays usable."""
    T, K, H, P, p = 64, 512, 512, 2, 0.5
    g = to_dev(I.make_rowpar_inputs(T, K, H, P, seed=90))
    bufs = _Buffers(T, H, P, p)
    h = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
    C.caat_rowpar_tp_finish_wait(g["R"][0].contiguous(), h, g["gamma"], p, out, bufs.peers(0, 7))
    st = C.caat_get_device_status()
    assert st & 0xFF == C.CAAT_ERR_TIMEOUT
    assert int(out.abs().sum()) == 0
    # the context still works: a full exchange afterwards
    d = I.make_rowpar_inputs(T, K, H, P, seed=91, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
    bufs = _Buffers(T, H, P, p)
    h2, out2 = _call(bufs, to_dev(d), P, p, epoch=1)
    _check(d, bufs, h2, out2, P, p)


def test_tp_peer_exchange_rejects_bad_descriptors():
    T, K, H, P, p = 64, 512, 1024, 2, 0.5
    g = to_dev(I.make_rowpar_inputs(T, K, H, P, seed=92))
    bufs = _Buffers(T, H, P, p)
    h = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    X, W, R = g["X"][0].contiguous(), g["W"][0].contiguous(), g["R"][0].contiguous()
    with pytest.raises(C.CaatError) as e:       # epoch 0 is never used
        C.caat_rowpar_tp_local_push(X, W, R, p, h, bufs.peers(0, 0), workspace=bufs.ws[0])
    assert e.value.code == C.CAAT_ERR_INVALID_ARG
    with pytest.raises(C.CaatError) as e:       # rank outside the world
        C.caat_rowpar_tp_local_push(X, W, R, p, h, C.tp_peers(2, 2, 1, bufs.recv, bufs.gather, bufs.flags),
                                    workspace=bufs.ws[0])
    assert e.value.code == C.CAAT_ERR_INVALID_ARG
    with pytest.raises(C.CaatError) as e:       # n_s = 480 is not a multiple of 32 * world = 64
        C.caat_rowpar_tp_local_push(X, W, R, 0.46875, h, bufs.peers(0, 1), workspace=bufs.ws[0])
    assert e.value.code == C.CAAT_ERR_UNSUPPORTED


def test_tp_p2p_module_single_rank():
    """TPRowParallelP2P with one rank and no process group: its buffers come from the CUDA
    runtime (the allocation path shared by IPC), the owner of every column is itself, and two
    calls (epochs 1 and 2) give the single-device layer with P = 1."""
    from partial_activation_sync_caat_b200.tp import TPRowParallelP2P
    T, K, H, p = 500, 1024, 1024, 0.5
    layer = TPRowParallelP2P(H, p, T_max=512)
    try:
        for call in range(2):
            d = I.make_rowpar_inputs(T, K, H, 1, seed=93 + call, x_std=1.0, w_std=0.05, r_std=1.0, gamma="uniform")
            g = to_dev(d)
            out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
            layer.forward(g["X"][0].contiguous(), g["W"][0].contiguous(), g["R"][0].contiguous(), g["gamma"], out)
            torch.cuda.synchronize()
            assert C.caat_get_device_status() == 0
            ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], 1, p)
            assert_out_close(out.cpu().unsqueeze(0), ref, "tp p2p module")
        assert layer.epoch == 2
    finally:
        layer.close()

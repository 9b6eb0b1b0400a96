"""The layer over real devices with the exchange over peer memory (TPRowParallelP2P), its
protocol on two CPU processes: the buffers every rank allocates are POSIX shared memory standing
in for device memory mapped by CUDA IPC (the handles travel over a gloo group exactly as the
IPC handles do), and the three steps are test-only float64/float32 stand-ins for the library's
kernels with the same buffer layouts and flag protocol (recv [world][T_max][w], gather
[T_max][n_s], flags [2][world] raised with the call's epoch; each step waits for the flags the
previous one raises).  Two calls with new inputs reuse the buffers.  Every rank's output is
compared with the float64 oracle of the whole layer (App. A.2 Eq. 22, §4 Eq. 9)."""
import os
import socket
import sys
import time

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


class ShmMemory:
    """Shared-memory stand-in for CUDA IPC buffers (test only)."""

    def __init__(self):
        self.own, self.mapped = [], []

    def alloc(self, nbytes):
        from multiprocessing import shared_memory
        shm = shared_memory.SharedMemory(create=True, size=int(nbytes))
        np.ndarray((int(nbytes),), dtype=np.uint8, buffer=shm.buf)[:] = 0
        self.own.append(shm)
        return shm.name.encode(), shm

    def open(self, handle):
        from multiprocessing import resource_tracker, shared_memory
        shm = shared_memory.SharedMemory(name=handle.decode())
        resource_tracker.unregister(shm._name, "shared_memory")  # the owner unlinks it
        self.mapped.append(shm)
        return shm

    def close_mapped(self):
        for shm in self.mapped:
            shm.close()
        self.mapped = []

    def free_own(self):
        for shm in self.own:
            shm.close()
            shm.unlink()
        self.own = []


def _wait(flags, phase, world, epoch, timeout=60.0):
    t0 = time.time()
    while not (flags[phase] >= epoch).all():
        if time.time() - t0 > timeout:
            raise TimeoutError(f"flags {flags} phase {phase} epoch {epoch}")
        time.sleep(0.001)


class StandInOps:
    """float64 stand-ins for caat_rowpar_tp_local_push / _reduce / _finish_wait (test only)."""

    def __init__(self, H, p, T_max):
        self.H, self.T_max = H, T_max
        self.ns = int(np.floor(H * p))

    def peers(self, world, rank, epoch, recv, gather, flags):
        w = self.ns // world
        return {"world": world, "rank": rank, "epoch": epoch, "w": w,
                "recv": [np.ndarray((world, self.T_max, max(w, 4)), np.float32, buffer=b.buf) for b in recv],
                "gather": [np.ndarray((self.T_max, max(self.ns, 4)), np.float32, buffer=b.buf) for b in gather],
                "flags": [np.ndarray((2, world), np.uint32, buffer=b.buf) for b in flags]}

    def push(self, X_r, W_r, R_r, p, h, pe, *, workspace, private_scale):
        ns, w, r, world = self.ns, pe["w"], pe["rank"], pe["world"]
        Z = X_r.double().numpy() @ W_r.double().numpy().T
        T = Z.shape[0]
        h[:, ns:] = torch.from_numpy(private_scale * Z[:, ns:] + R_r[:, ns:].double().numpy()).to(h.dtype)
        if ns == 0:
            return
        for q in range(world):
            pe["recv"][q][r, :T, :w] = Z[:, q * w:(q + 1) * w].astype(np.float32)
        for q in range(world):
            pe["flags"][q][0, r] = pe["epoch"]

    def reduce(self, T, H, p, pe, *, workspace):
        ns, w, q, world = self.ns, pe["w"], pe["rank"], pe["world"]
        if ns == 0:
            return
        _wait(pe["flags"][q], 0, world, pe["epoch"])
        s = pe["recv"][q][0, :T, :w].copy()
        for r in range(1, world):
            s += pe["recv"][q][r, :T, :w]
        for g in range(world):
            pe["gather"][g][:T, q * w:(q + 1) * w] = s
        for g in range(world):
            pe["flags"][g][1, q] = pe["epoch"]

    def finish(self, R_r, h, gamma, p, out, pe, *, eps):
        ns, r = self.ns, pe["rank"]
        T = h.shape[0]
        if ns:
            _wait(pe["flags"][r], 1, pe["world"], pe["epoch"])
            zs = torch.from_numpy(pe["gather"][r][:T, :ns].astype(np.float64))
            h[:, :ns] = (zs + R_r[:, :ns].double()).to(h.dtype)
        hd = h.double()
        rstd = 1.0 / torch.sqrt((hd * hd).mean(dim=1, keepdim=True) + eps)
        out.copy_((hd * rstd * gamma.double()).to(out.dtype))


def _worker(rank, world, port, p, out_q):
    sys.path.insert(0, ROOT)
    import datetime
    from oracle import caat_oracle as O
    from partial_activation_sync_caat_b200 import inputs as I
    from partial_activation_sync_caat_b200.tp import TPRowParallelP2P, peer_exchange_bytes
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    layer = None
    try:
        T_max, K, H, P = 32, 64, 256, world
        layer = TPRowParallelP2P(H, p, T_max, memory=ShmMemory(), ops=StandInOps(H, p, T_max))
        res = []
        for call, T in enumerate((24, 17)):  # two calls, new inputs, fewer tokens the second time
            d = I.make_rowpar_inputs(T, K, H, P, seed=21 + call, x_std=1.0, w_std=0.1, r_std=1.0, gamma="uniform")
            X_r, W_r, R_r = d["X"][rank].contiguous(), d["W"][rank].contiguous(), d["R"][rank].contiguous()
            out = torch.empty(T, H, dtype=torch.bfloat16)
            h = torch.empty(T, H, dtype=torch.bfloat16)
            layer.forward(X_r, W_r, R_r, d["gamma"], out, h=h, workspace=torch.empty(0))
            ref = O.rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], P, p, return_all=True)
            ok, max_abs, _ = O.within_tolerance(out.float(), ref["out"][rank])
            h_err = float(np.max(np.abs(O._f64(h.float()) - ref["h"][rank])))
            res.append((ok, max_abs, h_err))
        out_q[rank] = (res, layer.epoch, layer.n_s, peer_exchange_bytes(24, H, p, world))
        layer.close()  # unmap, barrier, free
        layer = None
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("p", [0.0, 0.25, 0.5, 1.0])
def test_two_processes_peer_exchange_protocol(p):
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()  # no fork of this (threaded) process
    res = manager.dict()
    mp.start_processes(_worker, args=(world, port, p, res), nprocs=world, start_method="spawn")
    for rank in range(world):
        calls, epoch, ns, nbytes = res[rank]
        assert epoch == 2
        assert ns == int(np.floor(256 * p))
        # each rank sends half its partials and half of the sums: (world - 1) / world of 2 T n_s fp32
        assert nbytes == 2 * 4 * 24 * (ns - ns // world)
        for ok, max_abs, h_err in calls:
            assert ok, f"rank {rank}: max_abs {max_abs}"
            assert h_err < 0.05, f"rank {rank}: h error {h_err}"


def test_peer_exchange_rejects_unaligned_share():
    from partial_activation_sync_caat_b200.tp import TPRowParallelP2P
    with pytest.raises(ValueError):  # floor(200 * 0.5) = 100 is not a multiple of 32
        TPRowParallelP2P(200, 0.5, 16, memory=ShmMemory(), ops=StandInOps(200, 0.5, 16))

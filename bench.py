"""Benchmark of the partially synchronized row-parallel FC2 (7B shape) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl caat|reference]
                    [--workload fc2-7b|fc2-1b|tiny] [--p 0.5] [--sweep]

One step = one call of caat_rowpar_forward on one batch of synthetic input: the P partial
GEMMs, the partial channel-reduce, the private scale, the residual add and the per-rank
RMSNorm.  Default workload: T=8192 tokens, H=4096, K=11008 split over P=8 emulated ranks,
p=0.5 with the first 2048 channels shared (the 7B-scale FC2).  Each step touches 1.34 GB,
more than the 126 MB L2, so no flush is needed between steps.

N > 1 (torchrun): every rank runs its own independent batch of the same workload on its own
GPU (tokens are independent through the whole path: no data-path collective), so per-GPU
work is fixed ("weak" scaling).  Timing: CUDA events around exactly K steps, barrier and
synchronize on both sides, max over ranks.

Prints ONE JSON line on rank 0.  --impl reference times the float64 CPU oracle (the only
reference this method has) on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (T, K, H, P, default p, random S?); for mlp-7b K is the FFN size F
    "fc2-7b": (8192, 11008, 4096, 8, 0.5, False),
    "fc2-1b": (4096, 5632, 2048, 4, 0.5, True),
    "tiny": (256, 768, 768, 2, 0.5, False),
    "mlp-7b": (4096, 11008, 4096, 8, 0.5, False),
    "decode-1": (1, 11008, 4096, 8, 0.5, False),
    "decode-8": (8, 11008, 4096, 8, 0.5, False),
    "decode-64": (64, 11008, 4096, 8, 0.5, False),
    # attention output projection (App. A.1 Eq. 24): the same row-parallel layer with
    # K = heads x head_dim = 4096 (Llama-2-7B: 32 heads of 128), 4 heads per rank
    "attn-out-7b": (8192, 4096, 4096, 8, 0.5, False),
}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------------------
# multi-rank helpers (weak scaling: every rank runs its own independent batch)
# ---------------------------------------------------------------------------------------
def rank_env():
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank (independent problems)."""
    return 1000 + rank


def max_over_ranks(value: float, device: str = "cuda") -> float:
    """The largest value over all ranks (device times: the job ends with its slowest rank)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of all ranks divided by the (max-over-ranks) step time."""
    return world * flops_per_rank_step / ms_per_step / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """sha256 over the sources of the forward GEMM and norm kernels: their headers (with tp.cuh,
    which the GEMM header includes) and the forward launch code of caat_api.cu (from
    launch_rowpar up to validate_rowpar)."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "partial_activation_sync_caat_b200", "csrc")
    for f in ("ptx.cuh", "tp.cuh", "rowpar_common.cuh", "rowpar_gemm.cuh", "rowpar_gemm2.cuh", "rownorm.cuh"):
        h.update(f.encode())
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(d, "caat_api.cu"), "rb") as fh:
        api = fh.read()
    a = api.find(b"caat_status launch_rowpar(")
    b = api.find(b"caat_status validate_rowpar(")
    h.update(api[a:b] if 0 <= a < b else api)
    return h.hexdigest()


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch (read + write) of `kernel` on `workload` from the committed ncu
    record, or None when there is none or the CUDA sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_sha256") != kernel_source_hash():
        return None
    e = rec.get("workloads", {}).get(workload, {}).get(kernel)
    return None if e is None else int(e["read_bytes"] + e["write_bytes"])


L2_BYTES = 126 * 1024 * 1024


def alg_bytes_of(T, K, H, P, mlp=False):
    """Bytes one step must move at least (bf16): the inputs read once and the output written
    once -- X, W, residual and gamma in, out written (h never needs to leave the chip)."""
    if mlp:   # K is the FFN size F: X [P,T,H], A [P,2F/P,H], Y [P,T,F/P] out and in, W2 [P,H,F/P], R, out
        return 2.0 * (P * T * H + 2 * K * H + 2 * T * K + K * H + 2 * P * T * H + H)
    return 2.0 * (T * K + H * K + 2 * P * T * H + H)


def shared_sums_once(case) -> bool:
    """Whether the forward stores the shared channels' cross-rank sums once (fp32) and its norm
    kernel (rownorm_zs_kernel) adds each rank's residual: the library takes that path for a
    contiguous sync set S = the first n_s channels with n_s % 8 == 0, H <= 4096, the CTA-pair
    GEMM (T > 128), the separate norm after the GEMM and the full workspace (CAAT_ZS_SUM=0
    turns it off).  Used to name the norm kernel and count its bytes."""
    from partial_activation_sync_caat_b200 import caat as C
    n_s = int(math.floor(case.H * case.p))
    other = (C.CAAT_FLAG_SINGLE_CTA | C.CAAT_FLAG_FUSED_NORM | C.CAAT_FLAG_OVERLAP_NORM |
             C.CAAT_FLAG_NORM_BESIDE_GEMM | C.CAAT_FLAG_W_PERMUTED | C.CAAT_FLAG_FORCE_DECODE_PATH)
    return (os.environ.get("CAAT_ZS_SUM", "1") != "0" and not case.bwd and not case.rand and
            not (case.flags & other) and 0 < n_s and n_s % 8 == 0 and case.H <= 4096 and case.T > 128)


def alg_flops_of(T, K, H, mlp=False):
    """FLOPs of one step: 2 T K H for the row-parallel GEMM (independent of p); the MLP adds
    FC1's 2 T H 2F (K = F)."""
    return 2.0 * T * K * H + (2.0 * T * H * 2 * K if mlp else 0.0)


def workload_desc(name, T, K, H, P, p, rand):
    layer = ("attention output projection (K = heads x head_dim)" if name.startswith("attn")
             else "row-parallel FC2")
    return (f"{name}: partially synced {layer} + residual + RMSNorm, T={T} H={H} K={K} P={P} "
            f"p={p} ({'seeded random' if rand else 'contiguous'} S)")


# ---------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons sampled during the timed region: NVML polled
    every ~2 ms from a thread (read-only queries), else `nvidia-smi -lms 100`."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.nvml = None
        self.samples = []
        self.stop_flag = False

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.gpu)
        bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            self.nvml = self._nvml_handle()
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _poll(self):
        nv, h = self.nvml
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        try:
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception:
            smax = None
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((sm, smax, pw, [n for n, bt in bits.items() if rs & bt]))
            except Exception:
                break
            time.sleep(0.002)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.stop_flag = True
            if self.thread:
                self.thread.join(timeout=2)
            busy = self.samples
            if not busy:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
            return {"sm_mhz": statistics.median(x[0] for x in busy), "sm_max_mhz": busy[0][1],
                    "samples": len(busy), "source": "NVML, polled every 2 ms",
                    "power_w_max": max(x[2] for x in busy),
                    "reasons": sorted({r for x in busy for r in x[3]})}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(self.NAMES, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------------------
# CPU baseline: the float64 oracle on a bounded row sample
# ---------------------------------------------------------------------------------------
def cpu_baseline(T, K, H, P, p, sync_idx, target_s=10.0, seed=0):
    import numpy as np
    from oracle import caat_oracle as O
    from partial_activation_sync_caat_b200 import inputs as I

    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = len(os.sched_getaffinity(0))
    # a sample of token rows; weights at full size
    n_rows = 16
    d = I.make_rowpar_inputs(min(T, 2048), K, H, P, seed=seed)
    flops_per_row = 2.0 * K * H
    t_total, rows_done = 0.0, 0
    t_rows = d["X"].shape[1]
    start = 0
    while True:
        # consecutive rows of the generated sample, wrapping around it
        rows = (start + np.arange(min(n_rows, t_rows))) % t_rows
        t0 = time.perf_counter()
        O.rowpar_rows(d["X"], d["W"], d["R"], d["gamma"], P, p, rows, sync_idx)
        dt = time.perf_counter() - t0
        t_total += dt
        rows_done += len(rows)
        start = (start + len(rows)) % t_rows
        if t_total >= target_s:
            break
        n_rows = int(max(16, min(2 * n_rows, len(rows) * (target_s - t_total) / max(dt, 1e-3))))
    tflops = flops_per_row * rows_done / t_total / 1e12
    return {"value": tflops, "unit": "TFLOP/s", "cores": int(threads), "kind": "oracle",
            "sample": f"{rows_done} token rows (all {P} ranks, full H={H}, K={K}) of the workload, "
                      f"{t_total:.1f} s of float64 NumPy on the host",
            "tokens_per_s": rows_done / t_total}


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------
class Case:
    """Inputs, workspace and one step (one library call) of a workload on the current GPU."""

    def __init__(self, name, *, tokens=None, p=None, seed=1000, flags=0, no_permute=False, backward=False):
        import torch
        from partial_activation_sync_caat_b200 import caat as C
        from partial_activation_sync_caat_b200 import inputs as I
        T, K, H, P, p_def, rand = WORKLOADS[name]
        if tokens:
            T = tokens
        p = p if p is not None else p_def
        self.name, self.T, self.K, self.H, self.P, self.p, self.rand = name, T, K, H, P, p, rand
        self.mlp = name.startswith("mlp")
        self.bwd = backward and not self.mlp
        self.sync_idx = I.random_sync_idx(H, int((H * p) // 1), seed=0) if rand else None
        self.user_flags = flags
        self.flags = flags
        self.flops = alg_flops_of(T, K, H, self.mlp)
        self.bytes = alg_bytes_of(T, K, H, P, self.mlp)
        if self.mlp:
            self.d = I.make_mlp_inputs(T, H, K, P, seed=seed, device="cuda")
            self.ws = C.alloc_workspace(C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_MLP), "cuda")
        else:
            self.d = I.make_rowpar_inputs(T, K, H, P, seed=seed, device="cuda")
            self.ws = C.alloc_workspace(C.caat_workspace_size(T, K, H, P), "cuda")
        self.out = torch.empty_like(self.d["R"])
        # A random sync list: W's output channels are permuted once (as at weight load time) so
        # that the shared channels are contiguous; every step then runs the permuted path.
        self.permute = rand and not self.mlp and not no_permute and not backward
        self.permute_ms = None
        if self.permute:
            Wp = torch.empty_like(self.d["W"])
            C.caat_permute_weights(self.d["W"], Wp, self.sync_idx, P, p)       # warm-up
            torch.cuda.synchronize()
            pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            st = torch.cuda.current_stream()
            pa.record(st)
            C.caat_permute_weights(self.d["W"], Wp, self.sync_idx, P, p, stream=st)
            pb.record(st)
            torch.cuda.synchronize()
            self.permute_ms = pa.elapsed_time(pb)
            self.d["W"] = Wp
            self.flags |= C.CAAT_FLAG_W_PERMUTED
        if self.bwd:
            # the layer's backward: the forward's h and a random dout are its inputs
            d = self.d
            self.h_saved = torch.empty_like(d["R"])
            C.caat_rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], self.sync_idx, P, p, self.out, workspace=self.ws,
                                  h_out=self.h_saved)
            gen = torch.Generator(device="cuda").manual_seed(seed + 7)
            self.dout = torch.randn(d["R"].shape, generator=gen, device="cuda").to(torch.bfloat16)
            self.dX, self.dW, self.dR = torch.empty_like(d["X"]), torch.empty_like(d["W"]), torch.empty_like(d["R"])
            self.dg = torch.empty(H, dtype=torch.float32, device="cuda")
            self.ws_b = C.alloc_workspace(C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR_BWD), "cuda")
            self.flops = 4.0 * T * K * H
        # Workloads whose bytes fit in L2 get an L2 flush before every timed step (see time_case).
        self.flush = self.bytes < 2 * L2_BYTES and not self.bwd

    def step(self, tm=None, st=None, clear_flags=0):
        import torch
        from partial_activation_sync_caat_b200 import caat as C
        st = torch.cuda.current_stream() if st is None else st
        d, P, p = self.d, self.P, self.p
        fl = self.flags & ~clear_flags
        if self.bwd:
            C.caat_rowpar_backward(d["X"], d["W"], self.h_saved, d["gamma"], self.dout, self.sync_idx, P, p, self.dX,
                                   self.dW, self.dg, dR=self.dR, workspace=self.ws_b, stream=st, timing=tm)
        elif self.mlp:
            C.caat_mlp_forward(d["X"], d["A"], d["W2"], d["R"], d["gamma"], self.sync_idx, P, p, self.out,
                               workspace=self.ws, stream=st, timing=tm, flags=fl)
        else:
            C.caat_rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], self.sync_idx, P, p, self.out,
                                  workspace=self.ws, stream=st, timing=tm, flags=fl)

    def launches_per_call(self, n_intervals):
        """Kernels one call launches (the recorder's intervals, plus the row norm that runs
        beside the GEMM inside the GEMM's interval)."""
        if self.bwd:
            return n_intervals
        overlapped = n_intervals == (2 if self.mlp else 1)
        return n_intervals + (1 if overlapped else 0)


def time_case(case, steps, warmup, world=1, sample_clocks=False, local=0, soak_ms=500.0, warmup_ms=0.0):
    """Times exactly `steps` steps after `warmup` untimed ones: CUDA events on the launching
    stream, synchronize (and a barrier across ranks) on both sides; the per-kernel split comes
    from `steps` more calls with the library's event recorder, after the timed region.  Workloads whose bytes fit
    in L2 (decode, tiny) get a READ of a buffer 3x the L2 size before every step (a write flush
    would leave dirty lines whose write-back the next step would pay for); each step is then
    timed alone, and is one replay of a CUDA graph holding the one library call (the same
    kernels), so that the host's submission after the flush does not leave the GPU idle inside
    the timed interval.  `warmup_ms` > 0: after the `warmup` steps, more untimed steps until that
    much wall time has passed (a part coming out of idle ramps its clocks over some milliseconds).
    Returns (ms_local over all steps, per-call kernel intervals, clocks)."""
    import torch
    import torch.distributed as dist
    from partial_activation_sync_caat_b200 import caat as C
    stream = torch.cuda.current_stream()
    timing = C.Timing(capacity=steps + 8)
    t_w = time.perf_counter()
    for _ in range(warmup):
        case.step()
    torch.cuda.synchronize()
    while (time.perf_counter() - t_w) * 1e3 < warmup_ms:
        for _ in range(4):
            case.step()
        torch.cuda.synchronize()
    if C.caat_get_device_status() != 0:
        raise SystemExit(f"device status set during warm-up of {case.name}")
    flush_buf = torch.ones(3 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if case.flush else None
    graph = None
    if case.flush:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            case.step(st=torch.cuda.current_stream())
        graph.replay()
        torch.cuda.synchronize()
    sampler = ClockSampler(local) if sample_clocks else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if case.flush:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a_ev, b_ev in evs:
            flush_buf.sum()
            a_ev.record(stream)
            graph.replay()
            b_ev.record(stream)
        torch.cuda.synchronize()
        ms_local = sum(a_ev.elapsed_time(b_ev) for a_ev, b_ev in evs)
        for _ in range(steps):   # per-kernel split (not part of the timed value)
            flush_buf.sum()
            case.step(timing)
        torch.cuda.synchronize()
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            case.step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms_local = e0.elapsed_time(e1)
        for _ in range(steps):   # per-kernel split: the library's events around each kernel (an
            case.step(timing)    # event between two kernels holds the second back), not timed
        torch.cuda.synchronize()
    # The timed region is short next to what NVML can sample (tens of ms): keep sampling while
    # the same step runs back to back for a while more (not timed), on every rank.
    soak_steps = 0
    if ms_local < soak_ms:
        soak_steps = int(min(20000, max(1, (soak_ms - ms_local) / max(ms_local / steps, 1e-3))))
        for _ in range(soak_steps):
            if case.flush:
                graph.replay()
            else:
                case.step()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    if clocks is not None:
        clocks["window"] = (f"timed region ({ms_local:.1f} ms) + {soak_steps} more steps of the same work run back "
                            f"to back right after it (not timed)")
    del flush_buf, graph
    per_kernel = timing.read()
    timing.close()
    return ms_local, per_kernel, clocks


def kernel_means(per_kernel):
    n = max((len(r) for r in per_kernel), default=0)
    return [statistics.mean(r[j] for r in per_kernel if len(r) > j) for j in range(n)]


def sequential_split(case, n):
    """The same step with the row norm after the GEMM (without CAAT_FLAG_NORM_BESIDE_GEMM),
    timed per kernel by the library's recorder: what each kernel takes alone (context for the
    overlapped step; not part of the timed value)."""
    import torch
    from partial_activation_sync_caat_b200 import caat as C
    tm = C.Timing(capacity=n + 2)
    for _ in range(2):
        case.step(clear_flags=C.CAAT_FLAG_NORM_BESIDE_GEMM)
    torch.cuda.synchronize()
    for _ in range(n):
        case.step(tm, clear_flags=C.CAAT_FLAG_NORM_BESIDE_GEMM)
    torch.cuda.synchronize()
    km = kernel_means(tm.read())
    tm.close()
    return km


def sub_workloads(args, peaks, peak_src):
    """The other configurations (rank 0, after the headline run), each timed the same way with
    its own clock record: ms (or us) per call, throughput and roofline fraction."""
    import torch
    res = {}
    names = ["fc2-1b", "mlp-7b", "attn-out-7b", "decode-1", "decode-8", "decode-64", "tiny"]
    for name in names:
        case = Case(name, seed=2000)
        # one second idle first: each workload starts from a comparable power state instead of
        # the sustained power cap the previous workload's clock soak left behind
        torch.cuda.synchronize()
        time.sleep(1.0)
        steps = 20
        # 5 warm-up steps, and at least 50 ms of them: the part is coming out of that idle second
        ms_local, per_kernel, clocks = time_case(case, steps, 5, sample_clocks=True, soak_ms=150.0, warmup_ms=50.0)
        ms = ms_local / steps
        km = kernel_means(per_kernel)
        tflops = case.flops / ms / 1e9
        gbs = case.bytes / ms / 1e6
        hbm_bound = case.flops / case.bytes < peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
        e = {"config": workload_desc(name, case.T, case.K, case.H, case.P, case.p, case.rand),
             "ms_per_call": round(ms, 4), "tflops": round(tflops, 1), "hbm_gbs_algorithmic": round(gbs, 1),
             "bound": "hbm" if hbm_bound else "tensor",
             "frac": round(gbs / peaks["hbm_gbs"] if hbm_bound else tflops / peaks["bf16_tflops"], 3),
             "peak": peaks["hbm_gbs"] if hbm_bound else peaks["bf16_tflops"],
             "peak_unit": "GB/s" if hbm_bound else "TFLOP/s", "peak_source": peak_src,
             "kernels_ms": [round(x, 4) for x in km], "l2_flushed": case.flush, "clocks": clocks}
        if case.T <= 64:
            e["us_per_call"] = round(ms * 1e3, 2)
        if case.permute:
            e["w_permuted_once_ms"] = round(case.permute_ms, 4)
        res[name] = e
        del case
        torch.cuda.empty_cache()
    return res


def run_tp(args):
    """--tp: the layer over real devices, one tensor-parallel rank per GPU (P = world size):
    local GEMM step, an NCCL all-reduce (sum, fp32) of the shared channels' partials [T, n_s],
    finishing step (residual + RMSNorm).  Whole-job TFLOP/s of the one layer (2 T K H over the
    max-over-ranks step time), plus the bytes each rank's collective reduces."""
    import datetime
    import torch
    import torch.distributed as dist
    from partial_activation_sync_caat_b200 import build as B
    from partial_activation_sync_caat_b200 import caat as C
    from partial_activation_sync_caat_b200 import inputs as I
    from partial_activation_sync_caat_b200.tp import TPRowParallel, TPRowParallelP2P, exchanged_bytes, peer_exchange_bytes

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if rank == 0:
        B.build()
    else:
        t_wait = time.time()
        while not B.up_to_date():
            if time.time() - t_wait > 900:
                raise SystemExit("libcaat.so was not built by rank 0 within 15 minutes")
            time.sleep(1.0)
    if world == 1:   # a one-rank group without torchrun
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if "MASTER_PORT" not in os.environ:
            import socket
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    C.lib()
    T, K, H, _, p_def, _ = WORKLOADS["fc2-7b"]
    if args.tokens:
        T = args.tokens
    p = args.p if args.p is not None else p_def
    P = world
    if K % P or (K // P) % 8:
        raise SystemExit(f"K={K} does not split over {P} ranks")
    # every rank draws the whole layer's inputs from one seed on its GPU and keeps its slice
    d = I.make_rowpar_inputs(T, K, H, P, seed=0, device="cuda")
    X, W, R = d["X"][rank].contiguous(), d["W"][rank].contiguous(), d["R"][rank].contiguous()
    del d["X"], d["W"], d["R"]
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    ws = C.alloc_workspace(256, "cuda")
    if args.tp_peer:
        # the exchange over peer memory (CUDA IPC buffers, the library's push / reduce / finish)
        layer = TPRowParallelP2P(H, p, T)
        h = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")

        def step():
            layer.forward(X, W, R, d["gamma"], out, h=h, workspace=ws)
    else:
        layer = TPRowParallel(H, p)
        zs, h = layer.buffers(T, "cuda")

        def step():
            layer.forward(X, W, R, d["gamma"], out, zs=zs, h=h, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b)) / args.steps
    status = C.caat_get_device_status()
    dist.barrier()
    if args.tp_peer:
        layer.close()
    dist.destroy_process_group()
    if rank != 0:
        return
    flops = 2.0 * T * K * H
    print(json.dumps({
        "metric": "TFLOP/s of the partially-synced row-parallel FC2 over real devices (one TP rank per GPU)",
        "value": round(flops / ms / 1e9, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"fc2-7b over {P} devices: T={T} H={H} K={K} (K/P={K // P} per rank) p={p}",
                   "parallelism": f"tp{P}"},
        "exchange": ({"collective": "none: partials pushed to their owners' buffers by the GEMM epilogue "
                                    "(peer memory), owners' reduce writes every rank's gather buffer",
                      "bytes_sent_per_rank": peer_exchange_bytes(T, H, p, P), "full_all_reduce_bytes": 4 * T * H}
                     if args.tp_peer else
                     {"collective": "NCCL all-reduce (sum) of the shared channels' fp32 partials",
                      "bytes_per_rank": exchanged_bytes(T, H, p), "full_all_reduce_bytes": 4 * T * H}),
        "gpu_launches": (3 if args.tp_peer else 2) * args.steps, "device_status": status}))


def run_caat(args):
    import torch
    import torch.distributed as dist
    from partial_activation_sync_caat_b200 import build as B
    from partial_activation_sync_caat_b200 import caat as C
    from partial_activation_sync_caat_b200 import inputs as I

    world, rank, local = rank_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    # The library is (re)built by rank 0 before the process group exists, so that a build
    # (a minute or more of nvcc) never runs into the group's timeout; the other ranks wait
    # for it (bounded).
    if rank == 0:
        B.build()
    else:
        t_wait = time.time()
        while not B.up_to_date():
            if time.time() - t_wait > 900:
                raise SystemExit("libcaat.so was not built by rank 0 within 15 minutes")
            time.sleep(1.0)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        dist.barrier()
    C.lib()

    case = Case(args.workload, tokens=args.tokens, p=args.p, seed=rank_seed(rank), flags=args.flags,
                no_permute=args.no_permute, backward=args.backward)
    T, K, H, P, p, rand, mlp, bwd = case.T, case.K, case.H, case.P, case.p, case.rand, case.mlp, case.bwd
    sync_idx, flops = case.sync_idx, case.flops
    stream = torch.cuda.current_stream()

    ms_local, per_kernel, clocks = time_case(case, args.steps, args.warmup, world, sample_clocks=(rank == 0),
                                             local=local)
    ms = max_over_ranks(ms_local)
    kernel_ms = kernel_means(per_kernel)
    n_intervals = len(kernel_ms)
    launches = case.launches_per_call(n_intervals) * args.steps
    status = C.caat_get_device_status()
    # the row norm ran beside the GEMM: one recorded interval holds both kernels
    overlapped = (not bwd) and not case.permute and n_intervals == (2 if mlp else 1)
    split = sequential_split(case, max(5, args.steps // 2)) if overlapped else None

    # optional p sweep (same shapes, fewer steps), rank 0 only
    sweep = None
    if args.sweep and rank == 0 and not mlp and not case.permute and not bwd:   # W permuted for one (p, S) only
        sweep = {}
        d, out, ws = case.d, case.out, case.ws
        for ps in (0.0, 0.25, 0.5, 0.75, 1.0):
            idx_s = I.random_sync_idx(H, int((H * ps) // 1), seed=0) if rand else None
            for _ in range(2):
                C.caat_rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], idx_s, P, ps, out, workspace=ws,
                                      flags=case.flags)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n = max(3, args.steps // 2)
            a.record()
            for _ in range(n):
                C.caat_rowpar_forward(d["X"], d["W"], d["R"], d["gamma"], idx_s, P, ps, out, workspace=ws,
                                      flags=case.flags)
            b.record()
            torch.cuda.synchronize()
            t_ms = a.elapsed_time(b) / n
            sweep[str(ps)] = {"ms_per_step": round(t_ms, 4), "tflops": round(flops / t_ms / 1e9, 1)}

    # end to end through the host-buffer entry point (pinned host tensors, copies timed)
    e2e = None
    if not args.no_e2e and not mlp and not bwd:
        d = case.d
        hX, hW, hR, hg = (d[k].cpu().pin_memory() for k in ("X", "W", "R", "gamma"))
        hout = torch.empty(hR.shape, dtype=torch.bfloat16).pin_memory()
        wsh = C.alloc_workspace(C.caat_workspace_size(T, K, H, P, C.CAAT_VARIANT_ROWPAR_HOST), "cuda")
        for _ in range(2):
            C.caat_rowpar_forward_host(hX, hW, hR, hg, sync_idx, P, p, hout, wsh, stream=stream, flags=case.flags)
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            C.caat_rowpar_forward_host(hX, hW, hR, hg, sync_idx, P, p, hout, wsh, stream=stream, flags=case.flags)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e)
        h2d = sum(x.numel() * 2 for x in (hX, hW, hR, hg))
        d2h = hout.numel() * 2
        e2e = {"value": round(whole_job_tflops(flops, world, e_ms), 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 3),
               "api": "caat_rowpar_forward_host (pinned host buffers; H2D of X, W, residual, gamma and "
                      "D2H of out inside the timed region)"}
        del wsh

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    default_case = not args.tokens and args.p is None and not args.flags  # the recorded ncu case
    ms_step = ms / args.steps
    value = whole_job_tflops(flops, world, ms_step)
    fc2_flops = 2.0 * T * K * H
    kg = 1 if mlp else 0           # index of the row-parallel GEMM's interval (FC1 comes first in the MLP)
    k1_ms = kernel_ms[kg] if len(kernel_ms) > kg else float("nan")
    k2_ms = kernel_ms[kg + 1] if len(kernel_ms) > kg + 1 else None
    k1_tflops = fc2_flops / k1_ms / 1e9
    zs_once = shared_sums_once(case)
    n_s = int(math.floor(H * p))
    # the norm reads h (or, for the shared channels, the fp32 sums and the residual) and writes out
    norm_bytes = 2.0 * P * T * H * 2 + (4.0 * T * n_s if zs_once else 0.0)
    alg_bytes = alg_bytes_of(T, K, H, P)
    if overlapped:
        t_g, t_n = recorded_traffic(args.workload, "gemm"), recorded_traffic(args.workload, "norm_overlapped")
        traffic = (t_g + t_n) if (default_case and t_g is not None and t_n is not None) else None
        kname = ("rowpar_gemm_pair_kernel (tcgen05 cta_group::2 GEMM + partial channel-reduce + residual) with "
                 "rownorm_consumer_kernel (RMSNorm on the SMs the GEMM leaves free) beside it: one overlapped "
                 "interval")
        algo = "2*T*K*H flops per call of the overlapped GEMM + norm"
    else:
        traffic = recorded_traffic(args.workload, "gemm") if default_case else None
        kname = ("rowpar_gemm_pair_kernel (tcgen05 cta_group::2 GEMM + partial channel-reduce "
                 + ("; residual on the private channels, the shared channels' sums stored once in fp32)"
                    if zs_once else "+ residual" + (")" if k2_ms else " + fused RMSNorm)")))
        algo = "2*T*K*H flops per launch"
    result = {
        "metric": "TFLOP/s & tokens/s of partially-synced row-parallel FC2 (7B shape), % bf16 peak",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations and residual, N(0,0.02) weights, gamma=1)",
        "config": {"workload": workload_desc(args.workload, T, K, H, P, p, rand), "T": T, "H": H, "K": K,
                   "P": P, "p": p, "parallelism": f"{world} independent GPU(s), P={P} emulated TP ranks each",
                   "l2": ("step bytes (%.1f MB) fit in L2: read-flush of a %d MB buffer before every step, "
                          "outside the per-step event intervals" % (case.bytes / 1e6, 3 * L2_BYTES // 2**20)
                          if case.flush else
                          "inputs larger than L2 (%.2f GB touched per step); no flush" % (case.bytes / 1e9))},
        "tokens_per_s": round(world * T / (ms_step / 1e3), 1),
        "pct_bf16_peak": {f"{peak_src}_burst": round(100 * value / world / peaks["bf16_tflops"], 1),
                          "datasheet_2250": round(100 * value / world / 2250.0, 1)},
        "roofline": {"kernel": kname, "bound": "tensor", "achieved": round(k1_tflops, 1), "peak": peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} bf16 burst", "unit": "TFLOP/s",
                     "frac": round(k1_tflops / peaks["bf16_tflops"], 3),
                     "frac_vs_sustained": round(k1_tflops / peaks["bf16_tflops_sustained"], 3),
                     "traffic": traffic, "launch_ms": round(k1_ms, 4), "algorithmic": algo},
        "gpu_launches": launches,
        "device_status": status,
        "clocks": clocks,
    }
    result["kernels_ms"] = [round(x, 4) for x in kernel_ms]
    if split is not None:
        sg = split[kg] if len(split) > kg else None
        sn = split[kg + 1] if len(split) > kg + 1 else None
        result["sequential_split"] = {
            "about": "the same call with the norm after the GEMM (no CAAT_FLAG_NORM_BESIDE_GEMM), per-kernel CUDA "
                     "events; not the timed value",
            "gemm_ms": round(sg, 4) if sg else None, "norm_ms": round(sn, 4) if sn else None,
            "gemm_tflops": round(fc2_flops / sg / 1e9, 1) if sg else None,
            "gemm_frac": round(fc2_flops / sg / 1e9 / peaks["bf16_tflops"], 3) if sg else None,
            "norm_gbs": round(norm_bytes / sn / 1e6, 1) if sn else None,
            "norm_frac": round(norm_bytes / sn / 1e6 / peaks["hbm_gbs"], 3) if sn else None,
            "gemm_traffic": recorded_traffic(args.workload, "gemm") if default_case else None,
            "norm_traffic": recorded_traffic(args.workload, "norm") if default_case else None}
    if mlp:
        result["metric"] = "TFLOP/s of the partially-synced MLP block (FC1+SwiGLU+FC2+residual+RMSNorm, 7B shape)"
        result["fc1_kernel"] = {"kernel": "fc1_swiglu_pair_kernel", "launch_ms": round(kernel_ms[0], 4),
                                "achieved_tflops": round(2.0 * T * H * 2 * K / kernel_ms[0] / 1e9, 1)}
    if T <= 64:
        result["decode"] = {"us_per_call": round(ms_step * 1e3, 2), "hbm_gbs": round(alg_bytes / ms_step / 1e6, 1),
                            "frac_of_measured_hbm": round(alg_bytes / ms_step / 1e6 / peaks["hbm_gbs"], 3)}
    if k2_ms and not overlapped:
        result["norm_kernel"] = {"kernel": ("rownorm_zs_kernel" if zs_once else
                                            "rownorm_reg_kernel" if H <= 4096 else "rownorm_kernel"),
                                 "bound": "hbm",
                                 "achieved": round(norm_bytes / k2_ms / 1e6, 1),
                                 "traffic": recorded_traffic(args.workload, "norm") if default_case else None,
                                 "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                 "frac": round(norm_bytes / k2_ms / 1e6 / peaks["hbm_gbs"], 3),
                                 "launch_ms": round(k2_ms, 4),
                                 "algorithmic": ("4*T*n_s + 2*P*T*H*2 bytes (read the shared sums once, the residual "
                                                 "of the shared and h of the private channels; write out)"
                                                 if zs_once else "2*P*T*H*2 bytes (read h, write out)")}
    if args.flags:
        result["config"]["flags"] = hex(args.flags)
    if not mlp:
        # the paper's speed-up model (App. C Eq. 34-35) for this shape: C = operations per exchanged
        # activation from the bf16 GEMM rate and an NVLink rate per direction (bf16 activations on
        # the wire).  The NVLink figure is an assumed constant (this pool's peer-copy figure from
        # its documentation), not measured by this run: every run here has one GPU.
        nvlink_gbs = 770.0
        c_ratio = peaks["bf16_tflops"] * 1e12 / (nvlink_gbs * 1e9 / 2.0)
        sp_m, ps_m = C.caat_speedup_model(H, T, P, p, c_ratio)
        result["speedup_model"] = {"source": "App. C Eq. 34-35", "h": H, "s": T, "r": P, "p": p,
                                   "C_ops_per_activation": round(c_ratio, 1),
                                   "C_inputs": f"{peaks['bf16_tflops']} TFLOP/s {peak_src} bf16 / "
                                               f"({nvlink_gbs} GB/s NVLink per direction, assumed, not measured "
                                               f"here / 2 B)",
                                   "speedup_vs_full_sync": round(sp_m, 4), "p_star": round(ps_m, 4)}
    if bwd:
        norm_names = ["rownorm_bwd_kernel (norm backward + reduction over ranks)", "dgamma_reduce_kernel"]
        if len(kernel_ms) == 4:   # both GEMMs read W, dZt and X MN-major: no transposes
            names = norm_names + ["GEMM dX = dZt W (W MN-major)", "GEMM dW = dZt^T X (dZt, X MN-major)"]
            gemm_idx = (2, 3)
        else:                     # fewer than 129 tokens or channels: K-major operands via transposes
            names = norm_names + ["transpose W", "GEMM dX = dZt W", "transpose dZt", "transpose X",
                                  "GEMM dW = dZt^T X"]
            gemm_idx = (3, 6)
        result["metric"] = "TFLOP/s of the partially-synced row-parallel layer's backward (dX + dW, 4 T K H flop)"
        result["backward_kernels_ms"] = {n: round(x, 4) for n, x in zip(names, kernel_ms)}
        if len(kernel_ms) > max(gemm_idx):
            gx, gw = kernel_ms[gemm_idx[0]], kernel_ms[gemm_idx[1]]
            result["roofline"] = {"kernel": "rowpar_gemm_pair_kernel as the batched dX GEMM", "bound": "tensor",
                                  "achieved": round(fc2_flops / gx / 1e9, 1), "peak": peaks["bf16_tflops"],
                                  "peak_source": f"{peak_src} bf16 burst", "unit": "TFLOP/s",
                                  "frac": round(fc2_flops / gx / 1e9 / peaks["bf16_tflops"], 3),
                                  "traffic": None, "launch_ms": round(gx, 4), "algorithmic": "2*T*K*H flops",
                                  "dW_gemm_tflops": round(fc2_flops / gw / 1e9, 1)}
        result.pop("norm_kernel", None)
    if case.permute:
        result["w_permuted"] = {"api": "caat_permute_weights, once before the steps (weights are static)",
                                "once_ms": round(case.permute_ms, 4)}
    if sweep is not None:
        result["p_sweep"] = sweep
    if e2e is not None:
        result["e2e"] = e2e
    del case
    torch.cuda.empty_cache()
    if world == 1 and not args.no_workloads and args.workload == "fc2-7b" and not args.tokens and not bwd:
        result["workloads"] = sub_workloads(args, peaks, peak_src)
    if not args.no_cpu_baseline and not bwd:
        result["cpu_baseline"] = cpu_baseline(T, K, H, P, p, sync_idx, target_s=args.cpu_seconds)
    print(json.dumps(result))


# ---------------------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import numpy as np
    from oracle import caat_oracle as O
    from partial_activation_sync_caat_b200 import inputs as I

    T, K, H, P, p_def, rand = WORKLOADS[args.workload]
    p = args.p if args.p is not None else p_def
    sync_idx = I.random_sync_idx(H, O.n_sync(H, p), seed=0) if rand else None
    rows_per_step = args.ref_rows
    d = I.make_rowpar_inputs(rows_per_step, K, H, P, seed=0)
    rows = np.arange(rows_per_step)
    for _ in range(args.warmup):
        O.rowpar_rows(d["X"], d["W"], d["R"], d["gamma"], P, p, rows, sync_idx)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.rowpar_rows(d["X"], d["W"], d["R"], d["gamma"], P, p, rows, sync_idx)
    dt = (time.perf_counter() - t0) / args.steps
    flops = 2.0 * rows_per_step * K * H
    value = flops / dt / 1e12
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = len(os.sched_getaffinity(0))
    sample = f"{rows_per_step} token rows per step (all {P} ranks, full H and K) of the workload"
    print(json.dumps({
        "impl": "reference",
        "metric": "TFLOP/s & tokens/s of partially-synced row-parallel FC2 (7B shape), % bf16 peak",
        "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(args.workload, T, K, H, P, p, rand), "T": T, "H": H, "K": K,
                   "P": P, "p": p, "parallelism": "host cores (float64 NumPy oracle)"},
        "tokens_per_s": round(rows_per_step / dt, 2),
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": int(threads), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["caat", "reference"], default="caat")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="fc2-7b")
    ap.add_argument("--p", type=float, default=None)
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling a smaller case)")
    ap.add_argument("--no-permute", action="store_true",
                    help="random sync list: run on the original W (mixed tiles) instead of permuting it once")
    ap.add_argument("--flags", type=lambda x: int(x, 0), default=0, help="CAAT_FLAG_* bits (tuning variants)")
    ap.add_argument("--sweep", action="store_true", help="also time p in {0,.25,.5,.75,1}")
    ap.add_argument("--backward", action="store_true",
                    help="time the layer's backward (caat_rowpar_backward) instead of the forward")
    ap.add_argument("--tp", action="store_true",
                    help="the layer over real devices: one tensor-parallel rank per GPU (P = --gpus), NCCL "
                         "all-reduce of the shared channels")
    ap.add_argument("--tp-peer", action="store_true",
                    help="with --tp: exchange over peer memory (library kernels) instead of NCCL")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload records of the other configurations (fc2-7b default run)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-rows", type=int, default=64)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.tp:
        run_tp(args)
    else:
        run_caat(args)


if __name__ == "__main__":
    main()

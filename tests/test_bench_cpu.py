"""Host logic of bench.py that needs no GPU: the byte counts behind the roofline, the DRAM
traffic record keyed to the kernel sources, and the clock-record parsing."""
import json

import pytest

import bench


def test_algorithmic_bytes_of_the_fc2_7b_step():
    # X [P,T,K/P] + W [P,H,K/P] + residual in + out (bf16) + gamma
    T, K, H, P = 8192, 11008, 4096, 8
    assert bench.alg_bytes_of(T, K, H, P) == 2.0 * (T * K + H * K + 2 * P * T * H + H)
    assert abs(bench.alg_bytes_of(T, K, H, P) / 1e6 - 1344.3) < 0.1


def test_algorithmic_bytes_of_the_mlp_block():
    # X [P,T,H] + A [P,2F/P,H] + Y [P,T,F/P] written and read + W2 [P,H,F/P] + residual + out + gamma
    T, F, H, P = 4096, 11008, 4096, 8
    x = P * T * H
    a = P * (2 * F // P) * H
    y = P * T * (F // P)
    w2 = P * H * (F // P)
    r = out = P * T * H
    assert bench.alg_bytes_of(T, F, H, P, mlp=True) == 2.0 * (x + a + 2 * y + w2 + r + out + H)


def test_algorithmic_flops():
    T, K, H = 8192, 11008, 4096
    assert bench.alg_flops_of(T, K, H) == 2.0 * T * K * H
    assert abs(bench.alg_flops_of(4096, 11008, 4096, mlp=True) / 1e9 - 1108.1) < 0.1


def test_traffic_record_follows_the_sources(monkeypatch, tmp_path):
    rec = {"source_sha256": "abc", "workloads": {"fc2-7b": {"gemm": {"read_bytes": 10, "write_bytes": 5}}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.recorded_traffic("fc2-7b", "gemm") == 15
    assert bench.recorded_traffic("fc2-7b", "norm") is None
    assert bench.recorded_traffic("decode-1", "gemm") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "changed")
    assert bench.recorded_traffic("fc2-7b", "gemm") is None


def test_kernel_source_hash_depends_on_the_forward_kernels(monkeypatch, tmp_path):
    import os
    import shutil
    src = os.path.join(bench.ROOT, "partial_activation_sync_caat_b200", "csrc")
    dst = tmp_path / "partial_activation_sync_caat_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (dst / "backward.cuh").write_text((dst / "backward.cuh").read_text() + "\n// x\n")
    assert bench.kernel_source_hash() == h0            # not a forward kernel
    (dst / "rownorm.cuh").write_text((dst / "rownorm.cuh").read_text() + "\n// x\n")
    assert bench.kernel_source_hash() != h0


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_record_from_nvidia_smi_lines():
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.lines = ["0, 1500, 1965, 900.5, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1400, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1600, 1965, 850.0, 0x0, Not Active, Not Active, Not Active, Not Active",
               "garbage"]
    c = s.stop()
    assert c["sm_mhz"] == 1500 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 980.0


def test_clock_record_from_nvml_samples():
    s = bench.ClockSampler(0)
    s.nvml = (None, None)
    s.samples = [(1500, 1965, 700.0, ["sw_power_cap"]), (1520, 1965, 800.0, []), (1480, 1965, 750.0, [])]
    c = s.stop()
    assert c["sm_mhz"] == 1500 and c["samples"] == 3 and c["reasons"] == ["sw_power_cap"]
    assert c["power_w_max"] == 800.0


def test_shared_sum_norm_rule(monkeypatch):
    """The bench names the norm kernel (and counts its Zs read) from the library's rule for the
    shared-sum path: a contiguous S with n_s % 8 == 0 and n_s > 0, H <= 4096, T > 128, the plain
    forward (no fused / overlapped / beside-the-GEMM norm, no permuted W), CAAT_ZS_SUM not 0."""
    from types import SimpleNamespace
    from partial_activation_sync_caat_b200 import caat as C
    monkeypatch.delenv("CAAT_ZS_SUM", raising=False)

    def case(**kw):
        base = dict(H=4096, p=0.5, T=8192, bwd=False, rand=False, flags=0)
        base.update(kw)
        return SimpleNamespace(**base)

    assert bench.shared_sums_once(case())
    assert bench.shared_sums_once(case(p=1.0))
    assert not bench.shared_sums_once(case(p=0.0))            # no shared channels
    assert not bench.shared_sums_once(case(H=776, p=0.5))     # n_s = 388, not a multiple of 8
    assert not bench.shared_sums_once(case(H=8192))           # rows wider than 4096
    assert not bench.shared_sums_once(case(T=128))            # one-CTA kernel
    assert not bench.shared_sums_once(case(rand=True))        # a sync list (permuted W)
    assert not bench.shared_sums_once(case(bwd=True))
    for f in (C.CAAT_FLAG_FUSED_NORM, C.CAAT_FLAG_OVERLAP_NORM, C.CAAT_FLAG_NORM_BESIDE_GEMM,
              C.CAAT_FLAG_SINGLE_CTA, C.CAAT_FLAG_W_PERMUTED, C.CAAT_FLAG_FORCE_DECODE_PATH):
        assert not bench.shared_sums_once(case(flags=f))
    monkeypatch.setenv("CAAT_ZS_SUM", "0")
    assert not bench.shared_sums_once(case())

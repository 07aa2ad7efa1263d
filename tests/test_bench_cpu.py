"""Host-side pieces of bench.py that need no GPU: the recorded GEMM traffic is reported only for
the workload and GEMM sources it was measured on; throughput and workload descriptions."""
import copy

import pytest

bench = pytest.importorskip("bench")


def test_gemm_traffic_only_for_the_measured_sources(monkeypatch):
    per_launch, per_step = bench.gemm_traffic("llama8b")
    if per_launch is not None:          # the GEMM sources are the measured ones
        assert per_step == bench.GEMM_TRAFFIC["bytes_per_step"]
        assert per_launch == per_step / bench.GEMM_TRAFFIC["launches"]
    assert bench.gemm_traffic("qwen3b_bf16") == (None, None)      # another workload
    changed = copy.deepcopy(bench.GEMM_TRAFFIC)
    changed["sources"]["gemm.cu"] = "0" * 16
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", changed)
    assert bench.gemm_traffic("llama8b") == (None, None)          # sources changed since


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1, 2048, 10, 1000.0) == pytest.approx(20480.0)
    assert bench.job_throughput(8, 2048, 10, 1000.0) == pytest.approx(8 * 20480.0)


def test_workloads_are_described():
    for name in ("llama8b", "qwen3b_bf16", "qwen32b", "tiny", "llama8b_layer"):
        wl = bench.workload(name)
        assert name in bench.describe(wl)

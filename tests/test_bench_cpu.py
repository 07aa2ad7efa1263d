"""Host-side pieces of bench.py that need no GPU: the copy / compute overlap summary of a read
timeline, throughput and workload descriptions."""
import pytest

bench = pytest.importorskip("bench")


def _row(kind, copy, deq, comp):
    return {"layer": 0, "kind": kind, "copy": copy, "dequant": deq, "compute": comp}


def test_timeline_summary_overlap_and_gaps():
    # read 0 copies alone (0-2); read 1's copy (2-4) runs under read 0's compute (2-5); read 2's
    # copy (5-7) is half under read 1's compute (5-6); read 2 computes 7-8, after a 1 ms wait
    tl = [_row("forward", (0.0, 2.0), (1.0, 2.0), (2.0, 5.0)),
          _row("forward", (2.0, 4.0), (4.0, 4.5), (5.0, 6.0)),
          _row("backward", (5.0, 7.0), (None, None), (7.0, 8.0))]
    s = bench.timeline_summary(tl)
    assert s["forward"]["reads"] == 2 and s["backward"]["reads"] == 1
    assert s["forward"]["copy_ms"] == pytest.approx(2.0)
    assert s["forward"]["compute_ms"] == pytest.approx(2.0)
    assert s["backward"]["dequant_ms"] is None
    # hidden copy: read 0 none, read 1 2 ms (under read 0), read 2 1 ms (under read 1) of 6 ms
    assert s["copy_hidden_frac"] == pytest.approx(3.0 / 6.0)
    assert s["compute_gap_ms_total"] == pytest.approx(0.0 + 1.0)
    assert s["first_compute_start_ms"] == 2.0 and s["last_compute_end_ms"] == 8.0


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1, 2048, 10, 1000.0) == pytest.approx(20480.0)
    assert bench.job_throughput(8, 2048, 10, 1000.0) == pytest.approx(8 * 20480.0)


def test_workloads_are_described():
    for name in ("llama8b", "qwen3b_bf16", "qwen32b", "tiny", "llama8b_layer"):
        wl = bench.workload(name)
        assert name in bench.describe(wl)


def test_gemm_traffic_only_for_the_captured_sources(monkeypatch):
    import copy
    from kernel_cases import GEMM_LAUNCHES_PER_STEP
    rec = {"workload": "llama8b", "bytes_per_launch": {c: 1000.0 * (i + 1) for i, c in enumerate(GEMM_LAUNCHES_PER_STEP)},
           "sources": {}}
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", rec)
    assert bench.gemm_traffic("llama8b") == (None, None)            # no hashes recorded
    import hashlib, os
    csrc = os.path.join(bench.ROOT, "layer_streamed_qlora_streaming_b200", "csrc")
    rec2 = copy.deepcopy(rec)
    rec2["sources"] = {f: hashlib.sha256(open(os.path.join(csrc, f), "rb").read()).hexdigest()[:16]
                       for f in ("gemm.cu", "gemm.cuh", "common.cuh")}
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", rec2)
    per_launch, per_step = bench.gemm_traffic("llama8b")
    want = sum(rec["bytes_per_launch"][c] * n for c, n in GEMM_LAUNCHES_PER_STEP.items())
    assert per_step == want and per_launch == want / sum(GEMM_LAUNCHES_PER_STEP.values())
    assert bench.gemm_traffic("qwen3b_bf16") == (None, None)        # another workload
    rec2["sources"]["gemm.cu"] = "0" * 16
    assert bench.gemm_traffic("llama8b") == (None, None)            # sources changed since


def test_recorded_gemm_traffic_covers_the_gemm_sources():
    # the recorded per-shape traffic belongs to the sources in this tree (so the bench line carries
    # it), and its hash gate covers gemm.cu and every local header gemm.cu includes
    import os
    import re
    per_launch, per_step = bench.gemm_traffic("llama8b")
    assert per_launch is not None and per_step > 0
    csrc = os.path.join(bench.ROOT, "layer_streamed_qlora_streaming_b200", "csrc")
    src = open(os.path.join(csrc, "gemm.cu")).read()
    local = set(re.findall(r'#include "([^"]+)"', src))
    assert local <= set(bench.GEMM_TRAFFIC["sources"]), local - set(bench.GEMM_TRAFFIC["sources"])


def test_reference_arm_prints_the_contract_line():
    # `bench.py --impl reference` times the oracle on the host cores and prints one JSON line with
    # the main line's metric and unit, impl "reference", its cpu_baseline and a zero-copy e2e
    import json
    import os
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "0", "--ref-seq", "16"],
                         capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["extrapolated"] is True and d["sample_shape"]["seq"] == 16

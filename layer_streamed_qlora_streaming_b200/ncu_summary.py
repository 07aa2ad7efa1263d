"""Summaries of ncu CSV logs of this library's runs, as printed in the profile notes.

    python -m layer_streamed_qlora_streaming_b200.ncu_summary launches.csv
        per-kernel launches, time and share of one training step (the launches between the last
        two `k_embed` launches of the capture, i.e. the last complete step), library kernels only
    python -m layer_streamed_qlora_streaming_b200.ncu_summary --traffic gemm_traffic.csv
        totals of dram__bytes_read.sum / dram__bytes_write.sum / gpu__time_duration.sum over the
        captured launches, and their average per launch

The input is the `--csv --log-file` output of `ncu --metrics ...`.
"""
from __future__ import annotations

import argparse
import collections
import csv

_SCALE = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "B": 1.0, "KB": 1e3, "MB": 1e6, "GB": 1e9,
          "ns": 1e-9, "us": 1e-6, "ms": 1e-3, "s": 1.0, "nsecond": 1e-9, "usecond": 1e-6, "msecond": 1e-3,
          "second": 1.0}


def read_launches(path: str) -> list[tuple[str, dict]]:
    """[(kernel name, {metric: value in bytes or seconds})] in launch order."""
    with open(path, newline="") as f:
        rows = list(csv.reader(f))
    head = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    h = rows[head]
    ki, mi, ui, vi, ii = (h.index(k) for k in ("Kernel Name", "Metric Name", "Metric Unit", "Metric Value", "ID"))
    by_id: dict[str, tuple[str, dict]] = {}
    order: list[str] = []
    for r in rows[head + 1:]:
        if len(r) <= vi:
            continue
        if r[ii] not in by_id:
            by_id[r[ii]] = (r[ki], {})
            order.append(r[ii])
        by_id[r[ii]][1][r[mi]] = float(r[vi].replace(",", "")) * _SCALE.get(r[ui], 1.0)
    return [by_id[i] for i in order]


def short_name(kernel: str) -> str:
    n = kernel.split("(")[0].replace("void ", "")
    for prefix in ("lst::<unnamed>::", "lst::(anonymous namespace)::", "<unnamed>::", "lst::"):
        n = n.replace(prefix, "")
    return n.strip()


def step_table(path: str) -> str:
    launches = read_launches(path)
    embeds = [i for i, (k, _) in enumerate(launches) if "k_embed" in k]
    if len(embeds) < 2:
        raise SystemExit("need two k_embed launches (one complete step) in the capture")
    step = launches[embeds[-2]:embeds[-1]]
    agg: dict[str, list] = collections.defaultdict(lambda: [0, 0.0])
    for k, m in step:
        if "k_" not in k:       # torch kernels of the caller
            continue
        a = agg[short_name(k)]
        a[0] += 1
        a[1] += m.get("gpu__time_duration.sum", 0.0)
    total = sum(t for _, t in agg.values())
    lines = [f"total {total * 1e3:.2f} ms over {sum(n for n, _ in agg.values())} launches", "",
             "| kernel | launches | ms (ncu) | share |", "|---|---:|---:|---:|"]
    for name, (n, t) in sorted(agg.items(), key=lambda kv: -kv[1][1]):
        lines.append(f"| `{name}` | {n} | {t * 1e3:.2f} | {100 * t / total:.1f}% |")
    return "\n".join(lines)


def traffic_table(path: str) -> str:
    launches = read_launches(path)
    n = len(launches)
    rd = sum(m.get("dram__bytes_read.sum", 0.0) for _, m in launches)
    wr = sum(m.get("dram__bytes_write.sum", 0.0) for _, m in launches)
    t = sum(m.get("gpu__time_duration.sum", 0.0) for _, m in launches)
    return "\n".join([
        "| quantity | total | per launch (average of %d) |" % n, "|---|---:|---:|",
        f"| dram__bytes_read.sum | {rd / 1e9:.2f} GB | {rd / n / 1e6:.1f} MB |",
        f"| dram__bytes_write.sum | {wr / 1e9:.2f} GB | {wr / n / 1e6:.1f} MB |",
        f"| read + write | {(rd + wr) / 1e9:.2f} GB | {(rd + wr) / n / 1e6:.1f} MB |",
        f"| gpu__time_duration.sum | {t * 1e3:.1f} ms | {t / n * 1e6:.0f} us |"])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("csv")
    ap.add_argument("--traffic", action="store_true")
    a = ap.parse_args()
    print(traffic_table(a.csv) if a.traffic else step_table(a.csv))


if __name__ == "__main__":
    main()

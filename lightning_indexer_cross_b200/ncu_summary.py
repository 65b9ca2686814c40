"""Summarise an ncu launch list (gpu__time_duration.sum CSV) per kernel:
launches, total time, mean, share. Usage: python -m lightning_indexer_cross_b200.ncu_summary launches.csv"""
import collections
import csv
import sys

UNIT = {"nsecond": 1e-3, "ns": 1e-3, "usecond": 1.0, "us": 1.0, "msecond": 1e3, "ms": 1e3, "second": 1e6}


def main(path):
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    h = rows[hi]
    ki, mi, vi, ui = (h.index(x) for x in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit"))
    agg = collections.defaultdict(lambda: [0, 0.0])
    for r in rows[hi + 1:]:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        name = r[ki].split("(")[0].replace("void ", "").replace("(anonymous namespace)::", "")
        agg[name][0] += 1
        agg[name][1] += float(r[vi].replace(",", "")) * UNIT.get(r[ui], 1e-3)
    tot = sum(t for _, t in agg.values())
    print(f"{'kernel':58s} {'launches':>8s} {'total_us':>11s} {'mean_us':>9s} {'share':>6s}")
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        print(f"{k[:58]:58s} {n:8d} {t:11.1f} {t / n:9.2f} {t / tot:6.3f}")


if __name__ == "__main__":
    main(sys.argv[1])

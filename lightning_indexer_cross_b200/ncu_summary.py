"""Summaries of ncu CSV output for the committed profile notes.

    python -m lightning_indexer_cross_b200.ncu_summary launches.csv
        per kernel: launches, total time, mean, share (a gpu__time_duration.sum
        launch list)
    python -m lightning_indexer_cross_b200.ncu_summary --traffic dram.csv NAME REGEX SOURCE...
        DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of
        the kernels whose names match REGEX, summed over one launch of each,
        as the traffic block bench.py reads: it records the SHA-256 of the
        kernel SOURCE files, so the figure stops being reported once they change
"""
import collections
import csv
import hashlib
import os
import re
import sys

UNIT = {"nsecond": 1e-3, "ns": 1e-3, "usecond": 1.0, "us": 1.0, "msecond": 1e3, "ms": 1e3, "second": 1e6}
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rows(path):
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    return rows[hi], rows[hi + 1:]


def _name(k):
    return k.split("(")[0].replace("void ", "").replace("(anonymous namespace)::", "")


def launches(path):
    h, body = _rows(path)
    ki, mi, vi, ui = (h.index(x) for x in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit"))
    agg = collections.defaultdict(lambda: [0, 0.0])
    for r in body:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        name = _name(r[ki])
        agg[name][0] += 1
        agg[name][1] += float(r[vi].replace(",", "")) * UNIT.get(r[ui], 1e-3)
    tot = sum(t for _, t in agg.values())
    print(f"{'kernel':58s} {'launches':>8s} {'total_us':>11s} {'mean_us':>9s} {'share':>6s}")
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        print(f"{k[:58]:58s} {n:8d} {t:11.1f} {t / n:9.2f} {t / tot:6.3f}")


def sources_sha256(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()


def traffic(path, name, regex, sources):
    h, body = _rows(path)
    ki, ii, mi, vi = (h.index(x) for x in ("Kernel Name", "ID", "Metric Name", "Metric Value"))
    per = collections.defaultdict(dict)  # launch id -> metric -> value
    kern = {}
    for r in body:
        if len(r) <= vi or not re.search(regex, r[ki]):
            continue
        per[r[ii]][r[mi]] = float(r[vi].replace(",", ""))
        kern[r[ii]] = _name(r[ki])
    first = {}  # one launch of each kernel
    for lid in sorted(per, key=int):
        first.setdefault(kern[lid], per[lid])
    total = 0.0
    for k, m in first.items():
        total += m.get("dram__bytes_read.sum", 0.0) + m.get("dram__bytes_write.sum", 0.0)
    print(f"traffic-kernel: {name}")
    print(f"traffic-sources: {' '.join(sources)}")
    print(f"traffic-sha256: {sources_sha256(sources)}")
    print(f"traffic-dram-bytes-per-launch: {int(total)}")
    for k, m in first.items():
        print(f"traffic-part: {k} read {int(m.get('dram__bytes_read.sum', 0))} write "
              f"{int(m.get('dram__bytes_write.sum', 0))}")


def read_traffic(kernel, profiles_dir):
    """DRAM bytes per launch for `kernel` from the traffic blocks under
    profiles_dir, if one matches the current source hash; else None."""
    if not os.path.isdir(profiles_dir):
        return None
    for fn in sorted(os.listdir(profiles_dir)):
        if not fn.endswith(".md"):
            continue
        text = open(os.path.join(profiles_dir, fn)).read()
        kv = dict(re.findall(r"^traffic-([a-z0-9-]+):\s*(.+)$", text, flags=re.M))
        if kv.get("kernel") != kernel or "dram-bytes-per-launch" not in kv:
            continue
        try:
            if sources_sha256(kv["sources"].split()) != kv["sha256"].strip():
                continue
        except OSError:
            continue
        return int(kv["dram-bytes-per-launch"])
    return None


if __name__ == "__main__":
    if sys.argv[1] == "--traffic":
        traffic(sys.argv[2], sys.argv[3], sys.argv[4], sys.argv[5:])
    else:
        launches(sys.argv[1])

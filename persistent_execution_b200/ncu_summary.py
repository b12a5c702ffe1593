"""Summaries of Nsight Compute output for the profiles/ folder.

    python -m persistent_execution_b200.ncu_summary launches <launches.csv>
    python -m persistent_execution_b200.ncu_summary raw <raw.csv> [metric ...]
    python -m persistent_execution_b200.ncu_summary traffic <config> <metrics.csv | raw.csv> <out.json>

`launches` reads the CSV of a `--metrics gpu__time_duration.sum --csv` run
and prints, per kernel, its launches, total device time and share.
`raw` reads `ncu -i <report> --page raw --csv` and prints the named metrics.
`traffic` writes the DRAM bytes of one persistent-kernel launch (read + write)
with the hash of the kernel sources it was measured on; bench.py reports it
as roofline.traffic only while the sources are unchanged.
"""

from __future__ import annotations

import collections
import csv
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))

DEFAULT_RAW = (
    "gpu__time_duration.sum", "dram__bytes_read.sum", "dram__bytes_write.sum",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed", "sm__throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__warps_active.avg.pct_of_peak_sustained_active", "smsp__issue_active.avg.pct_of_peak_sustained_active",
    "launch__registers_per_thread", "launch__shared_mem_per_block_dynamic", "launch__grid_size",
    "launch__block_size", "lts__t_sector_hit_rate.pct", "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active",
    "smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_barrier_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_membar_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_sleeping_per_issue_active.ratio",
)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(HERE, "csrc")
    for name in sorted(os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def _table(path):
    rows = list(csv.reader(open(path)))
    start = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    return rows[start], rows[start + 1:]


def launches(path) -> str:
    hdr, data = _table(path)
    ki, mi, vi = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    agg = collections.defaultdict(lambda: [0, 0.0])
    for r in data:
        if len(r) > vi and r[mi] == "gpu__time_duration.sum":
            name = r[ki].split("(")[0]
            agg[name][0] += 1
            agg[name][1] += float(r[vi].replace(",", ""))
    tot = sum(v[1] for v in agg.values()) or 1.0
    out = ["| kernel | launches | total ms | share |", "|---|---:|---:|---:|"]
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        out.append(f"| `{k}` | {n} | {t / 1e6:.3f} | {100 * t / tot:.2f}% |")
    return "\n".join(out)


def _col(hdr, name):
    """Column of a metric in a raw-page header, whose names may carry a section prefix."""
    if name in hdr:
        return hdr.index(name)
    for i, h in enumerate(hdr):
        if h.endswith("." + name):
            return i
    return -1


def raw(path, names=DEFAULT_RAW) -> str:
    rows = list(csv.reader(open(path)))
    hdr, units = rows[0], rows[1]
    out = ["| metric | value | unit |", "|---|---:|---|"]
    for r in rows[2:]:
        for n in names:
            i = _col(hdr, n)
            if i >= 0:
                out.append(f"| `{n}` | {r[i]} | {units[i]} |")
    return "\n".join(out)


def _to_bytes(v: str, unit: str) -> float:
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    return float(v.replace(",", "")) * scale.get(unit, 1)


def dram_bytes(path) -> float:
    """Read + write DRAM bytes of the first persistent-kernel launch in a
    metrics CSV (long format) or a raw-page CSV (wide format)."""
    rows = list(csv.reader(open(path)))
    if rows and rows[0] and rows[0][0] == "ID" and "Metric Name" not in rows[0]:  # raw page
        hdr, units, vals = rows[0], rows[1], rows[2]
        return sum(_to_bytes(vals[_col(hdr, m)], units[_col(hdr, m)])
                   for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"))
    hdr, data = _table(path)
    ki, mi, ui, vi = (hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Unit"),
                      hdr.index("Metric Value"))
    tot, seen = 0.0, set()
    for r in data:
        if "persistent" in r[ki] and r[mi] in ("dram__bytes_read.sum", "dram__bytes_write.sum") and r[mi] not in seen:
            tot += _to_bytes(r[vi], r[ui])
            seen.add(r[mi])
    return tot


def main(argv):
    if argv[0] == "launches":
        print(launches(argv[1]))
    elif argv[0] == "raw":
        print(raw(argv[1], tuple(argv[2:]) or DEFAULT_RAW))
    elif argv[0] == "traffic":
        cfg, src, out = int(argv[1]), argv[2], argv[3]
        j = {"config": cfg, "dram_bytes_per_launch": dram_bytes(src), "kernel_source_hash": kernel_source_hash(),
             "source": os.path.basename(src)}
        with open(out, "w") as f:
            json.dump(j, f, indent=1)
        print(json.dumps(j))
    else:
        raise SystemExit(__doc__)


if __name__ == "__main__":
    main(sys.argv[1:])

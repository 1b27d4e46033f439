"""Summarises ncu output for the profiles/ notes.

    python -m kv_cache_sparse_b200.ncu_summary launches <launches.csv>
    python -m kv_cache_sparse_b200.ncu_summary report <file.ncu-rep>
    python -m kv_cache_sparse_b200.ncu_summary traffic <file.ncu-rep> <kernel> <source.cu>

`launches` groups a `--metrics gpu__time_duration.sum` launch list by kernel
(launches, total time, share); `report` prints the counters used for the
rooflines from a saved report (read with `ncu -i ... --page raw --csv`).
"""
from __future__ import annotations

import collections
import csv
import hashlib
import json
import os
import subprocess
import sys

TRAFFIC_FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "profiles", "traffic.json")


def source_digest(path: str) -> str:
    """Digest of a kernel source together with the device headers it includes."""
    h = hashlib.sha256()
    csrc = os.path.dirname(os.path.abspath(path))
    for p in (path, os.path.join(csrc, "sm100.cuh"), os.path.join(csrc, "common.h")):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]

REPORT_KEYS = [
    "gpu__time_duration.sum", "dram__bytes_read.sum", "dram__bytes_write.sum",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_xu.avg.pct_of_peak_sustained_active",
    "sm__pipe_fma_cycles_active.avg.pct_of_peak_sustained_active",
    "sm__pipe_alu_cycles_active.avg.pct_of_peak_sustained_active",
    "smsp__issue_active.avg.pct_of_peak_sustained_active",
    "sm__warps_active.avg.pct_of_peak_sustained_active",
    "dram__throughput.avg.pct_of_peak_sustained_elapsed",
    "lts__throughput.avg.pct_of_peak_sustained_elapsed",
    "launch__registers_per_thread", "launch__grid_size", "launch__block_size",
    "smsp__average_warps_issue_stalled_wait_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_mio_throttle_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_barrier_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_short_scoreboard_per_issue_active.ratio",
]


def launches(path):
    per = collections.OrderedDict()
    with open(path) as f:
        rows = [r for r in csv.reader(f) if len(r) > 10]
    hdr = rows[0]
    ki, mi, vi, ui = (hdr.index("Kernel Name"), hdr.index("Metric Name"),
                      hdr.index("Metric Value"), hdr.index("Metric Unit"))
    for r in rows[1:]:
        if r[mi] != "gpu__time_duration.sum":
            continue
        name = r[ki].split("(")[0].split("<")[0].replace("void ", "").strip()
        name = name.split("::")[-1]
        v = float(r[vi].replace(",", ""))
        scale = {"ns": 1e-3, "us": 1.0, "usecond": 1.0, "nsecond": 1e-3, "ms": 1e3,
                 "msecond": 1e3}.get(r[ui], 1.0)
        n, t = per.get(name, (0, 0.0))
        per[name] = (n + 1, t + v * scale)
    total = sum(t for _, t in per.values())
    print("| kernel | launches | total us | mean us | share |")
    print("|---|---|---|---|---|")
    for name, (n, t) in sorted(per.items(), key=lambda kv: -kv[1][1]):
        print(f"| {name} | {n} | {t:.1f} | {t / n:.2f} | {t / total:.3f} |")


def report(path):
    out = subprocess.run(["ncu", "-i", path, "--page", "raw", "--csv"], capture_output=True,
                         text=True, check=True).stdout
    rows = list(csv.reader(out.splitlines()))
    hdr, units = rows[0], rows[1]
    for r in rows[2:]:
        name = r[hdr.index("Kernel Name")] if "Kernel Name" in hdr else "?"
        print(f"kernel: {name[:90]}")
        for k in REPORT_KEYS:
            if k in hdr:
                i = hdr.index(k)
                print(f"  {k} = {r[i]} {units[i]}")


def traffic(path, kernel, source):
    """Records dram read + write bytes of one captured launch of `kernel`,
    with the digest of its source file, in profiles/traffic.json."""
    out = subprocess.run(["ncu", "-i", path, "--page", "raw", "--csv"], capture_output=True,
                         text=True, check=True).stdout
    rows = list(csv.reader(out.splitlines()))
    hdr, units = rows[0], rows[1]
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    name_col = hdr.index("Kernel Name")
    mine = [r for r in rows[2:] if kernel in r[name_col]]
    if not mine:
        raise SystemExit(f"no launch of {kernel} in {path}")
    r = mine[0]
    total = 0.0
    for k in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
        i = hdr.index(k)
        total += float(r[i].replace(",", "")) * scale[units[i]]
    data = {}
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            data = json.load(f)
    data[kernel] = {"bytes_per_launch": total, "source": os.path.basename(source),
                    "source_sha256_16": source_digest(source)}
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
    print(kernel, total)


if __name__ == "__main__":
    cmd = sys.argv[1]
    if cmd == "traffic":
        traffic(sys.argv[2], sys.argv[3], sys.argv[4])
    else:
        {"launches": launches, "report": report}[cmd](sys.argv[2])

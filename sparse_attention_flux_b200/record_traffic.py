"""Record a kernel's measured DRAM traffic for the bench's roofline line.

    python -m sparse_attention_flux_b200.record_traffic KEY REPORT.ncu-rep --scale S \
        --workload "..." --capture SUMMARY SOURCE [SOURCE ...]

Reads dram__bytes_read.sum and dram__bytes_write.sum of the (single) launch in
an ncu report (``ncu -i REPORT --page raw --csv``), multiplies their sum by S
(for a capture made on a smaller case whose traffic grows in proportion, e.g.
batch 4 standing in for batch 16: S = 4) and stores it under KEY in
profiles/dram_traffic.json together with a SHA-256 of the listed source files'
code (comments and whitespace removed).  bench.py reports the figure only while
that code is unchanged.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")


def dram_bytes(report: str) -> tuple[int, int]:
    out = subprocess.run(["ncu", "-i", report, "--page", "raw", "--csv", "--print-units", "base"],
                         check=True, capture_output=True, text=True).stdout
    rows = list(csv.reader(io.StringIO(out)))
    hdr, units, vals = rows[0], rows[1], rows[2]
    got = []
    for name in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
        i = hdr.index(name)
        if units[i] != "byte":
            raise ValueError(f"{name}: unexpected unit {units[i]!r}")
        got.append(int(float(vals[i].replace(",", ""))))
    return got[0], got[1]


def code_of(text: str) -> str:
    """C++ source with comments and whitespace removed: edits to comments or layout do
    not change what the kernel is.  (The hashed sources hold no "//" or "/*" inside
    string literals.)"""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return re.sub(r"\s+", "", text)


def sources_sha256(sources) -> str:
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(code_of(f.read()).encode())
    return h.hexdigest()


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("key")
    ap.add_argument("report")
    ap.add_argument("sources", nargs="+", help="repo-relative source files of the kernel")
    ap.add_argument("--scale", type=float, default=1.0)
    ap.add_argument("--workload", required=True)
    ap.add_argument("--capture", required=True, help="the summary file of the capture")
    args = ap.parse_args()
    rd, wr = dram_bytes(args.report)
    rec = {}
    if os.path.exists(RECORD):
        with open(RECORD) as f:
            rec = json.load(f)
    rec[args.key] = {
        "workload": args.workload,
        "capture": args.capture,
        "dram_bytes_read": rd,
        "dram_bytes_write": wr,
        "scale": args.scale,
        "bytes_per_launch": int(round((rd + wr) * args.scale)),
        "sources": list(args.sources),
        "sources_sha256": sources_sha256(args.sources),
    }
    with open(RECORD, "w") as f:
        json.dump(rec, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps(rec[args.key], indent=1))


if __name__ == "__main__":
    main()

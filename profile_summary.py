"""Summarise an ncu metrics capture into the JSON record bench.py reads.

    python profile_summary.py --csv CAPTURE.csv --kernels REGEX --per-step N \\
        --sources FILE [FILE ...] --workload NAME --command "NCU COMMAND" --out OUT.json

CAPTURE.csv is ncu's `--csv` output of a `--metrics` run (one row per
launch and metric: "Kernel Name", "Metric Name", "Metric Unit",
"Metric Value").  The launches whose kernel name matches REGEX are taken in
capture order and grouped N at a time (the launches that make up one step of
the timed kernel, e.g. the attention launch, its split tail and the merge);
the record holds, per group, the summed dram__bytes_read.sum +
dram__bytes_write.sum and gpu__time_duration.sum, and the mean over the
groups as `traffic_bytes_per_step`.  `sources` maps each listed source file
to its sha256 at the time the record is written: bench.py uses the traffic
only while every listed file still has that hash, so a record goes stale by
itself when the kernel changes.
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import re

UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
         "nsecond": 1e-9, "usecond": 1e-6, "msecond": 1e-3, "second": 1.0,
         "ns": 1e-9, "us": 1e-6, "ms": 1e-3, "s": 1.0, "%": 1.0}


def sha256(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def read_launches(text: str, kernel_regex: str) -> list[dict]:
    """Per matching launch (capture order): kernel name and its metrics in
    base units (bytes, seconds)."""
    start = text.find('"ID"')
    rows = csv.DictReader(io.StringIO(text[start:] if start >= 0 else text))
    pat = re.compile(kernel_regex)
    launches: dict[str, dict] = {}
    order: list[str] = []
    for r in rows:
        name = r.get("Kernel Name", "")
        if not pat.search(name):
            continue
        lid = r["ID"]
        if lid not in launches:
            launches[lid] = {"kernel": name.split("(")[0].strip(), "metrics": {}}
            order.append(lid)
        unit = (r.get("Metric Unit") or "").strip().lower()
        try:
            v = float(str(r["Metric Value"]).replace(",", ""))
        except ValueError:
            continue
        launches[lid]["metrics"][r["Metric Name"]] = v * UNITS.get(unit, 1.0)
    return [launches[i] for i in order]


def summarise(launches: list[dict], per_step: int) -> dict:
    groups = []
    for g in range(len(launches) // per_step):
        part = launches[g * per_step:(g + 1) * per_step]
        rd = sum(x["metrics"].get("dram__bytes_read.sum", 0.0) for x in part)
        wr = sum(x["metrics"].get("dram__bytes_write.sum", 0.0) for x in part)
        t = sum(x["metrics"].get("gpu__time_duration.sum", 0.0) for x in part)
        groups.append({"kernels": [x["kernel"] for x in part], "dram_read_bytes": rd,
                       "dram_write_bytes": wr, "traffic_bytes": rd + wr, "duration_s": t})
    if not groups:
        raise SystemExit("no complete group of matching launches in the capture")
    return {"groups": groups,
            "traffic_bytes_per_step": round(sum(g["traffic_bytes"] for g in groups) / len(groups))}


def main() -> None:
    p = argparse.ArgumentParser()
    p.add_argument("--csv", required=True)
    p.add_argument("--kernels", required=True)
    p.add_argument("--per-step", type=int, default=1)
    p.add_argument("--sources", nargs="+", required=True)
    p.add_argument("--workload", required=True)
    p.add_argument("--command", required=True)
    p.add_argument("--out", required=True)
    a = p.parse_args()
    rec = {"workload": a.workload, "kernels": a.kernels, "per_step": a.per_step, "command": a.command,
           "sources": {f: sha256(f) for f in a.sources}}
    rec.update(summarise(read_launches(open(a.csv).read(), a.kernels), a.per_step))
    with open(a.out, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps({k: rec[k] for k in ("workload", "traffic_bytes_per_step")}))


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Write the DRAM-traffic record that bench.py reports as ``roofline.traffic``.

    python bench_traffic.py --csv launches.csv --kernel pa_decode_stream_kernel \\
        --source paged_kv_cache_370_b200/csrc/pa_decode.cu --workload llama8b \\
        --pool-blocks 16384 --command "<the ncu command that wrote the CSV>" \\
        --out profiles/pa_decode_llama8b_traffic.json

The CSV is ncu's ``--csv --print-units base`` output of a capture with the
metrics ``dram__bytes_read.sum``, ``dram__bytes_write.sum`` and
``gpu__time_duration.sum``. The record keeps, per launch of the named kernel,
the mean DRAM bytes read and written, together with the algorithmic bytes of
the captured case (computed here from the same seeded workload the capture
ran: one batch, so every captured launch moves the same bytes) and the
SHA-256 of the kernel's source file. bench.py scales the traffic to its own
launches by algorithmic bytes (traffic grows with the tokens processed) and
reports null once the source has changed since the capture.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import json
import os
import re
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

_SCALE = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
          "ns": 1, "nsecond": 1, "usecond": 1e3, "msecond": 1e6, "second": 1e9}


def read_launches(path: str, kernel: str) -> list[dict]:
    """Per launch of kernels whose name matches ``kernel``: metric -> value (base units)."""
    with open(path, newline="") as f:
        lines = f.read().splitlines()
    start = next(i for i, l in enumerate(lines) if l.startswith('"ID"'))
    rows = list(csv.DictReader(lines[start:]))
    by_id: dict[str, dict] = {}
    pat = re.compile(kernel)
    for r in rows:
        if not pat.search(r["Kernel Name"]):
            continue
        unit = (r.get("Metric Unit") or "").strip().lower()
        val = float(r["Metric Value"].replace(",", ""))
        by_id.setdefault(r["ID"], {"kernel": r["Kernel Name"]})[r["Metric Name"]] = \
            val * _SCALE.get(unit, 1)
    return list(by_id.values())


def algorithmic_bytes(workload: str, pool_blocks: int, fused: bool) -> float:
    """Algorithmic bytes of one launch of the captured case."""
    import numpy as np

    import synth
    from paged_kv_cache_370_b200.accounting import decode_step_bytes, new_token_bytes
    if workload == "llama8b":
        b = synth.llama8b(seed=synth.SEED_BASE + 2, variant=0, num_variants=1,
                          num_blocks=pool_blocks)
        total = decode_step_bytes(b.context_lens, b.num_q_heads, b.num_kv_heads, b.head_dim,
                                  b.block_size)["total"]
        return float(total + (new_token_bytes(b.num_seqs, b.num_kv_heads, b.head_dim)
                              if fused else 0))
    if workload == "prefill":
        import bench
        b = synth.llama8b_prefill(seed=synth.SEED_BASE + 7, num_blocks=pool_blocks)
        return float(bench.prefill_flops(b))  # a contraction: FLOPs, not bytes
    raise ValueError(f"unknown workload {workload!r}")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--csv", required=True)
    ap.add_argument("--kernel", required=True, help="regex on the kernel name")
    ap.add_argument("--source", required=True, help="kernel source file (hashed)")
    ap.add_argument("--workload", required=True, choices=["llama8b", "prefill"])
    ap.add_argument("--pool-blocks", type=int, required=True)
    ap.add_argument("--not-fused", action="store_true")
    ap.add_argument("--command", required=True, help="the ncu command that wrote the CSV")
    ap.add_argument("--out", required=True)
    a = ap.parse_args()
    launches = read_launches(a.csv, a.kernel)
    if not launches:
        raise SystemExit(f"no launch of {a.kernel!r} in {a.csv}")
    need = ("dram__bytes_read.sum", "dram__bytes_write.sum", "gpu__time_duration.sum")
    for m in need:
        if any(m not in l for l in launches):
            raise SystemExit(f"metric {m} missing from {a.csv}")
    mean = {m: sum(l[m] for l in launches) / len(launches) for m in need}
    rec = {
        "kernel": launches[0]["kernel"],
        "launches": len(launches),
        "dram_read_bytes_per_launch": round(mean["dram__bytes_read.sum"]),
        "dram_write_bytes_per_launch": round(mean["dram__bytes_write.sum"]),
        "traffic_bytes_per_launch": round(mean["dram__bytes_read.sum"] +
                                          mean["dram__bytes_write.sum"]),
        "gpu_time_ns_per_launch_serialised": round(mean["gpu__time_duration.sum"]),
        "workload": a.workload, "pool_blocks": a.pool_blocks, "fused": not a.not_fused,
        "algorithmic_per_launch": algorithmic_bytes(a.workload, a.pool_blocks, not a.not_fused),
        "algorithmic_unit": "FLOP" if a.workload == "prefill" else "byte",
        "source": os.path.relpath(os.path.abspath(a.source), ROOT),
        "source_sha256": hashlib.sha256(open(a.source, "rb").read()).hexdigest(),
        "command": a.command,
    }
    with open(a.out, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))


if __name__ == "__main__":
    main()

"""Summarise the parity records of a GPU test run.

    WKV_PARITY_RECORD=out.json python -m pytest tests -m gpu
    python tests/parity_report.py out.json > summary.md

Each GPU parity test compares the CUDA path (through the C ABI) with the fp64 oracle, or
with another call of the library where the test says so, and every comparison is recorded
by tests/gpu_util.py.  This script reads only that record file.  Per test it prints the
number of compared tensors, the largest infinity-norm relative error (the gated quantity,
||got - ref||_inf / ||ref||_inf) and the largest floored element-wise relative error
(max |got - ref| / max(|ref|, 1e-3 rms(ref)), reported, never gated).  A comparison a test
labels "expected miss" (one that shows another input path failing the tolerance) is listed
on its own and left out of the per-test maxima.
"""
import json
import sys
from collections import OrderedDict


def main(path):
    with open(path) as f:
        recs = json.load(f)
    by = OrderedDict()
    misses = [r for r in recs if (r.get("what") or "").startswith("expected miss")]
    for r in recs:
        if r in misses:
            continue
        by.setdefault(r["test"], []).append(r)
    print("| test | comparisons | max inf-norm rel | max floored elementwise rel |")
    print("|---|---:|---:|---:|")
    worst = 0.0
    for test, rs in by.items():
        e = max(r["inf_rel"] for r in rs)
        fe = max(r["elem_rel_floored"] for r in rs)
        worst = max(worst, e)
        print(f"| {test} | {len(rs)} | {e:.3e} | {fe:.3e} |")
    n = sum(len(rs) for rs in by.values())
    print(f"\n{n} comparisons in {len(by)} tests; largest inf-norm relative error {worst:.3e}.")
    for r in misses:
        print(f"\nExpected miss, {r['test']} ({r['what']}): inf-norm relative error {r['inf_rel']:.3e}.")


if __name__ == "__main__":
    main(sys.argv[1])

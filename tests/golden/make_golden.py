"""Writes the stored expected values under tests/golden/ from the oracle alone.

index_memory.json -- bytes of the fan-in index store per workload: one int32 per
  (group, slot) when indices are stored once per group, against one per
  (label, slot) for per-label fixed fan-in.  The ratio is the group size G
  ("HASTE: Hardware-Aware Dynamic Sparse Training for Large Output Spaces",
  summary page, Methodology 1, "memory efficiency").
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import oracle as O                       # noqa: E402
from structured_sparse_output_b200 import inputs as I  # noqa: E402


def main():
    rows = {}
    for name, wl in I.WORKLOADS.items():
        rows[name] = {
            "L": wl.L, "G": wl.G, "k": wl.k, "n_groups": wl.n_groups,
            "group_shared_bytes": O.index_bytes(wl.n_groups, wl.k),
            "per_label_bytes": 4 * wl.L * wl.k,
        }
    out = {
        "source": "HASTE summary page, Methodology 1, memory efficiency: indices are "
                  "stored once per group, shrinking index memory by the group size",
        "workloads": rows,
    }
    with open(os.path.join(HERE, "index_memory.json"), "w") as fh:
        json.dump(out, fh, indent=1)
        fh.write("\n")


if __name__ == "__main__":
    main()

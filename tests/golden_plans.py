"""Loader for the hand-derived plan tables under tests/golden/plan_*.txt."""
import glob
import os

from conftest import GOLDEN


def load(path):
    meta, rows = {}, []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                meta[k.strip()] = v.strip()
            else:
                rows.append(tuple(int(x) for x in line.split()))
    shapes = [tuple(int(d) for d in s.split("x")) for s in meta["shapes"].split()]
    totals = dict(kv.split("=") for kv in meta["totals"].split())
    return {
        "name": os.path.basename(path),
        "shapes": shapes,
        "world_size": int(meta["world_size"]),
        "mode": {"flat": 0, "whole": 1}[meta["mode"]],
        "cap_bytes": int(meta["cap_bytes"]),
        "N": int(totals["N"]), "padded": int(totals["padded"]), "C": int(totals["C"]),
        "n_buckets": int(totals["n_buckets"]),
        "owned_numel": [int(x) for x in meta["owned_numel"].split()] if "owned_numel" in meta else None,
        # one group id per tensor (one bucket per group), or None for the cap rule
        "groups": [int(x) for x in meta["groups"].split()] if "groups" in meta else None,
        # bucket tensor owner offset_in_tensor length global_offset owned_offset
        "segments": rows,
    }


def all_golden_plans():
    return [load(p) for p in sorted(glob.glob(os.path.join(GOLDEN, "plan_*.txt")))]

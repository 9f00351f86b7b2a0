"""Writes the stored expected values under tests/golden/ from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
Only `oracle/` and the seeded input generators are called; nothing here runs
the CUDA library.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from grouped_expert_ffn_top_b200 import workloads  # noqa: E402


def tiny_fp32_routing():
    w = workloads.WORKLOADS["tiny_fp32"]
    p = workloads.make_params(w)
    bt = workloads.make_batch(w)
    z = oracle.router_logits_f32(bt["x"].numpy(), p["Wr"].numpy(), p["b"].numpy())
    idx, gw, flags = oracle.route(z.astype(np.float64), w.k)
    lay = oracle.dispatch_layout(idx, w.E, w.ep_groups)
    return {
        "workload": w.name,
        "seed": 0,
        "flags": int(flags),
        "counts": lay["counts"].tolist(),
        "offsets": lay["offsets"].tolist(),
        "group_counts": lay["group_counts"].tolist(),
        "group_offsets": lay["group_offsets"].tolist(),
        "topk_idx_first16": idx[:16].tolist(),
        "pair_of_row_first32": lay["pair_of_row"][:32].tolist(),
    }


def main():
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_routing.json")
    with open(out, "w") as fh:
        json.dump(tiny_fp32_routing(), fh, indent=1)
        fh.write("\n")
    print("wrote", out)


if __name__ == "__main__":
    main()

"""Writes tiny_seed0.json: sampled oracle outputs of the 1024-token workload.

Calls only the oracle (and the seeded input generator).  The fixture is a
regression pin: it freezes the oracle's values so that a later change to the
oracle's arithmetic shows up as a failing test.
Run:  python tests/golden/make_golden.py
"""
import json
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import workloads  # noqa: E402

ROWS = [0, 1, 127, 128, 522, 523, 650, 651, 868, 869, 1023]


def main():
    b = workloads.make_batch("tiny", 0)
    scale = 1.0 / math.sqrt(b.workload.d)
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    out = {
        "what": "oracle forward of the 1024-token, 4-document workload, seed 0, scale 1/sqrt(64)",
        "cu_seqlens": [int(x) for x in b.cu_seqlens],
        "rows": ROWS,
        "lse": {str(r): [float(lse[h, r]) for h in range(b.workload.hq)] for r in ROWS},
        "o_head0_first8": {str(r): [float(x) for x in o[r, 0, :8]] for r in ROWS},
        "n_items": int(len(oracle.tile_list(b.cu_seqlens, 1024, 2))),
    }
    with open(os.path.join(HERE, "tiny_seed0.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()

"""The oracle still reproduces its committed fixture (tests/golden/tiny_seed0.json)."""
import json
import math
import os

import numpy as np

import oracle
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_fixture():
    with open(os.path.join(HERE, "golden", "tiny_seed0.json")) as f:
        g = json.load(f)
    b = workloads.make_batch("tiny", 0)
    assert [int(x) for x in b.cu_seqlens] == g["cu_seqlens"]
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, 1.0 / math.sqrt(64))
    for r in g["rows"]:
        np.testing.assert_allclose(lse[:, r], g["lse"][str(r)], atol=1e-12)
        np.testing.assert_allclose(o[r, 0, :8], g["o_head0_first8"][str(r)], atol=1e-12)
    assert len(oracle.tile_list(b.cu_seqlens, 1024, 2)) == g["n_items"]

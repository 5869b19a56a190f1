"""The two-CTA forward variant (tcgen05 cta_group::2) against the oracle.

With sap_set_forward_variant(1), head_dim 128 and a GQA group that is a multiple of 4, the
forward runs on clusters of two CTAs: one M = 256 MMA per step covers the same q tile of four
query heads of a kv group, and each SM of the pair loads half of every K and V tile.  The result
must match the oracle within the parity bounds (and the one-CTA forward within rounding), on
small cases that span several tiles, chunks, a ragged tail and documents across chunk bounds,
and the backward run on its O and LSE must match too.  The first case is the smallest possible
(one cluster, one kv tile) under a 200 ms wait limit, so that a synchronisation error would end
as a reported timeout within a fraction of a second.
"""
import math

import pytest
import torch

import oracle
import packed_sequence_causal_b200 as sap
import workloads
from gpu_helpers import Run, assert_close, assert_lse

pytestmark = pytest.mark.gpu


def _two_cta(fn):
    sap.sap_set_forward_variant(1)
    try:
        return fn()
    finally:
        sap.sap_set_forward_variant(0)
        sap.sap_set_wait_limit_ns(0)


def _check(lens, hq, hkv, nchunks, seed, bwd=False):
    b = workloads.custom_batch(lens, hq, hkv, 128, seed=seed, with_do=bwd)
    r = Run(b, nchunks)
    o1, l1 = (t.clone() for t in r.fwd())  # one-CTA forward
    o, lse = _two_cta(r.fwd)
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    assert_close(o, ro, "O (two-CTA forward)")
    assert_lse(lse, rl, "LSE (two-CTA forward)")
    assert_close(o, o1.double().cpu().numpy(), "O two-CTA vs one-CTA")
    assert torch.allclose(lse, l1, atol=1e-4, rtol=0)
    if bwd:
        dq, dk, dv = r.bwd()
        rdq, rdk, rdv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, r.scale)
        assert_close(dq, rdq, "dQ (after the two-CTA forward)")
        assert_close(dk, rdk, "dK (after the two-CTA forward)")
        assert_close(dv, rdv, "dV (after the two-CTA forward)")


def test_two_cta_smallest_case_under_a_short_wait_limit():
    b = workloads.custom_batch([128], 4, 1, 128, seed=70, with_do=False)
    r = Run(b, 1)
    r.fwd()  # plan uploaded, one-CTA result

    def run():
        sap.sap_set_wait_limit_ns(200_000_000)
        sap.sap_attn_fwd(r.plan, r.q, r.k, r.v, r.scale, r.o, r.lse, r.ws_fwd)
        return sap.sap_device_status()

    assert _two_cta(run) == 0
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    assert_close(r.o, ro, "O (two-CTA, one tile)")
    assert_lse(r.lse[:, :128], rl, "LSE (two-CTA, one tile)")


@pytest.mark.parametrize("lens,hq,hkv,nchunks,seed", [
    ([1500, 300, 248], 4, 1, 4, 71),             # one kv group, several chunks (partials + merge)
    ([700, 60, 1500, 300, 37, 900, 599], 8, 2, 4, 72),  # two kv groups
    ([10, 500, 490], 8, 1, 1, 73),               # GQA 8, N = 1000: ragged last tile
])
def test_two_cta_forward_matches_oracle(lens, hq, hkv, nchunks, seed):
    _check(lens, hq, hkv, nchunks, seed)


def test_two_cta_forward_then_backward():
    _check([4096, 300, 1200, 1700, 896], 8, 2, 4, 74, bwd=True)


def test_two_cta_falls_back_where_it_does_not_apply():
    """hq / hkv = 2 (not a multiple of 4): the variant switch leaves the one-CTA kernel in place."""
    _check([700, 324], 4, 2, 2, 75)

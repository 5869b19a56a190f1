"""Sequence-parallel rank plans on one GPU, against the oracle element by element.

Every device of a sequence-parallel split runs the library's kernels on its rank plan: windowed
buffers (its chunk's queries; keys and values from the start of the document that reaches into
the chunk), and afterwards adds the fp32 dK/dV partials that later devices computed for its
tokens (sap_attn_bwd_kv_add).  Here all ranks run one after another in one process on one GPU;
the transfers between them are emulated by slicing the batch (the receive leaves the rows before
the span at zero, as the NCCL exchange does) and handing each owner the partial rows of the
other ranks' accumulators.  The assembled O, LSE, dQ, dK, dV must match the oracle of the unsplit
batch within the parity bounds, for balanced and equal cuts, GQA and MHA, d = 64 and 128, and a
ragged last tile.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import assert_close, assert_lse
from packed_sequence_causal_b200 import sap_dist

pytestmark = pytest.mark.gpu


def emulate_ranks(b, nchunks, balanced=True, bounds=None, fused_merge=False):
    """Run every rank plan of the split on this GPU; returns the assembled (O, LSE, dQ, dK, dV)."""
    import packed_sequence_causal_b200 as sap
    n, hq, d = b.q.shape
    hkv = b.k.shape[1]
    q, k, v, do = (t.to("cuda").contiguous() for t in (b.q, b.k, b.v, b.do))
    ranks = [sap_dist.SapAttention(b.cu_seqlens, n, hq, hkv, d, c, nchunks, balanced=balanced, bounds=bounds)
             for c in range(nchunks)]
    if fused_merge:
        for r in ranks:
            sap.sap_plan_set_fused_merge(r.plan, True)
    o = torch.empty_like(q)
    lse = torch.empty((hq, n), dtype=torch.float32, device="cuda")
    for r in ranks:
        w = r.window
        kv0, q0, q1, s0 = w["kv_begin"], w["q_begin"], w["q_end"], w["span_begin"]
        k_win = torch.zeros((q1 - kv0, hkv, d), dtype=k.dtype, device="cuda")
        v_win = torch.zeros_like(k_win)
        k_win[s0 - kv0:] = k[s0:q1]
        v_win[s0 - kv0:] = v[s0:q1]
        o_r, lse_r = r.attend(q[q0:q1].contiguous(), k_win, v_win)
        o[q0:q1] = o_r
        lse[:, q0:q1] = lse_r
    dq = torch.empty_like(q)
    for r in ranks:
        w = r.window
        dq[w["q_begin"]:w["q_end"]] = r.local_backward(do[w["q_begin"]:w["q_end"]].contiguous())
    received = {c: [] for c in range(nchunks)}
    for r in ranks:  # partial dK/dV rows of other ranks' tokens travel back to their owners
        kv0 = r.window["kv_begin"]
        for src, lo, hi in r.recv:
            received[src].append((lo, hi, r._dk_acc[lo - kv0:hi - kv0].clone(),
                                  r._dv_acc[lo - kv0:hi - kv0].clone()))
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    for c, r in enumerate(ranks):
        w = r.window
        dk[w["q_begin"]:w["q_end"]], dv[w["q_begin"]:w["q_end"]] = r.add_partials(received[c])
    torch.cuda.synchronize()
    import packed_sequence_causal_b200 as sap
    assert sap.sap_device_status() == 0
    return o, lse, dq, dk, dv, ranks


def test_forward_parts_equal_the_whole_forward():
    """Own-chunk units (part 1, on a capped grid) then the others (part 2) give the bytes of the
    one-launch forward: the forward is deterministic and the parts write disjoint outputs."""
    import packed_sequence_causal_b200 as sap
    b = workloads.custom_batch([700, 60, 1500, 300, 37, 900, 599], 4, 2, 128, seed=54, with_do=False)
    n = b.q.shape[0]
    q, k, v = (t.to("cuda").contiguous() for t in (b.q, b.k, b.v))
    for c in range(4):
        r = sap_dist.SapAttention(b.cu_seqlens, n, 4, 2, 128, c, 4)
        n_local, n_units = sap.sap_plan_fwd_local_units(r.plan)
        assert 0 <= n_local <= n_units
        w = r.window
        k_win = torch.zeros((w["q_end"] - w["kv_begin"], 2, 128), dtype=k.dtype, device="cuda")
        v_win = torch.zeros_like(k_win)
        k_win[w["span_begin"] - w["kv_begin"]:] = k[w["span_begin"]:w["q_end"]]
        v_win[w["span_begin"] - w["kv_begin"]:] = v[w["span_begin"]:w["q_end"]]
        qr = q[w["q_begin"]:w["q_end"]].contiguous()
        o0, l0 = (t.clone() for t in r.attend(qr, k_win, v_win))
        r.overlap_sms = 100  # part 1 on a grid of far fewer CTAs than SMs
        assert r.attend(qr, k_win, v_win, part=1) is None
        o2, l2 = r.attend(qr, k_win, v_win, part=2)
        assert torch.equal(o0, o2) and torch.equal(l0, l2)
        assert sap.sap_device_status() == 0


def _check(lens, hq, hkv, d, nchunks, balanced=True, seed=0, fused_merge=False):
    b = workloads.custom_batch(lens, hq, hkv, d, seed=seed, with_do=True)
    o, lse, dq, dk, dv, ranks = emulate_ranks(b, nchunks, balanced, fused_merge=fused_merge)
    scale = 1.0 / math.sqrt(d)
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    assert_close(o, ro, "O (rank plans)")
    assert_lse(lse, rl, "LSE (rank plans)")
    rdq, rdk, rdv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    assert_close(dq, rdq, "dQ (rank plans)")
    assert_close(dk, rdk, "dK (rank plans)")
    assert_close(dv, rdv, "dV (rank plans)")
    return ranks


@pytest.mark.parametrize("d", [64, 128])
def test_rank_plans_balanced_gqa(d):
    ranks = _check([700, 60, 1500, 300, 37, 900, 599], 4, 2, d, 4, seed=51)
    # the documents reach across chunk bounds: some rank receives keys from an earlier chunk
    assert any(r.recv for r in ranks)


@pytest.mark.parametrize("d", [64, 128])
def test_rank_plans_equal_chunks_mha(d):
    _check([2100, 50, 1946], 2, 2, d, 4, balanced=False, seed=52)


def test_rank_plans_ragged_tail_and_long_span():
    """N = 5000 (ragged last tile); a 3000-token document spans three chunks, so the last of them
    receives two spans and its window starts inside a kv tile (rows before the span are zeros)."""
    ranks = _check([70, 3000, 1, 929, 1000], 8, 2, 128, 5, seed=53)
    assert max(len(r.recv) for r in ranks) >= 2
    assert any(r.window["kv_begin"] < r.window["span_begin"] for r in ranks if r.recv)


def test_rank_plans_with_fused_merge():
    """Each device's rank plan in fused-merge mode (one forward unit per q tile over every kv chunk
    it sees, received spans included): same result as the oracle."""
    _check([700, 60, 1500, 300, 37, 900, 599], 4, 2, 128, 4, seed=55, fused_merge=True)

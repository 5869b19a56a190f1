"""CUDA path (through the C ABI) against the fp64 oracle, element by element,
on sizes the oracle finishes in seconds: several tiles, GQA and MHA, d = 64
and 128, multiple chunks, ragged documents and a ragged tail, and the
degenerate cases (empty batch, one-token documents, one document, tile-aligned
documents, zero-length documents)."""
import math

import numpy as np
import pytest
import torch

import oracle
import packed_sequence_causal_b200 as sap
import workloads
from gpu_helpers import Run, assert_close, assert_lse, bwd_rounding_bound

pytestmark = pytest.mark.gpu


def _fwd_bwd_full(lens, hq, hkv, d, nchunks, seed=0, scale=None, bwd=True):
    b = workloads.custom_batch(lens, hq, hkv, d, seed=seed, with_do=bwd)
    r = Run(b, nchunks, scale)
    o, lse = r.fwd()
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    assert_close(o, ro, "O")
    assert_lse(lse, rl)
    if bwd:
        dq, dk, dv = r.bwd()
        rdq, rdk, rdv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, r.scale)
        assert_close(dq, rdq, "dQ")
        assert_close(dk, rdk, "dK")
        assert_close(dv, rdv, "dV")
    return r


@pytest.mark.parametrize("seed", [0, 1])
def test_tiny_workload_fwd_merge(seed):
    """1024 tokens, 4 documents (each >= 64), MHA 4 heads, d = 64, P = 2: fwd + merge."""
    b = workloads.make_batch("tiny", seed)
    r = Run(b, b.workload.p)
    o, lse = r.fwd()
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    assert_close(o, ro, "O")
    assert_lse(lse, rl)


def test_partials_match_chunked_oracle():
    """The fp32 partials left in the workspace equal the oracle's per-chunk partial attention."""
    lens = [700, 60, 500, 788]
    b = workloads.custom_batch(lens, 2, 1, 64, seed=3, with_do=False)
    nchunks = 4
    r = Run(b, nchunks)
    sap.sap_attn_fwd(r.plan, r.q, r.k, r.v, r.scale, r.o, r.lse, r.ws_fwd)
    torch.cuda.synchronize()
    _, _, op, lp = oracle.attn_fwd_chunked(b.q, b.k, b.v, b.cu_seqlens, r.scale, nchunks)
    units, _, merges = sap.sap_plan_fwd_schedule(r.plan)
    items = sap.sap_plan_items(r.plan)
    slots = sap.sap_plan_stats(r.plan)["n_partial_slots"]
    assert slots > 0
    hq, d = 2, 64
    ws = r.ws_fwd
    o_part = ws[: slots * hq * 128 * d * 4].view(torch.float32).reshape(slots, hq, 128, d).cpu().double().numpy()
    off = ((slots * hq * 128 * d * 4 + 255) // 256) * 256
    l_part = ws[off: off + slots * hq * 128 * 4].view(torch.float32).reshape(slots, hq, 128).cpu().double().numpy()
    for qt, ib, ic, slot in units:
        if slot < 0:
            continue
        kc = items[ib, 3]
        rows = slice(qt * 128, qt * 128 + 128)
        ref_o = op[kc][rows].transpose(1, 0, 2)      # [hq, 128, d]
        ref_l = lp[kc][:, rows]                      # [hq, 128]
        empty = np.isneginf(ref_l)
        assert np.array_equal(np.isneginf(l_part[slot]), empty)
        np.testing.assert_allclose(l_part[slot][~empty], ref_l[~empty], atol=1e-3)
        np.testing.assert_allclose(o_part[slot], ref_o, atol=5e-3)


@pytest.mark.parametrize("d", [64, 128])
def test_gqa_multichunk(d):
    _fwd_bwd_full([300, 1, 129, 594, 512, 300, 212], 4, 2, d, 4)


@pytest.mark.parametrize("d", [64, 128])
def test_gqa4_three_chunks(d):
    _fwd_bwd_full([1000, 37, 200, 299], 4, 1, d, 3, seed=2)


@pytest.mark.parametrize("d", [64, 128])
def test_mha_ragged_tail(d):
    """N = 1000 is not a multiple of the 128 tile (P = 1)."""
    _fwd_bwd_full([10, 500, 490], 2, 2, d, 1, seed=4)


def test_ragged_smaller_than_a_tile():
    _fwd_bwd_full([30, 47], 2, 1, 128, 1, seed=5)


def test_one_document_is_plain_causal():
    _fwd_bwd_full([640], 2, 1, 64, 5, seed=6)


def test_single_token_documents():
    _fwd_bwd_full([1] * 256, 2, 2, 128, 2, seed=7)


def test_tile_aligned_documents():
    """Documents of exactly 128 tokens: only CAUSAL diagonal tiles."""
    _fwd_bwd_full([128] * 6, 2, 1, 64, 3, seed=8)


def test_zero_length_documents():
    _fwd_bwd_full([0, 200, 0, 0, 312, 0], 2, 2, 64, 2, seed=9)


def test_custom_scale():
    """A softmax scale other than 1/sqrt(d) reaches the kernels (forward and backward)."""
    _fwd_bwd_full([400, 112], 2, 1, 128, 2, seed=10, scale=0.1)


@pytest.mark.parametrize("lens,hq,hkv,nchunks,seed,scale", [
    ([400, 112], 2, 1, 2, 10, 0.37),
    ([256, 384], 2, 2, 1, 11, 1.0 / math.sqrt(8.0)),
])
def test_large_scores(lens, hq, hkv, nchunks, seed, scale):
    """Logits with ~4x the usual spread (scale 0.37 or 1/sqrt(8) on d = 128): exercises the lazy O
    rescaling of the forward, and the backward where the softmax is peaky.

    O and LSE are held to the usual bounds.  dQ and dK get, on top of them, the first-order rounding
    term of bwd_rounding_bound (D_i from the bf16 O, dS rounded to bf16), which grows with the logit
    spread; dV keeps the usual bound."""
    b = workloads.custom_batch(lens, hq, hkv, 128, seed=seed, with_do=True)
    r = Run(b, nchunks, scale)
    o, lse = r.fwd()
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    assert_close(o, ro, "O (large scores)")
    assert_lse(lse, rl, "LSE (large scores)")
    dq, dk, dv = r.bwd()
    rdq, rdk, rdv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, r.scale)
    eq, ek = bwd_rounding_bound(b.q, b.k, b.v, b.do, b.cu_seqlens, r.scale, ro, rl)
    assert_close(dq, rdq, "dQ (large scores)", extra_bound=eq, mean_extra=float(eq.mean()))
    assert_close(dk, rdk, "dK (large scores)", extra_bound=ek, mean_extra=float(ek.mean()))
    assert_close(dv, rdv, "dV (large scores)")


@pytest.mark.parametrize("d", [64, 128])
def test_running_max_grows_along_the_kv_walk(d):
    """Keys of the long document scaled per kv tile by factors from 1 to 4 in a scrambled order, with
    logits about 3x the usual spread: a q tile's running max keeps jumping by more than 2^8 between
    kv steps of one unit, so the forward's lazy O rescale runs at later kv steps -- where, at d = 64,
    the next S has already been issued and the rescale first waits for the previous PV."""
    b = workloads.custom_batch([1500, 300], 4, 2, d, seed=71, with_do=False)
    tile = torch.arange(b.k.shape[0]) // 128
    factor = 1.0 + 3.0 * ((tile * 5) % 11).float() / 10.0
    factor[1500:] = 1.0
    b.k = (b.k.float() * factor[:, None, None]).to(torch.bfloat16)
    r = Run(b, 1, 0.35)
    o, lse = r.fwd()
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    assert_close(o, ro, "O (growing running max)")
    assert_lse(lse, rl, "LSE (growing running max)")


def test_empty_batch_is_a_no_op():
    plan = sap.sap_plan([0], 0, 1)
    z = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((2, 1), dtype=torch.float32, device="cuda")
    ws = sap.alloc_workspace(plan, 2, 2, 64, sap.SAP_WS_BWD)
    sap.sap_attn_fwd(plan, z, z, z, 0.125, z, lse, ws)
    sap.sap_merge(plan, ws, 2, 64, z, lse)
    sap.sap_attn_bwd(plan, z, z, z, z, lse, z, 0.125, z, z, z, ws)
    assert sap.sap_device_status() == 0


def test_repeat_calls_are_identical_forward():
    """Forward has no atomics: two calls give identical bytes."""
    b = workloads.custom_batch([300, 700, 24], 4, 2, 64, seed=12, with_do=False)
    r = Run(b, 1)
    o1, l1 = r.fwd()
    o1, l1 = o1.clone(), l1.clone()
    o2, l2 = r.fwd()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128])
def test_forward_work_order_does_not_change_the_result(d):
    """The forward takes its work items dynamically (a counter in the workspace) or round-robin (no
    workspace, allowed without partial slots), on any grid: every item is computed the same way
    whichever CTA takes it, so all orders give the same bytes.  Fused-merge plan (no slots), GQA 2
    (shared K/V) and MHA (K/V per tile)."""
    for hq, hkv in ((4, 2), (4, 4)):
        b = workloads.custom_batch([900, 40, 1300, 257, 575], hq, hkv, d, seed=45, with_do=False)
        n = b.q.shape[0]  # 3072: three chunks of eight tiles
        q, k, v = (t.to("cuda").contiguous() for t in (b.q, b.k, b.v))
        plan = sap.sap_plan(b.cu_seqlens, n, 3)
        sap.sap_plan_set_fused_merge(plan, True)
        assert sap.sap_plan_stats(plan)["n_partial_slots"] == 0
        ws = sap.alloc_workspace(plan, hq, hkv, d, sap.SAP_WS_FWD, "cuda")
        scale = 1.0 / math.sqrt(d)
        outs = []
        for workspace, max_ctas in ((ws, 0), (ws, 3), (None, 0), (None, 5)):
            o = torch.empty_like(q)
            lse = torch.empty((hq, n), dtype=torch.float32, device="cuda")
            sap.sap_attn_fwd_part(plan, 0, q, k, v, scale, o, lse, workspace, max_ctas=max_ctas)
            outs.append((o, lse))
        assert sap.sap_device_status() == 0
        for o, lse in outs[1:]:
            assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])
        ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
        assert_close(outs[0][0], ro, "O (work orders)")
        assert_lse(outs[0][1], rl, "LSE (work orders)")


def test_workspace_too_small_is_rejected():
    b = workloads.custom_batch([700, 324], 2, 1, 64, seed=13, with_do=True)
    r = Run(b, 8)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(sap.SapError) as e:
        sap.sap_attn_fwd(r.plan, r.q, r.k, r.v, r.scale, r.o, r.lse, small)
    assert e.value.status == -4


def test_long_document_elementwise():
    """A 4096-token document among shorter ones (d = 128, GQA 4, P = 4): every
    element of O, LSE, dQ, dK, dV against the full oracle, with kv tiles that
    loop over 32 q tiles x 4 heads."""
    _fwd_bwd_full([4096, 300, 1200, 1700, 896], 8, 2, 128, 4, seed=21)


@pytest.mark.parametrize("d", [64, 128])
def test_documents_across_backward_bands(d):
    """A kv tile's list longer than 16 q tiles is cut into backward units of one band of 16 q
    tiles (2048 tokens) each, whose fp32 dK/dV partials are summed in the workspace; a shorter
    list is one unit that stores bf16 dK/dV directly.  Here documents start and end inside
    bands and span up to four of them (N = 10240, GQA 2, P = 5), so both kinds of kv tile occur:
    every element against the full oracle."""
    lens = [5000, 1100, 3, 2900, 1237]
    direct = sap.sap_plan_bwd_direct(sap.sap_plan(workloads.cu_seqlens_from_lengths(lens), sum(lens), 5))
    assert 0 < direct.sum() < len(direct)
    _fwd_bwd_full(lens, 4, 2, d, 5, seed=22)


@pytest.mark.parametrize("d", [64, 128])
def test_fused_merge_mode(d):
    """Fused-merge schedule (one pass over all kv chunks of a q-tile): same result as the oracle,
    and within rounding of the chunked path."""
    b = workloads.custom_batch([1500, 300, 248], 4, 2, d, seed=41, with_do=True)
    r = Run(b, 4)
    o_c, l_c = r.fwd()
    o_c, l_c = o_c.clone(), l_c.clone()
    sap.sap_plan_set_fused_merge(r.plan, True)
    o, lse = r.fwd()
    ro, rl = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    assert_close(o, ro, "O (fused merge)")
    assert_lse(lse, rl)
    assert_close(o, o_c.double().cpu().numpy(), "O fused vs chunked")
    dq, dk, dv = r.bwd()
    rdq, rdk, rdv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, r.scale)
    assert_close(dq, rdq, "dQ")
    assert_close(dk, rdk, "dK")
    assert_close(dv, rdv, "dV")


@pytest.mark.parametrize("d", [64, 128])
def test_odd_gqa_group_pairs_heads_with_their_own_kv(d):
    """Group size 3 (odd), 6 query heads: the two-tile forward pairs heads (0, 1), (2, 3), (4, 5),
    and the pair (2, 3) straddles two kv heads, so every tile loads its own K/V tiles; plus the
    backward."""
    _fwd_bwd_full([700, 200, 124], 6, 2, d, 2, seed=42)


@pytest.mark.parametrize("d", [64, 128])
def test_mha_pairs_with_long_kv_lists(d):
    """MHA (4/4 heads): pairs of heads with their own K/V in the two-tile forward, over units of
    up to 7 kv tiles (longer than the K/V rings), P = 3 (N = 2688, seven tiles per chunk)."""
    _fwd_bwd_full([1500, 300, 700, 188], 4, 4, d, 3, seed=43)


@pytest.mark.parametrize("d", [64, 128])
def test_odd_head_count_uses_one_tile_forward(d):
    """3 query heads on one kv head: an odd number of heads cannot be paired, so the one-tile
    forward kernel runs; plus the backward."""
    _fwd_bwd_full([700, 200, 124], 3, 1, d, 2, seed=44)

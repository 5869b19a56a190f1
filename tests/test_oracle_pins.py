"""Pins of the fp64 oracle to things other than itself (CPU only).

* brute force: each document run alone through torch's fp64 scaled-dot-product
  attention (a library routine) and its autograd gradients;
* finite differences of the oracle's own forward for its backward;
* closed forms (Q = 0, one-token documents, constant V);
* invariants from the pages: packing does not leak across documents (SAP/HSAP
  abstract), the chunked computation merged with its LSE equals the plain one
  (sequence-parallel explainer, FAQ on equivalence with one device), softmax
  rows sum to one, and the result does not depend on the number of chunks.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

RNG_CASES = [
    # (doc lengths, hq, hkv, d)
    ([5, 1, 9, 3], 2, 2, 8),
    ([1, 1, 1, 7, 12], 4, 2, 16),
    ([17], 3, 1, 4),
    ([4, 0, 6, 0, 2], 2, 1, 8),  # zero-length documents are allowed and have no effect
]


def _batch(lens, hq, hkv, d, seed=0):
    return workloads.custom_batch(lens, hq, hkv, d, seed=seed)


def _sdpa_per_doc(b, scale, need_grad=False):
    """Library attention per document, fp64 (GQA via enable_gqa)."""
    q = b.q.double().clone().requires_grad_(need_grad)
    k = b.k.double().clone().requires_grad_(need_grad)
    v = b.v.double().clone().requires_grad_(need_grad)
    outs = []
    cu = b.cu_seqlens
    for s, e in zip(cu[:-1], cu[1:]):
        if e == s:
            continue
        qs = q[s:e].permute(1, 0, 2).unsqueeze(0)
        ks = k[s:e].permute(1, 0, 2).unsqueeze(0)
        vs = v[s:e].permute(1, 0, 2).unsqueeze(0)
        o = F.scaled_dot_product_attention(qs, ks, vs, is_causal=True, scale=scale, enable_gqa=True)
        outs.append(o.squeeze(0).permute(1, 0, 2))
    o = torch.cat(outs, 0)
    return q, k, v, o


@pytest.mark.parametrize("lens,hq,hkv,d", RNG_CASES)
def test_fwd_matches_library_attention_per_document(lens, hq, hkv, d):
    b = _batch(lens, hq, hkv, d)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    _, _, _, o_ref = _sdpa_per_doc(b, scale)
    np.testing.assert_allclose(o, o_ref.detach().numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("lens,hq,hkv,d", RNG_CASES)
def test_lse_matches_library_logsumexp_per_document(lens, hq, hkv, d):
    b = _batch(lens, hq, hkv, d, seed=3)
    scale = 0.37
    _, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    G = hq // hkv
    cu = b.cu_seqlens
    for s, e in zip(cu[:-1], cu[1:]):
        if e == s:
            continue
        L = e - s
        mask = torch.ones(L, L, dtype=torch.bool).tril()
        for h in range(hq):
            sc = scale * b.q[s:e, h].double() @ b.k[s:e, h // G].double().T
            ref = torch.logsumexp(sc.masked_fill(~mask, float("-inf")), dim=1)
            np.testing.assert_allclose(lse[h, s:e], ref.numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("lens,hq,hkv,d", RNG_CASES)
def test_bwd_matches_library_autograd_per_document(lens, hq, hkv, d):
    b = _batch(lens, hq, hkv, d, seed=1)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    q, k, v, o = _sdpa_per_doc(b, scale, need_grad=True)
    (o * b.do.double()).sum().backward()
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-11, rtol=0)


def test_bwd_matches_finite_differences():
    lens, hq, hkv, d = [3, 1, 5], 2, 1, 4
    b = _batch(lens, hq, hkv, d, seed=7)
    scale = 0.61
    q, k, v, do = (oracle.widen(b.q, b.k, b.v, b.do))
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, b.cu_seqlens, scale)

    def f(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, b.cu_seqlens, scale)
        return float(np.sum(o * do))

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy()
            xp[idx] += eps
            xm = x.copy()
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (f(args_p["q"], args_p["k"], args_p["v"]) - f(args_m["q"], args_m["k"], args_m["v"])) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, rtol=0, err_msg=name)


def test_closed_form_zero_queries():
    """Q = 0: uniform weights over the document prefix, LSE = log(prefix length)."""
    lens, hq, hkv, d = [6, 1, 4], 2, 1, 8
    b = _batch(lens, hq, hkv, d)
    q0 = torch.zeros_like(b.q)
    o, lse = oracle.attn_fwd(q0, b.k, b.v, b.cu_seqlens, 0.3)
    v = b.v.double().numpy()
    cu = b.cu_seqlens
    for s, e in zip(cu[:-1], cu[1:]):
        for i in range(s, e):
            for h in range(hq):
                np.testing.assert_allclose(o[i, h], v[s:i + 1, 0].mean(0), atol=1e-14)
                assert abs(lse[h, i] - math.log(i - s + 1)) < 1e-14


def test_closed_form_single_token_documents():
    """Every document of length 1: O = V of its group, LSE = S_ii; dQ = dK = 0, dV = sum of dO over the group."""
    n, hq, hkv, d = 9, 4, 2, 8
    b = _batch([1] * n, hq, hkv, d, seed=5)
    scale = 0.25
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    q, k, v, do = (t.double().numpy() for t in (b.q, b.k, b.v, b.do))
    G = hq // hkv
    for h in range(hq):
        np.testing.assert_allclose(o[:, h], v[:, h // G], atol=1e-14)
        np.testing.assert_allclose(lse[h], scale * np.sum(q[:, h] * k[:, h // G], -1), atol=1e-13)
    dq, dk, dv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14
    for g in range(hkv):
        np.testing.assert_allclose(dv[:, g], do[:, g * G:(g + 1) * G].sum(1), atol=1e-13)


def test_closed_form_constant_values():
    """Constant V: O = V, and dQ = dK = 0 exactly (softmax rows sum to one)."""
    lens, hq, hkv, d = [7, 2, 5], 2, 2, 4
    b = _batch(lens, hq, hkv, d, seed=9)
    vc = torch.ones_like(b.v) * torch.tensor([0.5, -1.25, 2.0, 3.0]).to(torch.bfloat16)
    o, _ = oracle.attn_fwd(b.q, b.k, vc, b.cu_seqlens, 0.4)
    np.testing.assert_allclose(o, np.broadcast_to([0.5, -1.25, 2.0, 3.0], o.shape), atol=1e-13)
    dq, dk, _ = oracle.attn_bwd(b.q, b.k, vc, b.do, b.cu_seqlens, 0.4)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12


def test_closed_form_hand_example():
    """A 3-token, 2-document, d = 1 example worked by hand.

    q = [1, 2, 0], k = [1, 0, 3], v = [1, 2, 5], scale 1, docs [0,2) and [2,3).
    row 0 sees key 0: S = 1, O = 1, LSE = 1.
    row 1 sees keys 0,1: S = (2, 0), LSE = log(e^2 + 1), O = (e^2 + 2) / (e^2 + 1).
    row 2 sees key 2 only: S = 0, O = 5, LSE = 0.
    With dO = 1: P_1 = (e^2, 1)/(e^2+1), D_1 = O_1, dS_1 = P_1 * ((1, 2) - D_1);
    dQ_1 = dS_10 * k_0, dK_0 = dS_10 * q_1, dK_1 = dS_11 * q_1, dV_0 = 1 + P_10,
    dV_1 = P_11, dV_2 = 1, and the other gradients are 0.
    """
    t = lambda x: torch.tensor(x, dtype=torch.float64).reshape(3, 1, 1)
    q, k, v, do = t([1.0, 2.0, 0.0]), t([1.0, 0.0, 3.0]), t([1.0, 2.0, 5.0]), t([1.0, 1.0, 1.0])
    cu = [0, 2, 3]
    o, lse = oracle.attn_fwd(q, k, v, cu, 1.0)
    e2 = math.exp(2.0)
    np.testing.assert_allclose(o[:, 0, 0], [1.0, (e2 + 2) / (e2 + 1), 5.0], atol=1e-15)
    np.testing.assert_allclose(lse[0], [1.0, math.log(e2 + 1), 0.0], atol=1e-15)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, cu, 1.0)
    p10, p11 = e2 / (e2 + 1), 1 / (e2 + 1)
    d1 = (e2 + 2) / (e2 + 1)
    ds10, ds11 = p10 * (1 - d1), p11 * (2 - d1)
    np.testing.assert_allclose(dq[:, 0, 0], [0.0, ds10 * 1.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(dk[:, 0, 0], [ds10 * 2.0, ds11 * 2.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(dv[:, 0, 0], [1 + p10, p11, 1.0], atol=1e-15)


@pytest.mark.parametrize("seed", [0, 1])
def test_packed_equals_each_document_alone(seed):
    """No cross-contamination: the packed result equals running every document by itself."""
    b = _batch([9, 1, 14, 6], 4, 2, 8, seed=seed)
    scale = 0.35
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    dq, dk, dv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    cu = b.cu_seqlens
    for s, e in zip(cu[:-1], cu[1:]):
        sl = slice(s, e)
        cu1 = [0, e - s]
        o1, l1 = oracle.attn_fwd(b.q[sl], b.k[sl], b.v[sl], cu1, scale)
        np.testing.assert_array_equal(o[sl], o1)
        np.testing.assert_array_equal(lse[:, sl], l1)
        g1 = oracle.attn_bwd(b.q[sl], b.k[sl], b.v[sl], b.do[sl], cu1, scale)
        np.testing.assert_allclose(dq[sl], g1[0], atol=1e-14)
        np.testing.assert_allclose(dk[sl], g1[1], atol=1e-14)
        np.testing.assert_allclose(dv[sl], g1[2], atol=1e-14)


@pytest.mark.parametrize("nchunks", [1, 2, 4, 8])
def test_chunked_merge_equals_unchunked(nchunks):
    """Partials over kv chunks merged through their LSE equal the plain result to 1e-12."""
    b = workloads.custom_batch([40, 3, 70, 15], 2, 1, 16, seed=2)
    scale = 0.25
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    oc, lc, op, lp = oracle.attn_fwd_chunked(b.q, b.k, b.v, b.cu_seqlens, scale, nchunks)
    np.testing.assert_allclose(oc, o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lc, lse, atol=1e-12, rtol=0)
    # a row never sees keys of a later chunk: those partials are empty
    c = 128 // nchunks
    for bb in range(nchunks):
        assert np.all(np.isneginf(lp[bb][:, : bb * c]))
        assert np.all(op[bb][: bb * c] == 0)


def test_merge_special_cases():
    """Merging with an empty partial is the identity; two equal partials add log 2 to the LSE."""
    rng = np.random.default_rng(0)
    o1 = rng.normal(size=(1, 5, 2, 3))
    l1 = rng.normal(size=(1, 2, 5))
    empty_o = np.zeros_like(o1)
    empty_l = np.full_like(l1, -np.inf)
    o, l = oracle.merge(np.concatenate([o1, empty_o]), np.concatenate([l1, empty_l]))
    np.testing.assert_allclose(o, o1[0], atol=1e-15)
    np.testing.assert_allclose(l, l1[0], atol=1e-15)
    o, l = oracle.merge(np.concatenate([o1, o1]), np.concatenate([l1, l1]))
    np.testing.assert_allclose(o, o1[0], atol=1e-15)
    np.testing.assert_allclose(l, l1[0] + math.log(2.0), atol=1e-14)


def test_gqa_equals_mha_with_repeated_kv():
    """kv head of q head h is floor(h / G): GQA equals MHA over K, V repeated G times per head."""
    b = _batch([11, 5, 8], 6, 2, 8, seed=4)
    scale = 0.3
    G = 3
    kr = b.k.repeat_interleave(G, dim=1)
    vr = b.v.repeat_interleave(G, dim=1)
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    o2, lse2 = oracle.attn_fwd(b.q, kr, vr, b.cu_seqlens, scale)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    dq, dk, dv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    dq2, dk2, dv2 = oracle.attn_bwd(b.q, kr, vr, b.do, b.cu_seqlens, scale)
    np.testing.assert_allclose(dq, dq2, atol=1e-14)
    np.testing.assert_allclose(dk, dk2.reshape(dk2.shape[0], 2, G, 8).sum(2), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(dv2.shape[0], 2, G, 8).sum(2), atol=1e-13)


def test_sampled_rows_match_full():
    b = _batch([30, 2, 50, 18], 4, 2, 8, seed=6)
    scale = 0.35
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    rows = [0, 29, 30, 31, 45, 99]
    heads = [0, 3]
    orow, lrow = oracle.attn_fwd_rows(b.q, b.k, b.v, b.cu_seqlens, scale, rows, heads)
    for a, r in enumerate(rows):
        for t, h in enumerate(heads):
            np.testing.assert_allclose(orow[a, t], o[r, h], atol=1e-14)
            assert abs(lrow[a, t] - lse[h, r]) < 1e-14
    dq, dk, dv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    for g in (0, 1):
        sq, sk, sv = oracle.attn_bwd_sampled(b.q, b.k, b.v, b.do, b.cu_seqlens, scale, g, rows, rows)
        for a, r in enumerate(rows):
            np.testing.assert_allclose(sq[a], dq[r, 2 * g:2 * g + 2], atol=1e-13)
            np.testing.assert_allclose(sk[a], dk[r, g], atol=1e-13)
            np.testing.assert_allclose(sv[a], dv[r, g], atol=1e-13)


def test_rejects_bad_seqlens():
    b = _batch([4, 4], 1, 1, 4)
    with pytest.raises(ValueError):
        oracle.attn_fwd(b.q, b.k, b.v, [0, 3, 7], 1.0)      # does not end at N
    with pytest.raises(ValueError):
        oracle.attn_fwd(b.q, b.k, b.v, [1, 4, 8], 1.0)      # does not start at 0
    with pytest.raises(ValueError):
        oracle.attn_fwd(b.q, b.k, b.v, [0, 5, 4, 8], 1.0)   # decreasing
    with pytest.raises(ValueError):
        oracle.tile_list([0, 100], 100, 3)                   # N not divisible by P
    with pytest.raises(ValueError):
        oracle.tile_list([0, 256], 256, 4)                   # chunk 64 not a multiple of the tile

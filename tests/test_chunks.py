"""Explicit and balanced chunk partitions, rank plans and their exchange lists (CPU only).

Pins of the oracle's balanced cut: on small batches every composition of the
q tiles into P non-empty contiguous parts is enumerated, with the work of a q
tile counted from the dense mask; the oracle must return the smallest possible
largest part and, among the cuts that reach it, the lexicographically largest
bounds.  The planner must then agree with the oracle bit for bit: the bounds,
the tile list over those bounds, and every rank plan's items.  Rank windows
and exchange lists are checked against the dense mask: the keys that a
chunk's queries may see and that lie before the chunk are exactly the spans
the chunk's owner receives.
"""
import itertools

import numpy as np
import pytest

import oracle
import packed_sequence_causal_b200 as sap
import workloads


def _dense_mask(cu, n):
    doc = np.repeat(np.arange(len(cu) - 1), np.diff(cu))
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    return (doc[:, None] == doc[None, :]) & (j <= i)


def _tile_work(cu, n, block):
    """Non-empty (q tile, kv tile) boxes per q tile, from the dense mask."""
    mask = _dense_mask(cu, n)
    T = (n + block - 1) // block
    work = np.zeros(T, dtype=np.int64)
    for qt in range(T):
        for kt in range(T):
            if mask[qt * block:(qt + 1) * block, kt * block:(kt + 1) * block].any():
                work[qt] += 1
    return work


def _brute_force_cut(work, nchunks):
    """(best max part work, lexicographically largest optimal interior bounds in tiles)."""
    T = len(work)
    pre = np.concatenate([[0], np.cumsum(work)])
    best, best_cuts = None, []
    for cuts in itertools.combinations(range(1, T), nchunks - 1):
        b = (0,) + cuts + (T,)
        m = max(pre[b[k + 1]] - pre[b[k]] for k in range(nchunks))
        if best is None or m < best:
            best, best_cuts = m, [cuts]
        elif m == best:
            best_cuts.append(cuts)
    return best, max(best_cuts)


def _random_batch(seed, block):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(4, 11))
    n = T * block - int(rng.integers(0, block // 2))  # ragged last tile half of the time
    lens = []
    while sum(lens) < n:
        lens.append(int(min(n - sum(lens), rng.integers(1, 4 * block))))
    return workloads.cu_seqlens_from_lengths(lens), n


@pytest.mark.parametrize("seed", range(12))
def test_oracle_balanced_cut_is_the_lexicographically_largest_optimal_cut(seed):
    block = 16
    cu, n = _random_batch(seed, block)
    T = (n + block - 1) // block
    work = _tile_work(cu, n, block)
    for nchunks in range(1, min(T, 5) + 1):
        b = oracle.balanced_bounds(cu, n, nchunks, block)
        best, cuts = _brute_force_cut(work, nchunks)
        assert b[0] == 0 and b[-1] == n
        assert tuple(int(x) // block for x in b[1:-1]) == cuts
        pre = np.concatenate([[0], np.cumsum(work)])
        tb = [0] + [int(x) // block for x in b[1:-1]] + [T]
        assert max(pre[tb[k + 1]] - pre[tb[k]] for k in range(nchunks)) == best


def test_oracle_balanced_cut_errors():
    cu = workloads.cu_seqlens_from_lengths([100, 28])
    with pytest.raises(ValueError):
        oracle.balanced_bounds(cu, 128, 9, 16)  # more chunks than tiles
    with pytest.raises(ValueError):
        oracle.balanced_bounds(cu, 128, 0, 16)
    np.testing.assert_array_equal(oracle.balanced_bounds([0], 0, 1, 16), [0, 0])


@pytest.mark.parametrize("seed", range(12))
def test_planner_balanced_cut_matches_oracle_random(seed):
    block = 16
    cu, n = _random_batch(seed, block)
    T = (n + block - 1) // block
    for nchunks in range(1, min(T, 6) + 1):
        np.testing.assert_array_equal(sap.sap_balanced_chunks(cu, n, nchunks, block),
                                      oracle.balanced_bounds(cu, n, nchunks, block))


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
def test_planner_balanced_cut_matches_oracle_workloads(name):
    w = workloads.WORKLOADS[name]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    for nchunks in sorted({2, 4, w.p}):
        b = sap.sap_balanced_chunks(cu, w.n, nchunks)
        np.testing.assert_array_equal(b, oracle.balanced_bounds(cu, w.n, nchunks))
        plan = sap.sap_plan_chunks(cu, w.n, b)
        np.testing.assert_array_equal(sap.sap_plan_items(plan), oracle.tile_list(cu, w.n, nchunks, bounds=b))
        np.testing.assert_array_equal(sap.sap_plan_chunk_bounds(plan), b)


@pytest.mark.parametrize("name,nchunks", [("llama31_8b_128k", 8), ("hybrid_512k", 16), ("llama32_1b_32k", 8),
                                          ("llama2_13b_64k_short", 16)])
def test_balanced_cut_evens_out_the_work(name, nchunks):
    """Per-chunk item counts and unmasked pairs: max / mean <= 1.1 with the balanced cut (equal
    chunks reach ~3x at 128K and 512K)."""
    w = workloads.WORKLOADS[name]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    plan = sap.sap_plan_chunks(cu, w.n, sap.sap_balanced_chunks(cu, w.n, nchunks))
    st = sap.sap_plan_chunk_stats(plan)
    items, pairs = st["items"], st["pairs"]
    assert items.sum() == len(sap.sap_plan_items(plan))
    assert pairs.sum() == oracle.unmasked_pairs(cu)
    assert items.max() / items.mean() <= 1.1, items
    assert pairs.max() / pairs.mean() <= 1.1, pairs
    eq = sap.sap_plan_chunk_stats(sap.sap_plan(cu, w.n, nchunks))["items"]
    assert items.max() <= eq.max()


def test_explicit_chunks_reject_bad_bounds():
    cu = workloads.cu_seqlens_from_lengths([300, 212])
    for bad in ([0, 100, 512], [0, 256, 256, 512], [0, 256, 500], [1, 256, 512], [0, 384, 256, 512]):
        with pytest.raises(sap.SapError) as e:
            sap.sap_plan_chunks(cu, 512, bad)
        assert e.value.status == -3
    assert len(sap.sap_plan_items(sap.sap_plan_chunks(cu, 512, [0, 256, 512]))) > 0


def _check_rank_plans(cu, n, bounds, block=128):
    full = sap.sap_plan_chunks(cu, n, bounds, block, block)
    items = sap.sap_plan_items(full)
    nchunks = len(bounds) - 1
    mask_starts = np.zeros(n, dtype=np.int64)
    for s, e in zip(cu[:-1], cu[1:]):
        mask_starts[s:e] = s
    total_pairs = 0
    for c in range(nchunks):
        r = sap.sap_plan_rank(full, c)
        mine = items[items[:, 2] == c]
        np.testing.assert_array_equal(sap.sap_plan_items(r), mine)
        win = sap.sap_plan_window(r)
        q0, q1 = int(bounds[c]), int(bounds[c + 1])
        assert (win["q_begin"], win["q_end"]) == (q0, q1)
        # the earliest key any query of the chunk may see, and its tile
        assert win["span_begin"] == int(mask_starts[q0:q1].min())
        assert win["kv_begin"] == win["span_begin"] // block * block
        if len(mine):
            assert mine[:, 1].min() * block >= win["kv_begin"]
        # exchange list = the earlier chunks' keys in [span_begin, q0), split by owner
        spans = sap.sap_plan_rank_spans(full, c)
        need = np.zeros(n, dtype=bool)
        for i in range(q0, q1):
            need[mask_starts[i]:min(i + 1, q0)] = True
        got = np.zeros(n, dtype=bool)
        for src, lo, hi in spans:
            assert bounds[src] <= lo < hi <= bounds[src + 1] and src < c
            assert not got[lo:hi].any()
            got[lo:hi] = True
        np.testing.assert_array_equal(got, need)
        # the sources are exactly the earlier kv chunks of this q chunk's chunk pairs
        assert sorted(int(s) for s in spans[:, 0]) == sorted({int(x) for x in mine[:, 3]} - {c})
        st = sap.sap_plan_stats(r)
        pairs = int(sum(i - mask_starts[i] + 1 for i in range(q0, q1)))
        assert st["unmasked_pairs"] == pairs
        total_pairs += pairs
        assert sap.sap_plan_chunk_stats(full)["pairs"][c] == pairs
        # schedules of the rank plan satisfy the same invariants as a full plan's
        from test_plan import _check_schedules
        _check_schedules(r, mine, n, nchunks, block, block, is_rank=True)
    assert total_pairs == oracle.unmasked_pairs(cu)


@pytest.mark.parametrize("seed", range(4))
def test_rank_plans_random(seed):
    rng = np.random.default_rng(100 + seed)
    n = 128 * int(rng.integers(8, 20)) - int(rng.integers(0, 100))
    lens = []
    while sum(lens) < n:
        lens.append(int(min(n - sum(lens), rng.integers(1, 900))))
    cu = workloads.cu_seqlens_from_lengths(lens)
    for nchunks in (2, 3, 5):
        _check_rank_plans(cu, n, sap.sap_balanced_chunks(cu, n, nchunks))
    T = (n + 127) // 128
    _check_rank_plans(cu, n, [0, 128 * (T // 2), n])


def test_rank_plans_128k_workload():
    w = workloads.WORKLOADS["llama31_8b_128k"]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    bounds = sap.sap_balanced_chunks(cu, w.n, 8)
    full = sap.sap_plan_chunks(cu, w.n, bounds)
    items = sap.sap_plan_items(full)
    for c in range(8):
        r = sap.sap_plan_rank(full, c)
        np.testing.assert_array_equal(sap.sap_plan_items(r), items[items[:, 2] == c])
    with pytest.raises(sap.SapError):
        sap.sap_plan_rank(full, 8)
    with pytest.raises(sap.SapError):
        sap.sap_plan_rank(sap.sap_plan_rank(full, 1), 0)  # no rank plan of a rank plan

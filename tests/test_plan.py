"""Host planner (libsap.so, no GPU needed): bit-exact tile list against the
oracle, schedule invariants, statistics and argument errors."""
import numpy as np
import pytest

import oracle
import packed_sequence_causal_b200 as sap
import workloads


def _plan_and_check(cu, n, nchunks, bm=128, bn=128):
    plan = sap.sap_plan(cu, n, nchunks, bm, bn)
    items = sap.sap_plan_items(plan)
    ref = oracle.tile_list(cu, n, nchunks, bm, bn)
    np.testing.assert_array_equal(items, ref)
    st = sap.sap_plan_stats(plan)
    assert st["unmasked_pairs"] == oracle.unmasked_pairs(cu)
    assert st["n_chunk_pairs"] == len({(int(a), int(b)) for a, b in ref[:, 2:4]}) if len(ref) else True
    _check_schedules(plan, items, n, nchunks, bm, bn)
    return plan, items


def _check_schedules(plan, items, n, nchunks, bm, bn, is_rank=False):
    units, order, merges = sap.sap_plan_fwd_schedule(plan)
    # units tile the item list contiguously, one (q-tile, kv-chunk) each
    pos = 0
    slots_of_tile = {}
    for qt, b, c, slot in units:
        assert b == pos and c > 0
        run = items[b:b + c]
        assert np.all(run[:, 0] == qt) and len(set(run[:, 3].tolist())) == 1
        pos += c
        slots_of_tile.setdefault(int(qt), []).append(int(slot))
    assert pos == len(items)
    # a q-tile with several units gets consecutive partial slots; one unit writes directly
    mi = 0
    next_slot = 0
    for qt in sorted(slots_of_tile):
        s = slots_of_tile[qt]
        if len(s) == 1:
            assert s == [-1]
        else:
            assert s == list(range(next_slot, next_slot + len(s)))
            assert tuple(merges[mi]) == (qt, next_slot, len(s))
            next_slot += len(s)
            mi += 1
    assert mi == len(merges)
    assert sap.sap_plan_stats(plan)["n_partial_slots"] == next_slot
    # heavy-first order: a permutation, non-increasing item counts; among equal counts the kv chunk
    # of the unit's items ascending, then the unit index.  A rank plan lists its own-chunk units
    # first (units whose items all have kv_chunk = the plan's chunk) and keeps that order in each part.
    assert sorted(order.tolist()) == list(range(len(units)))
    n_local, n_units = sap.sap_plan_fwd_local_units(plan)
    assert n_units == len(units)
    rank = sap.sap_plan_window(plan)
    own = None
    if rank["q_end"] - rank["q_begin"] < n or rank["kv_begin"] > 0:
        own = int(items[0, 2]) if len(items) else None
    if own is not None:
        for i, u in enumerate(order):
            is_local = bool(np.all(items[units[u, 1]:units[u, 1] + units[u, 2], 3] == own))
            assert is_local == (i < n_local)
    else:
        assert n_local == n_units
    chunk = {u: items[units[u, 1]][3] for u in range(len(units))}
    for part in (order[:n_local], order[n_local:]):
        assert np.all(np.diff(units[part, 2]) <= 0)
        for a, b in zip(part[:-1], part[1:]):
            if units[a, 2] == units[b, 2]:
                assert (chunk[a], a) < (chunk[b], b)
    # backward: every item once; a kv tile's q-descending list of at most 16 q tiles is one unit,
    # a longer list is cut into the parts that fall in one band of 16 q tiles; units band-major
    # (top band first, a unit's band is that of its top q tile), heavy-first within a band, ties by
    # kv tile
    kv_units, entries = sap.sap_plan_bwd_schedule(plan)
    band = 16
    list_len = np.bincount(items[:, 1], minlength=int(items[:, 1].max()) + 1 if len(items) else 0)
    seen = set()
    covered = np.zeros(len(entries), dtype=np.int64)
    prev = None
    for kt, e0, ne in kv_units:
        assert ne > 0
        grp = entries[e0:e0 + ne]
        assert np.all(np.diff(grp[:, 0]) < 0)
        if list_len[kt] <= band:
            assert ne == list_len[kt]
        else:
            assert len(set((grp[:, 0] // band).tolist())) == 1
        covered[e0:e0 + ne] += 1
        for qt, tag in grp:
            seen.add((int(qt), int(kt), int(tag)))
        key = (int(grp[0, 0]) // band, int(ne), int(kt))
        if prev is not None:
            assert key[0] < prev[0] or (key[0] == prev[0] and (key[1] < prev[1] or
                                                               (key[1] == prev[1] and key[2] > prev[2])))
        prev = key
    assert np.all(covered == 1)
    assert len(seen) == len(entries)
    # units of one kv tile do not share a band (each band piece is maximal)
    pieces = {(int(kt), int(entries[e0, 0]) // band) for kt, e0, _ in kv_units}
    assert len(pieces) == len(kv_units)
    # direct dK/dV stores: exactly the kv tiles of a single unit, in full plans only
    direct = sap.sap_plan_bwd_direct(plan)
    win = sap.sap_plan_window(plan)
    n_units_of = np.bincount(kv_units[:, 0], minlength=len(list_len)) if len(kv_units) else np.zeros(0, int)
    kt0 = win["kv_begin"] // bn
    expect = np.zeros((win["q_end"] - win["kv_begin"] + bn - 1) // bn, dtype=np.int32)
    if not is_rank:
        for l in range(len(expect)):
            expect[l] = int(kt0 + l < len(n_units_of) and n_units_of[kt0 + l] == 1)
    np.testing.assert_array_equal(direct, expect)
    assert seen == {(int(a), int(b), int(t)) for a, b, _, _, t in items}


@pytest.mark.parametrize("name", ["tiny", "llama32_1b_32k", "llama31_8b_128k", "llama2_13b_64k_short"])
def test_planner_matches_oracle_on_workloads(name):
    w = workloads.WORKLOADS[name]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    _plan_and_check(cu, w.n, w.p)


def test_planner_matches_oracle_512k():
    w = workloads.WORKLOADS["hybrid_512k"]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    _plan_and_check(cu, w.n, w.p)


@pytest.mark.parametrize("seed", range(20))
def test_planner_matches_oracle_random(seed):
    rng = np.random.default_rng(100 + seed)
    bm = int(rng.choice([16, 32, 128]))
    nchunks = int(rng.choice([1, 2, 4, 8]))
    n = bm * nchunks * int(rng.integers(1, 8))
    lens = []
    while sum(lens) < n:
        lens.append(int(min(n - sum(lens), rng.integers(1, 4 * bm))))
        if rng.random() < 0.1:
            lens.append(0)
    _plan_and_check(workloads.cu_seqlens_from_lengths(lens), n, nchunks, bm, bm)


@pytest.mark.parametrize("n", [1, 5, 127, 129, 300, 1000])
def test_planner_ragged_single_chunk(n):
    lens = [max(1, n // 4), n - max(1, n // 4)] if n > 1 else [1]
    _plan_and_check(workloads.cu_seqlens_from_lengths(lens), n, 1)


def test_planner_rectangular_tiles():
    cu = workloads.cu_seqlens_from_lengths([100, 28, 200, 56])
    _plan_and_check(cu, 384, 3, 32, 64)


def test_planner_empty_batch():
    plan = sap.sap_plan([0], 0, 1)
    assert len(sap.sap_plan_items(plan)) == 0
    assert sap.sap_plan_stats(plan)["unmasked_pairs"] == 0


def test_planner_single_token_docs_only_diagonal():
    n = 512
    plan, items = _plan_and_check(np.arange(n + 1, dtype=np.int32), n, 4)
    assert len(items) == n // 128 and np.all(items[:, 0] == items[:, 1])


def test_planner_errors():
    with pytest.raises(sap.SapError) as e:
        sap.sap_plan([0, 10, 9, 20], 20, 1)
    assert e.value.status == -2
    with pytest.raises(sap.SapError) as e:
        sap.sap_plan([1, 20], 20, 1)
    assert e.value.status == -2
    with pytest.raises(sap.SapError) as e:
        sap.sap_plan([0, 20], 21, 1)
    assert e.value.status == -2
    with pytest.raises(sap.SapError) as e:
        sap.sap_plan([0, 300], 300, 3)       # chunk 100 not a multiple of 128
    assert e.value.status == -3
    with pytest.raises(sap.SapError) as e:
        sap.sap_plan([0, 512], 512, 0)
    assert e.value.status == -3
    with pytest.raises(sap.SapError) as e:
        sap.sap_plan([0, 512], 512, 3)       # N not divisible by P
    assert e.value.status == -3
    with pytest.raises(sap.SapError) as e:
        sap.sap_plan([0, 512], 512, 1, 0, 128)
    assert e.value.status == -1


def test_workspace_sizes_and_head_checks():
    w = workloads.WORKLOADS["tiny"]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    plan = sap.sap_plan(cu, w.n, w.p)
    slots = sap.sap_plan_stats(plan)["n_partial_slots"]
    fwd = sap.sap_workspace_size(plan, 4, 4, 64, sap.SAP_WS_FWD)
    assert fwd >= slots * 4 * 128 * (64 + 1) * 4
    bwd = sap.sap_workspace_size(plan, 4, 4, 64, sap.SAP_WS_BWD)
    assert bwd >= 1024 * 4 * 64 * 4 + 2 * 4 * 1024 * 4
    with pytest.raises(sap.SapError) as e:
        sap.sap_workspace_size(plan, 6, 4, 64, sap.SAP_WS_FWD)   # hq % hkv != 0
    assert e.value.status == -1
    with pytest.raises(sap.SapError) as e:
        sap.sap_workspace_size(plan, 4, 4, 96, sap.SAP_WS_FWD)   # unsupported head_dim
    assert e.value.status == -7


@pytest.mark.parametrize("name", ["tiny", "llama31_8b_128k"])
def test_fused_merge_schedule(name):
    """Fused-merge mode: one forward unit per q-tile covering all its items, no slots, no merges;
    switching back restores the chunked schedule exactly."""
    w = workloads.WORKLOADS[name]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    plan = sap.sap_plan(cu, w.n, w.p)
    items = sap.sap_plan_items(plan)
    chunked = sap.sap_plan_fwd_schedule(plan)
    sap.sap_plan_set_fused_merge(plan, True)
    units, order, merges = sap.sap_plan_fwd_schedule(plan)
    qts = np.unique(items[:, 0])
    assert len(units) == len(qts) and len(merges) == 0
    assert np.all(units[:, 3] == -1) and sap.sap_plan_stats(plan)["n_partial_slots"] == 0
    pos = 0
    for qt, b, c, _ in units:
        assert b == pos and np.all(items[b:b + c, 0] == qt) and (b + c == len(items) or items[b + c, 0] != qt)
        pos += c
    assert pos == len(items)
    assert sorted(order.tolist()) == list(range(len(units)))
    assert sap.sap_workspace_size(plan, w.hq, w.hkv, w.d, sap.SAP_WS_FWD) == 256  # the work counter only
    sap.sap_plan_set_fused_merge(plan, False)
    for a, b in zip(chunked, sap.sap_plan_fwd_schedule(plan)):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("tiles", [15, 16, 17, 33])
def test_backward_units_at_the_band_limit(tiles):
    """One document of `tiles` q tiles: kv tile 0's list has `tiles` entries.  Up to 16 entries it
    is one backward unit (and, in a full plan, its dK/dV are stored directly); 17 or more are cut at
    the 16-tile band boundaries into one unit per band, accumulated in fp32."""
    n = 128 * tiles
    plan = sap.sap_plan([0, n], n, 1)
    kv_units, entries = sap.sap_plan_bwd_schedule(plan)
    direct = sap.sap_plan_bwd_direct(plan)
    for kt in range(tiles):
        mine = kv_units[kv_units[:, 0] == kt]
        list_len = tiles - kt  # q tiles kt .. tiles - 1
        assert mine[:, 2].sum() == list_len
        if list_len <= 16:
            assert len(mine) == 1 and direct[kt] == 1
        else:
            bands = {int(q) // 16 for q in range(kt, tiles)}
            assert len(mine) == len(bands) and direct[kt] == 0
            for _, e0, ne in mine:
                qs = entries[e0:e0 + ne, 0]
                assert len({int(q) // 16 for q in qs}) == 1

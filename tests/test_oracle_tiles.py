"""Pins of the oracle's tile list (CPU only).

The tile list is checked against brute force on every (i, j) pair: each
unmasked pair of the packed causal mask lies in exactly one emitted item, no
emitted item is empty, and each tag says what the kernels rely on (FULL: no
pair of the box is masked; CAUSAL: inside the box the mask is exactly j <= i;
MASKED: neither), in both directions: a diagonal box that holds exactly the
causal pattern is tagged CAUSAL, not MASKED.  The interval-based and exhaustive evaluations must agree.
"""
import numpy as np
import pytest

import oracle
import workloads


def _dense_mask(cu, n):
    doc = np.zeros(n, dtype=np.int64)
    for k, (s, e) in enumerate(zip(cu[:-1], cu[1:])):
        doc[s:e] = k
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    return (doc[:, None] == doc[None, :]) & (j <= i)


def _check_against_mask(cu, n, nchunks, bm, bn):
    items = oracle.tile_list(cu, n, nchunks, bm, bn)
    mask = _dense_mask(cu, n)
    covered = np.zeros_like(mask, dtype=np.int64)
    chunk = n // nchunks if nchunks > 1 else n
    prev = (-1, -1)
    for qt, kt, qc, kc, tag in items:
        assert (qt, kt) > prev  # canonical order, no duplicates
        prev = (qt, kt)
        i0, j0 = qt * bm, kt * bn
        box = np.zeros((bm, bn), dtype=bool)
        sub = mask[i0:i0 + bm, j0:j0 + bn]
        box[: sub.shape[0], : sub.shape[1]] = sub
        assert box.any()
        covered[i0:i0 + bm, j0:j0 + bn] += 1
        assert qc == i0 // chunk and kc == j0 // chunk
        ii = np.arange(bm)[:, None] + i0
        jj = np.arange(bn)[None, :] + j0
        causal_box = qt * bm == kt * bn and bm == bn and np.array_equal(box, (jj <= ii) & (ii < n))
        if tag == oracle.TAG_FULL:
            assert box.all()
        elif tag == oracle.TAG_CAUSAL:
            assert qt == kt and bm == bn
            assert causal_box
        else:
            assert tag == oracle.TAG_MASKED and not box.all()
        # converse: a box that is not fully unmasked but holds exactly the causal pattern of its
        # diagonal (one document covers every real row of the tile) must be tagged CAUSAL
        if causal_box and not box.all():
            assert tag == oracle.TAG_CAUSAL, (qt, kt, tag)
    assert np.all(covered[mask] == 1)
    assert int(mask.sum()) == oracle.unmasked_pairs(cu)
    ex = oracle.tile_list(cu, n, nchunks, bm, bn, exhaustive=True)
    np.testing.assert_array_equal(items, ex)
    return items


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("bm", [8, 16])
def test_tile_list_random(seed, bm):
    rng = np.random.default_rng(seed)
    nchunks = int(rng.choice([1, 2, 4]))
    n = bm * nchunks * int(rng.integers(1, 6))
    lens = []
    while sum(lens) < n:
        lens.append(int(min(n - sum(lens), rng.integers(1, 3 * bm))))
    if seed % 3 == 0:
        lens.insert(1, 0)  # an empty document
    cu = workloads.cu_seqlens_from_lengths(lens)
    _check_against_mask(cu, n, nchunks, bm, bm)


@pytest.mark.parametrize("n", [1, 7, 16, 37, 100])
def test_tile_list_ragged_single_chunk(n):
    """N not a multiple of the tile: the partial last tile is never FULL."""
    lens = [n // 3, n - n // 3] if n > 2 else [n]
    cu = workloads.cu_seqlens_from_lengths(lens)
    items = _check_against_mask(cu, n, 1, 16, 16)
    last = (n - 1) // 16
    for qt, kt, _, _, tag in items:
        if qt == last and n % 16:
            assert tag != oracle.TAG_FULL


def test_tile_list_rectangular_tiles():
    cu = workloads.cu_seqlens_from_lengths([20, 5, 39])
    _check_against_mask(cu, 64, 2, 16, 8)


def test_tile_list_empty_batch():
    assert len(oracle.tile_list([0], 0, 1)) == 0


def test_tile_list_tiny_workload():
    """The 1024-token, 4-document workload with 2 chunks (seed 0)."""
    b = workloads.make_batch("tiny", 0)
    items = _check_against_mask(b.cu_seqlens, 1024, 2, 128, 128)
    assert len(items) == 21


def test_tile_list_diagonal_tiles_of_one_document_are_causal():
    """One document over five 16-token tiles: every diagonal tile is CAUSAL and every tile below
    the diagonal FULL.  With N = 100 (ragged last tile, two documents) the partial last diagonal
    tile lies inside the second document and is CAUSAL too."""
    items = _check_against_mask(workloads.cu_seqlens_from_lengths([80]), 80, 1, 16, 16)
    for qt, kt, _, _, tag in items:
        assert tag == (oracle.TAG_CAUSAL if qt == kt else oracle.TAG_FULL)
    assert len(items) == 15
    items = _check_against_mask(workloads.cu_seqlens_from_lengths([33, 67]), 100, 1, 16, 16)
    tags = {(int(qt), int(kt)): int(tag) for qt, kt, _, _, tag in items}
    assert tags[(6, 6)] == oracle.TAG_CAUSAL
    assert tags[(2, 2)] == oracle.TAG_MASKED  # tokens 32 | 33..47: a document boundary inside the tile

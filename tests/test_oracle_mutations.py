"""Mutation tests of the oracle's pins (CPU only).

Each case copies oracle/oracle.c, plants one plausible mistake (a dropped
term, a wrong sign or index, an off-by-one, a wrong weight or tag), builds the
mutant in a temporary directory and checks that the pins used in
test_oracle_pins.py / test_oracle_tiles.py reject it.  The committed oracle is
never modified.
"""
import importlib.util
import math
import os
import shutil

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")


def _mutant(tmp_path, name, old, new):
    src = open(os.path.join(ORACLE_DIR, "oracle.c")).read()
    assert src.count(old) == 1, f"mutation site not unique: {old!r}"
    d = tmp_path / name
    d.mkdir()
    (d / "oracle.c").write_text(src.replace(old, new))
    shutil.copy(os.path.join(ORACLE_DIR, "__init__.py"), d / "__init__.py")
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{name}", d / "__init__.py",
                                                  submodule_search_locations=[str(d)])
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _fwd_matches_library(mod):
    b = workloads.custom_batch([5, 1, 9, 3], 4, 2, 8, seed=0)
    scale = 1.0 / math.sqrt(8)
    o, _ = mod.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    outs = []
    for s, e in zip(b.cu_seqlens[:-1], b.cu_seqlens[1:]):
        qs, ks, vs = (t[s:e].double().permute(1, 0, 2).unsqueeze(0) for t in (b.q, b.k, b.v))
        outs.append(F.scaled_dot_product_attention(qs, ks, vs, is_causal=True, scale=scale, enable_gqa=True)
                    .squeeze(0).permute(1, 0, 2))
    return np.allclose(o, torch.cat(outs).numpy(), atol=1e-12, rtol=0)


def _bwd_matches_autograd(mod):
    b = workloads.custom_batch([7, 2, 6], 4, 2, 8, seed=1)
    scale = 0.3
    dq, dk, dv = mod.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    q, k, v = (t.double().clone().requires_grad_(True) for t in (b.q, b.k, b.v))
    outs = []
    for s, e in zip(b.cu_seqlens[:-1], b.cu_seqlens[1:]):
        qs, ks, vs = (t[s:e].permute(1, 0, 2).unsqueeze(0) for t in (q, k, v))
        outs.append(F.scaled_dot_product_attention(qs, ks, vs, is_causal=True, scale=scale, enable_gqa=True)
                    .squeeze(0).permute(1, 0, 2))
    (torch.cat(outs) * b.do.double()).sum().backward()
    return all(np.allclose(a, r.grad.numpy(), atol=1e-11, rtol=0) for a, r in ((dq, q), (dk, k), (dv, v)))


def _chunked_equals_plain(mod):
    b = workloads.custom_batch([40, 3, 70, 15], 2, 1, 16, seed=2)
    o, lse = mod.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, 0.25)
    oc, lc, _, _ = mod.attn_fwd_chunked(b.q, b.k, b.v, b.cu_seqlens, 0.25, 4)
    return np.allclose(oc, o, atol=1e-12) and np.allclose(lc, lse, atol=1e-12)


def _tiles_match_brute_force(mod):
    cu = workloads.cu_seqlens_from_lengths([20, 5, 39])
    n, bm = 64, 16
    items = mod.tile_list(cu, n, 2, bm, bm, exhaustive=True)
    doc = np.repeat(np.arange(3), np.diff(cu))
    i, j = np.arange(n)[:, None], np.arange(n)[None, :]
    mask = (doc[:, None] == doc[None, :]) & (j <= i)
    for qt, kt, _, _, tag in items:
        box = mask[qt * bm:(qt + 1) * bm, kt * bm:(kt + 1) * bm]
        if tag == 0 and not box.all():
            return False
    covered = np.zeros_like(mask)
    for qt, kt, *_ in items:
        covered[qt * bm:(qt + 1) * bm, kt * bm:(kt + 1) * bm] = True
    return bool(np.all(covered[mask]))


def _tags_match_brute_force(mod):
    """Every tag against the dense mask, in both directions: FULL iff the box is fully unmasked,
    CAUSAL iff (otherwise) it is a diagonal box holding exactly the pattern j <= i."""
    cu = workloads.cu_seqlens_from_lengths([20, 5, 39, 16, 21])
    n, bm = 101, 16
    items = mod.tile_list(cu, n, 1, bm, bm)
    doc = np.repeat(np.arange(len(cu) - 1), np.diff(cu))
    i, j = np.arange(n)[:, None], np.arange(n)[None, :]
    mask = (doc[:, None] == doc[None, :]) & (j <= i)
    for qt, kt, _, _, tag in items:
        box = np.zeros((bm, bm), dtype=bool)
        sub = mask[qt * bm:(qt + 1) * bm, kt * bm:(kt + 1) * bm]
        box[: sub.shape[0], : sub.shape[1]] = sub
        ii = np.arange(bm)[:, None] + qt * bm
        jj = np.arange(bm)[None, :] + kt * bm
        causal = qt == kt and np.array_equal(box, (jj <= ii) & (ii < n))
        want = 0 if box.all() else (1 if causal else 2)
        if tag != want:
            return False
    return True


MUTATIONS = [
    ("no_diagonal", "int64_t hi = i < kv_hi - 1 ? i : kv_hi - 1;",
     "int64_t hi = (i - 1) < kv_hi - 1 ? (i - 1) : kv_hi - 1;", _fwd_matches_library),
    ("gqa_map", "int32_t g = h / (hq / hkv);", "int32_t g = h % hkv;", _fwd_matches_library),
    ("no_max_shift", "for (int64_t j = lo; j <= hi; ++j) sum += exp(s[j - lo] - m);",
     "for (int64_t j = lo; j <= hi; ++j) sum += exp(s[j - lo]);", _fwd_matches_library),
    ("dq_without_scale", "dqi[c] += scale * ds * kj[c];", "dqi[c] += ds * kj[c];", _bwd_matches_autograd),
    ("ds_sign", "double ds = p * (dp - Di);", "double ds = p * (dp + Di);", _bwd_matches_autograd),
    ("merge_weight", "double w = exp(lse_parts[((size_t)b * hq + h) * n + i] - l_all);",
     "double w = exp(lse_parts[((size_t)b * hq + h) * n + i] - m);", _chunked_equals_plain),
    ("full_tag", "if (all)\n        tag = 0;", "if (any)\n        tag = 0;", _tiles_match_brute_force),
    ("causal_tag_dropped", "        tag = 1;\n", "        tag = 2;\n", _tags_match_brute_force),
]


def test_unmutated_oracle_passes_every_check():
    import oracle
    for check in (_fwd_matches_library, _bwd_matches_autograd, _chunked_equals_plain, _tiles_match_brute_force,
                  _tags_match_brute_force):
        assert check(oracle), check.__name__


@pytest.mark.parametrize("name,old,new,check", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_reject_planted_mistake(tmp_path, name, old, new, check):
    mod = _mutant(tmp_path, name, old, new)
    assert not check(mod), f"the pin did not notice the planted mistake '{name}'"
